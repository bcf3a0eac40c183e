// lq_perstep.cuh -- entering and reading back the naive per-step baselines:
// a dense state stored in BF16, or in FP8 E4M3 with one FP32 scale per value
// column (the BF16 and FP8 rows of the accuracy table of the news post
// "Linear attention has to move state every token it generates; LeapQuant
// compresses it to 8-bit without losing accuracy": quantizing at every step
// lets the rounding error compound, which LeapQuant's per-window scheme
// avoids).  The decode step of these formats is dense_step_kernel
// (lq_dense.cuh), which rounds the same way:
//  * BF16: each entry rounded to bfloat16, ties to even;
//  * FP8: scale_j = fl32(max_i |S_ij| / 448), code = E4M3(fl32(S_ij /
//    scale_j)) with ties to even and saturation at 448 (an all-zero column:
//    scale 0, codes 0); the value read back is fl32(E4M3 value * scale_j).
// One CTA of 128 threads per (slot, head) and block of 64 value columns;
// thread t owns rows TI*(t%16).. (TI = D/16) of columns 8*(t/16).. of the
// block.  MODE 1 stores a caller's FP32 state (entering a sequence), MODE 2
// writes the dense FP32 values back out.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "lq_fp32.cuh"

namespace lq {

constexpr int kPsCols = 64;  // value columns per CTA
constexpr int kPsCpt = 8;    // value columns per thread

// e4m3 code -> its value (exact in FP32)
__device__ __forceinline__ float e4m3_value(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)(code & 0xFFu), __NV_E4M3);
    return __half2float(__half(h));
}

template <int D, int FMT, int MODE>
__global__ void __launch_bounds__(kFp32Threads) perstep_kernel(Fp32Args A) {
    constexpr int TI = D / 16, NB = D / kPsCols, CPT = kPsCpt;
    static_assert(FMT == 16 || FMT == 8, "BF16 or FP8 state");
    static_assert(MODE == 1 || MODE == 2, "init or read-back");
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x;
    const int ic = tid & 15, jc = tid >> 4, i0 = TI * ic;
    const size_t head = blockIdx.x / NB;
    const int cb = blockIdx.x % NB, j0 = kPsCols * cb + CPT * jc;
    const Layout &L = A.L;
    uint8_t *blob = A.state + head * L.blob;

    __shared__ float s_pk[16][kPsCols], s_sc[kPsCols];

    // ---- the current state in FP32
    float Sd[TI][CPT];
    if constexpr (MODE == 1) {
#pragma unroll
        for (int ii = 0; ii < TI; ++ii) {
            const float *row = A.S0 + head * (size_t)D * D + (size_t)(i0 + ii) * D + j0;
            const float4 a4 = *reinterpret_cast<const float4 *>(row);
            const float4 b4 = *reinterpret_cast<const float4 *>(row + 4);
            Sd[ii][0] = a4.x; Sd[ii][1] = a4.y; Sd[ii][2] = a4.z; Sd[ii][3] = a4.w;
            Sd[ii][4] = b4.x; Sd[ii][5] = b4.y; Sd[ii][6] = b4.z; Sd[ii][7] = b4.w;
        }
    } else {
        if constexpr (FMT == 16) {
            const uint16_t *Sb = reinterpret_cast<const uint16_t *>(blob + L.codes_off);
#pragma unroll
            for (int ii = 0; ii < TI; ++ii) {
                const uint4 w4 = *reinterpret_cast<const uint4 *>(Sb + (size_t)(i0 + ii) * D + j0);
                const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    Sd[ii][2 * x] = __uint_as_float(w[x] << 16);
                    Sd[ii][2 * x + 1] = __uint_as_float(w[x] & 0xFFFF0000u);
                }
            }
        } else {
            const float4 sa = *reinterpret_cast<const float4 *>(blob + L.qs_off + 4 * j0);
            const float4 sb = *reinterpret_cast<const float4 *>(blob + L.qs_off + 4 * j0 + 16);
            const float sc[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
            const uint8_t *C = blob + L.codes_off;
#pragma unroll
            for (int ii = 0; ii < TI; ++ii) {
                const uint2 w = *reinterpret_cast<const uint2 *>(C + (size_t)(i0 + ii) * D + j0);
#pragma unroll
                for (int jj = 0; jj < CPT; ++jj)
                    Sd[ii][jj] = __fmul_rn(e4m3_value((jj < 4 ? w.x : w.y) >> (8 * (jj & 3))), sc[jj]);
            }
        }
    }
    if constexpr (MODE == 2) {
        float *So = A.S_out + head * (size_t)D * D;
#pragma unroll
        for (int ii = 0; ii < TI; ++ii) {
            float *row = So + (size_t)(i0 + ii) * D + j0;
            *reinterpret_cast<float4 *>(row) = make_float4(Sd[ii][0], Sd[ii][1], Sd[ii][2], Sd[ii][3]);
            *reinterpret_cast<float4 *>(row + 4) = make_float4(Sd[ii][4], Sd[ii][5], Sd[ii][6], Sd[ii][7]);
        }
        return;
    }

    // ---- store the new FP32 values in the narrow format
    if constexpr (FMT == 16) {
        uint16_t *Sb = reinterpret_cast<uint16_t *>(blob + L.codes_off);
#pragma unroll
        for (int ii = 0; ii < TI; ++ii) {
            uint32_t w[4];
#pragma unroll
            for (int x = 0; x < 4; ++x)
                w[x] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(Sd[ii][2 * x])) |
                       ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(Sd[ii][2 * x + 1])) << 16);
            *reinterpret_cast<uint4 *>(Sb + (size_t)(i0 + ii) * D + j0) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else {
        // column maxima of the block (the partial-sum arrays are free here)
#pragma unroll
        for (int jj = 0; jj < CPT; ++jj) {
            float m = 0.f;
#pragma unroll
            for (int ii = 0; ii < TI; ++ii) m = fmaxf(m, fabsf(Sd[ii][jj]));
            s_pk[ic][CPT * jc + jj] = m;
        }
        __syncthreads();
        if (tid < kPsCols) {
            float m = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) m = fmaxf(m, s_pk[r][tid]);
            const float sc = __fdiv_rn(m, 448.f);
            s_sc[tid] = sc;
            reinterpret_cast<float *>(blob + L.qs_off)[kPsCols * cb + tid] = sc;
        }
        __syncthreads();
        uint8_t *C = blob + L.codes_off;
#pragma unroll
        for (int ii = 0; ii < TI; ++ii) {
            uint32_t w[2] = {0u, 0u};
#pragma unroll
            for (int jj = 0; jj < CPT; ++jj) {
                const float sc = s_sc[CPT * jc + jj];
                const uint32_t code =
                    sc == 0.f ? 0u
                              : (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(Sd[ii][jj], sc), __NV_SATFINITE, __NV_E4M3);
                w[jj >> 2] |= (code & 0xFFu) << (8 * (jj & 3));
            }
            *reinterpret_cast<uint2 *>(C + (size_t)(i0 + ii) * D + j0) = make_uint2(w[0], w[1]);
        }
    }
    if (MODE == 1 && cb == 0 && tid == 0) {
        uint32_t *h = reinterpret_cast<uint32_t *>(blob);
        h[0] = 0u;
        h[1] = 0u;
        h[2] = 0u;
        h[3] = kMagic;
        *reinterpret_cast<float *>(blob + kHdrG) = 1.f;
    }
}

}  // namespace lq
