// lq_perstep.cuh -- the naive per-step baselines: a dense state stored in
// BF16, or in FP8 E4M3 with one FP32 scale per value column, rounded again
// after every token.  These are the comparison points of the accuracy table
// of the news post "Linear attention has to move state every token it
// generates; LeapQuant compresses it to 8-bit without losing accuracy" (its
// BF16 and FP8 rows): quantizing at every step lets the rounding error
// compound, which LeapQuant's per-window scheme avoids.
//
// Same decomposition as the FP32-state kernel: the update separates by value
// column, so one CTA of 128 threads takes one (slot, head) and a block of 64
// value columns; thread t owns rows TI*(t%16).. (TI = D/16) of columns
// 8*(t/16).. of the block (16-byte BF16 / 8-byte FP8 row segments).  The state is read and converted to FP32, the FP32
// delta-rule step runs as in that kernel, and the new FP32 values are stored
// back in the narrow format:
//  * BF16: each entry rounded to bfloat16, ties to even;
//  * FP8: the column maxima meet in shared memory, scale_j =
//    fl32(max_i |S_ij| / 448), code = E4M3(fl32(S_ij / scale_j)) with ties to
//    even and saturation at 448 (an all-zero column: scale 0, codes 0); the
//    value read back is fl32(E4M3 value * scale_j).
// MODE 0 is the decode step, MODE 1 stores a caller's FP32 state (entering a
// sequence), MODE 2 writes the dense FP32 values back out.
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
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ic = tid & 15, jc = tid >> 4, i0 = TI * ic;
    const size_t head = blockIdx.x / NB;
    const int cb = blockIdx.x % NB, j0 = kPsCols * cb + CPT * jc;
    const Flags &F = A.F;
    const Layout &L = A.L;
    uint8_t *blob = A.state + head * L.blob;

    __shared__ float s_pk[16][kPsCols], s_pq[16][kPsCols], s_u[kPsCols], s_sc[kPsCols];
    __shared__ float s_kq[kFp32Threads / 32];

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
        if constexpr (MODE == 0) {
            const uint4 hdr = *reinterpret_cast<const uint4 *>(blob);
            if (!(hdr.w == kMagic && hdr.y == 0)) {
                if (tid < kPsCols) A.out[head * D + kPsCols * cb + tid] = 0.f;
                if (hdr.w != kMagic && hdr.y == 0 && cb == 0 && tid == 0) set_status(blob, LQ_DEV_CORRUPT);
                return;
            }
        }
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

    // ---- MODE 0: the FP32 delta-rule step (as in the FP32-state kernel)
    if constexpr (MODE == 0) {
        float kr[TI], qr[TI];
#pragma unroll
        for (int ii = 0; ii < TI; ++ii) {
            const size_t o = head * D + i0 + ii;
            kr[ii] = load_in(A.k, o, F.bf16_in);
            qr[ii] = load_in(A.q, o, F.bf16_in);
            const float a = F.kda ? A.decay[o] : A.decay[head];
#pragma unroll
            for (int jj = 0; jj < CPT; ++jj) Sd[ii][jj] = a * Sd[ii][jj];
        }
        float kq = 0.f;
        if (tid < D) {
            const size_t o = head * D + tid;
            kq = load_in(A.k, o, F.bf16_in) * load_in(A.q, o, F.bf16_in);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) kq += __shfl_xor_sync(0xFFFFFFFFu, kq, off);
        if (lane == 0) s_kq[warp] = kq;
        float pk[CPT], pq[CPT];
#pragma unroll
        for (int jj = 0; jj < CPT; ++jj) pk[jj] = pq[jj] = 0.f;
#pragma unroll
        for (int ii = 0; ii < TI; ++ii)
#pragma unroll
            for (int jj = 0; jj < CPT; ++jj) {
                pk[jj] = fmaf(Sd[ii][jj], kr[ii], pk[jj]);
                pq[jj] = fmaf(Sd[ii][jj], qr[ii], pq[jj]);
            }
#pragma unroll
        for (int jj = 0; jj < CPT; ++jj) {
            s_pk[ic][CPT * jc + jj] = pk[jj];
            s_pq[ic][CPT * jc + jj] = pq[jj];
        }
        __syncthreads();
        if (tid < kPsCols) {
            float a = 0.f, b = 0.f, kq_all = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                a += s_pk[r][tid];
                b += s_pq[r][tid];
            }
#pragma unroll
            for (int w = 0; w < kFp32Threads / 32; ++w) kq_all += s_kq[w];
            const size_t o = head * D + kPsCols * cb + tid;
            const float u = A.beta[head] * (load_in(A.v, o, F.bf16_in) - a);
            s_u[tid] = u;
            A.out[o] = fmaf(kq_all, u, b);
        }
        __syncthreads();
        float uu[CPT];
#pragma unroll
        for (int jj = 0; jj < CPT; ++jj) uu[jj] = s_u[CPT * jc + jj];
#pragma unroll
        for (int ii = 0; ii < TI; ++ii)
#pragma unroll
            for (int jj = 0; jj < CPT; ++jj) Sd[ii][jj] = fmaf(kr[ii], uu[jj], Sd[ii][jj]);
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
