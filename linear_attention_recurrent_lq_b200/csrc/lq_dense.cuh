// lq_dense.cuh -- one decode token of a dense recurrent state stored in FP32
// (the reference path, bits = 32) or in a narrow per-step format (the naive
// baselines of the accuracy table: BF16, or FP8 E4M3 with one FP32 scale per
// value column), on sm_100a.
//
// Every token reads the whole dk x dv state of each head from HBM, updates it
// and writes it back: the cost LeapQuant removes (news post "Linear attention
// has to move state every token it generates; LeapQuant compresses it to
// 8-bit without losing accuracy", second paragraph; the BF16 and FP8 rows of
// its accuracy table store the state again after every token).  The step is
// the delta rule
//     S' = D_t S,  u = beta (v - S'^T k),  S_new = S' + k u^T,
//     o = S_new^T q = S'^T q + (k . q) u,
// so one pass over S' gives both column sums S'^T k and S'^T q.
//
// The kernel is bound by HBM traffic (read and write the state once each), so
// it is built to keep the copy engine busy:
//  * persistent, one CTA per SM, walking the heads b, b + G, ...;
//  * a ring of bulk-copy stages (cp.async.bulk, mbarrier completion, no
//    multicast) holds the blob prefix (header + stored state) and the token's
//    q, k, v (and KDA decay) of the next heads while the current one is
//    computed; thread 0 refills a stage as soon as every thread has taken its
//    entries into registers;
//  * a thread owns RPT consecutive key rows x 4 value columns; a warp reads a
//    whole row segment per instruction, so shared loads are conflict-free;
//  * the new state goes from registers straight to global memory (16-byte
//    streaming stores for FP32 and BF16; 4-byte stores for FP8 codes).
// The FP32 arithmetic is the same for every format: the narrow formats only
// convert on the way in and out, so a per-step state's pre-rounding values
// are bit for bit those the FP32 kernel produces from the same stored state.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "lq_common.cuh"

namespace lq {

struct DenseArgs {
    uint8_t *state;
    Layout L;
    Flags F;
    const void *q, *k, *v;
    const float *beta, *decay;
    float *out;
    int num_heads;
    uint32_t flags;  // kEarlyState: the kernel before this one does not write the state
};

constexpr int kDenseRowGroups = 16;

template <int D>
struct DenseShape {
    static constexpr int CL = D / 4;                       // column lanes (4 columns each)
    static constexpr int NT = CL * kDenseRowGroups;        // threads: 512 (D 128), 256 (D 64)
    static constexpr int RPT = D / kDenseRowGroups;        // key rows per thread
};

// Stored bytes of a dense state after the 128-byte header.
__host__ __device__ inline uint32_t dense_state_bytes(int D, int fmt) {
    if (fmt == 32) return (uint32_t)D * D * 4u;
    if (fmt == 16) return (uint32_t)D * D * 2u;
    return align_up((uint32_t)D * 4u, 128u) + (uint32_t)D * D;  // FP8: scales, then codes
}

struct DenseStage {
    uint32_t in_off, qkv_bytes, dec_off, bytes;
};

__host__ __device__ inline DenseStage dense_stage(int D, int fmt, int bf16, int kda) {
    DenseStage S;
    S.in_off = align_up(kHdrBytes + dense_state_bytes(D, fmt), 128u);
    S.qkv_bytes = align_up((uint32_t)D * (bf16 ? 2u : 4u), 16u);
    S.dec_off = S.in_off + 3u * S.qkv_bytes;
    S.bytes = align_up(S.dec_off + (kda ? (uint32_t)D * 4u : 0u), 128u);
    return S;
}

// barriers at 0, column partials [2][16][D] f32, u [D], column scales [D], kq [16]
__host__ __device__ inline uint32_t dense_fixed_smem(int D) {
    return 128u + 4u * (2u * kDenseRowGroups * D + 2u * D + kDenseRowGroups);
}

constexpr uint32_t kDenseSmemBudget = 220u * 1024u;

__host__ __device__ inline int dense_stages(int D, int fmt, int bf16, int kda) {
    const uint32_t sb = dense_stage(D, fmt, bf16, kda).bytes;
    const uint32_t avail = kDenseSmemBudget - dense_fixed_smem(D);
    const int n = (int)(avail / sb);
    return n > 4 ? 4 : n;
}

inline uint32_t dense_smem_bytes(int D, int fmt, int bf16, int kda) {
    return dense_fixed_smem(D) + (uint32_t)dense_stages(D, fmt, bf16, kda) * dense_stage(D, fmt, bf16, kda).bytes;
}

// e4m3 code -> its value (exact in FP32)
__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)(code & 0xFFu), __NV_E4M3);
    return __half2float(__half(h));
}

// E4M3 code of fl32(x / sc), ties to even, saturating at 448 (sc > 0)
__device__ __forceinline__ uint32_t e4m3_code(float x, float sc) {
    return (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(x, sc), __NV_SATFINITE, __NV_E4M3) & 0xFFu;
}

__device__ __forceinline__ void dsync(int n) { asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory"); }

template <int D, int FMT>
__global__ void __launch_bounds__(DenseShape<D>::NT, 1) dense_step_kernel(DenseArgs A) {
    using SH = DenseShape<D>;
    constexpr int NT = SH::NT, CL = SH::CL, RPT = SH::RPT, NRG = kDenseRowGroups;
    const int tid = threadIdx.x, lane = tid & 31;
    const int cq = tid % CL, rg = tid / CL;  // column quad, row group
    const int j0 = 4 * cq, i0 = RPT * rg;
    const Layout L = A.L;
    const Flags F = A.F;
    const DenseStage SG = dense_stage(D, FMT, F.bf16_in, F.kda);
    const int NS = dense_stages(D, FMT, F.bf16_in, F.kda);
    const uint32_t prefix = kHdrBytes + dense_state_bytes(D, FMT);
    const uint32_t in_bytes = 3u * SG.qkv_bytes + (F.kda ? (uint32_t)D * 4u : 0u);
    const int G = gridDim.x;
    const int n_mine = (A.num_heads - (int)blockIdx.x + G - 1) / G;
    const bool early = (A.flags & kEarlyState) != 0u;

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);  // [NS <= 4]
    float *s_pk = reinterpret_cast<float *>(smem + 128);  // [NRG][D]
    float *s_pq = s_pk + NRG * D;                          // [NRG][D]
    float *s_u = s_pq + NRG * D;                           // [D]
    float *s_sc = s_u + D;                                 // [D]
    float *s_kq = s_sc + D;                                // [NRG]
    uint8_t *stages = smem + dense_fixed_smem(D);

    auto blob_of = [&](int it) -> const uint8_t * {
        return A.state + ((size_t)blockIdx.x + (size_t)it * G) * L.blob;
    };
    auto issue_inputs = [&](int it, int s) {
        const size_t h = (size_t)blockIdx.x + (size_t)it * G;
        uint8_t *in = stages + (size_t)s * SG.bytes + SG.in_off;
        const size_t qo = h * (size_t)SG.qkv_bytes;
        bulk_g2s(in, static_cast<const uint8_t *>(A.q) + qo, SG.qkv_bytes, &full[s]);
        bulk_g2s(in + SG.qkv_bytes, static_cast<const uint8_t *>(A.k) + qo, SG.qkv_bytes, &full[s]);
        bulk_g2s(in + 2 * SG.qkv_bytes, static_cast<const uint8_t *>(A.v) + qo, SG.qkv_bytes, &full[s]);
        if (F.kda) bulk_g2s(stages + (size_t)s * SG.bytes + SG.dec_off, A.decay + h * D, (uint32_t)D * 4u, &full[s]);
    };

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
        if (early)  // the previous kernel does not write the state: stage it now
            for (int it = 0; it < NS && it < n_mine; ++it) {
                mbar_expect_tx(&full[it], prefix);
                bulk_g2s(stages + (size_t)it * SG.bytes, blob_of(it), prefix, &full[it]);
            }
        else
            for (int it = 0; it < NS && it < n_mine; ++it) bulk_prefetch_l2(blob_of(it), prefix);
    }
    pdl_wait();
    pdl_trigger();
    if (tid == 0) {
        for (int it = 0; it < NS && it < n_mine; ++it) {
            if (early) {
                mbar_arrive_expect_tx(&full[it], in_bytes);
            } else {
                mbar_arrive_expect_tx(&full[it], prefix + in_bytes);
                bulk_g2s(stages + (size_t)it * SG.bytes, blob_of(it), prefix, &full[it]);
            }
            issue_inputs(it, it);
        }
    }
    __syncthreads();

    for (int it = 0; it < n_mine; ++it) {
        const int s = it % NS;
        const size_t h = (size_t)blockIdx.x + (size_t)it * G;
        uint8_t *blob = A.state + h * L.blob;
        const uint8_t *st = stages + (size_t)s * SG.bytes;
        const float beta = A.beta[h];
        const float alpha = F.kda ? 1.f : A.decay[h];
        const bool landed = mbar_wait_bounded(&full[s], (uint32_t)(it / NS) & 1u);
        if (!__syncthreads_and(landed)) {
            if (tid == 0) {
                set_status(blob, LQ_DEV_TIMEOUT);
                // let the copies still in flight land before the CTA leaves
                for (int x = it; x < it + NS && x < n_mine; ++x)
                    mbar_wait_bounded(&full[x % NS], (uint32_t)(x / NS) & 1u);
            }
            for (int x = tid; x < D; x += NT) A.out[h * D + x] = 0.f;
            break;
        }
        const uint4 hdr = *reinterpret_cast<const uint4 *>(st);
        const bool run = hdr.w == kMagic && hdr.y == 0;  // uniform over the CTA

        // ---- the stored state of this thread's tile, as FP32
        float S[RPT][4];
        if (run) {
            if constexpr (FMT == 32) {
                const float *Sp = reinterpret_cast<const float *>(st + kHdrBytes);
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const float4 v4 = *reinterpret_cast<const float4 *>(Sp + (size_t)(i0 + r) * D + j0);
                    S[r][0] = v4.x; S[r][1] = v4.y; S[r][2] = v4.z; S[r][3] = v4.w;
                }
            } else if constexpr (FMT == 16) {
                const uint16_t *Sb = reinterpret_cast<const uint16_t *>(st + kHdrBytes);
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const uint2 w = *reinterpret_cast<const uint2 *>(Sb + (size_t)(i0 + r) * D + j0);
                    S[r][0] = __uint_as_float(w.x << 16);
                    S[r][1] = __uint_as_float(w.x & 0xFFFF0000u);
                    S[r][2] = __uint_as_float(w.y << 16);
                    S[r][3] = __uint_as_float(w.y & 0xFFFF0000u);
                }
            } else {
                const float4 sc = *reinterpret_cast<const float4 *>(st + kHdrBytes + 4 * j0);
                const uint8_t *C = st + kHdrBytes + align_up((uint32_t)D * 4u, 128u);
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(C + (size_t)(i0 + r) * D + j0);
                    S[r][0] = __fmul_rn(e4m3_to_float(w), sc.x);
                    S[r][1] = __fmul_rn(e4m3_to_float(w >> 8), sc.y);
                    S[r][2] = __fmul_rn(e4m3_to_float(w >> 16), sc.z);
                    S[r][3] = __fmul_rn(e4m3_to_float(w >> 24), sc.w);
                }
            }
        }
        float kr[RPT], qr[RPT], ar[RPT];
        float kq = 0.f, vt = 0.f;
        if (run) {
            const uint8_t *in = st + SG.in_off;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                kr[r] = load_in(in + SG.qkv_bytes, i0 + r, F.bf16_in);
                qr[r] = load_in(in, i0 + r, F.bf16_in);
                ar[r] = F.kda ? reinterpret_cast<const float *>(st + SG.dec_off)[i0 + r] : alpha;
            }
            if (tid < D) {
                kq = load_in(in + SG.qkv_bytes, tid, F.bf16_in) * load_in(in, tid, F.bf16_in);
                vt = load_in(in + 2 * SG.qkv_bytes, tid, F.bf16_in);
            }
        }

        // ---- S' = D_t S and this tile's column partials of S'^T k, S'^T q
        float2 pk01 = make_float2(0.f, 0.f), pk23 = pk01, pq01 = pk01, pq23 = pk01;
        if (run) {
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float2 a2 = make_float2(ar[r], ar[r]);
                float2 s01 = __fmul2_rn(a2, make_float2(S[r][0], S[r][1]));
                float2 s23 = __fmul2_rn(a2, make_float2(S[r][2], S[r][3]));
                S[r][0] = s01.x; S[r][1] = s01.y; S[r][2] = s23.x; S[r][3] = s23.y;
                const float2 k2 = make_float2(kr[r], kr[r]), q2 = make_float2(qr[r], qr[r]);
                pk01 = __ffma2_rn(s01, k2, pk01);
                pk23 = __ffma2_rn(s23, k2, pk23);
                pq01 = __ffma2_rn(s01, q2, pq01);
                pq23 = __ffma2_rn(s23, q2, pq23);
            }
            *reinterpret_cast<float4 *>(s_pk + rg * D + j0) = make_float4(pk01.x, pk01.y, pk23.x, pk23.y);
            *reinterpret_cast<float4 *>(s_pq + rg * D + j0) = make_float4(pq01.x, pq01.y, pq23.x, pq23.y);
            if (tid < D) {
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) kq += __shfl_xor_sync(0xFFFFFFFFu, kq, off);
                if (lane == 0) s_kq[tid >> 5] = kq;
            }
        }
        dsync(NT);  // every thread holds its entries: the stage may be refilled
        if (tid == 0 && it + NS < n_mine) {
            mbar_arrive_expect_tx(&full[s], prefix + in_bytes);
            bulk_g2s(stages + (size_t)s * SG.bytes, blob_of(it + NS), prefix, &full[s]);
            issue_inputs(it + NS, s);
        }
        if (!run) {
            for (int x = tid; x < D; x += NT) A.out[h * D + x] = 0.f;
            if (tid == 0 && hdr.w != kMagic && hdr.y == 0) set_status(blob, LQ_DEV_CORRUPT);
            dsync(NT);  // keep the CTA in step (the partial arrays are reused)
            continue;
        }
        // ---- u and o per value column (thread j < D), in row-group order
        if (tid < D) {
            float a = 0.f, b = 0.f, kqa = 0.f;
#pragma unroll
            for (int w = 0; w < NRG; ++w) {
                a += s_pk[w * D + tid];
                b += s_pq[w * D + tid];
            }
#pragma unroll
            for (int w = 0; w < D / 32; ++w) kqa += s_kq[w];
            const float u = beta * (vt - a);
            s_u[tid] = u;
            A.out[h * D + tid] = fmaf(kqa, u, b);
        }
        dsync(NT);
        // ---- S_new = S' + k u^T
        {
            const float4 u4 = *reinterpret_cast<const float4 *>(s_u + j0);
            const float2 u01 = make_float2(u4.x, u4.y), u23 = make_float2(u4.z, u4.w);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float2 k2 = make_float2(kr[r], kr[r]);
                const float2 n01 = __ffma2_rn(k2, u01, make_float2(S[r][0], S[r][1]));
                const float2 n23 = __ffma2_rn(k2, u23, make_float2(S[r][2], S[r][3]));
                S[r][0] = n01.x; S[r][1] = n01.y; S[r][2] = n23.x; S[r][3] = n23.y;
            }
        }
        // ---- store the new state in its format
        if constexpr (FMT == 32) {
            float *Sp = reinterpret_cast<float *>(blob + kHdrBytes);
#pragma unroll
            for (int r = 0; r < RPT; ++r)
                __stcs(reinterpret_cast<float4 *>(Sp + (size_t)(i0 + r) * D + j0),
                       make_float4(S[r][0], S[r][1], S[r][2], S[r][3]));
        } else if constexpr (FMT == 16) {
            uint16_t *Sb = reinterpret_cast<uint16_t *>(blob + kHdrBytes);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const uint32_t w0 = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(S[r][0])) |
                                    ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(S[r][1])) << 16);
                const uint32_t w1 = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(S[r][2])) |
                                    ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(S[r][3])) << 16);
                __stcs(reinterpret_cast<uint2 *>(Sb + (size_t)(i0 + r) * D + j0), make_uint2(w0, w1));
            }
        } else {
            // column maxima over the tile's rows, then over the row groups
            float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) m[c] = fmaxf(m[c], fabsf(S[r][c]));
            *reinterpret_cast<float4 *>(s_pk + rg * D + j0) = make_float4(m[0], m[1], m[2], m[3]);
            dsync(NT);
            if (tid < D) {
                float mm = 0.f;
#pragma unroll
                for (int w = 0; w < NRG; ++w) mm = fmaxf(mm, s_pk[w * D + tid]);
                const float sc = __fdiv_rn(mm, 448.f);
                s_sc[tid] = sc;
                reinterpret_cast<float *>(blob + kHdrBytes)[tid] = sc;
            }
            dsync(NT);
            const float4 sc4 = *reinterpret_cast<const float4 *>(s_sc + j0);
            const float sc[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
            uint8_t *C = blob + kHdrBytes + align_up((uint32_t)D * 4u, 128u);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                uint32_t w = 0u;
#pragma unroll
                for (int c = 0; c < 4; ++c) w |= (sc[c] == 0.f ? 0u : e4m3_code(S[r][c], sc[c])) << (8 * c);
                __stcs(reinterpret_cast<unsigned int *>(C + (size_t)(i0 + r) * D + j0), w);
            }
        }
    }
}

}  // namespace lq
