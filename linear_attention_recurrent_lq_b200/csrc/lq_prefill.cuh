// lq_prefill.cuh -- prompt handoff: run the delta rule over a prompt with the
// FP32 state held on chip, then compress that state into a fresh LeapQuant
// blob without writing it to global memory first (sm_100a).
//
// The pages have the state produced by prefill enter the quantized cache and
// only then decode from it (news post "Linear attention has to move state
// every token it generates; LeapQuant compresses it to 8-bit without losing
// accuracy", per-window paragraph).  The step is the same delta rule as in
// decode, in FP32:
//     S' = diag(a_t) S,  u_t = beta_t (v_t - S'^T k_t),  S = S' + k_t u_t^T,
//     o_t = S^T q_t = S'^T q_t + (k_t . q_t) u_t,
// token after token (the recurrent form, not a chunkwise-parallel one), and
// the final S goes through the same compression as a window flush.
//
// One CTA of 256 threads per (slot, head), the state as the flush's register
// tile (each thread TI x TJ entries as float2 pairs of adjacent key rows).
// Per token: every thread forms its column partials of S'^T k and S'^T q,
// the partials meet in shared memory, thread j (< dv) forms u_j and o_j, and
// every thread applies the rank-one update to its tile.  The prompt's q, k, v
// (and the KDA decay) arrive in chunks of kPfChunk tokens through a
// two-stage ring of bulk copies issued by thread 0; beta and the GDN alpha
// are loaded one chunk ahead by plain loads.
#pragma once

#include "lq_flush.cuh"

namespace lq {

constexpr int kPfChunk = 16;  // tokens per staged chunk

struct PrefillArgs {
    uint8_t *state;
    Layout L;
    Flags F;
    const float *S0;          // [rows, H, dk, dv] or null (zero state)
    const void *q, *k, *v;    // [rows, T, H, d]
    const float *beta;        // [rows, T, H]
    const float *decay;       // [rows, T, H] (GDN) or [rows, T, H, dk] (KDA)
    const int32_t *lengths;   // [rows] prompt length of each row (clamped to [0, T]) or null (all T)
    float *out;               // [rows, T, H, dv] or null
    float *S_final;           // [rows, H, dk, dv] or null
    int tokens;               // T
    int num_heads;            // work items: rows * H
    SlotMap map;
};

struct PrefillStage {
    uint32_t qkv_bytes, tok_bytes, dec_off, ba_off, bytes;
};

// One stage: per token [q | k | v] (in_dtype, 16-byte aligned rows), then the
// KDA decay rows [kPfChunk][D] f32, then beta [kPfChunk] and alpha [kPfChunk].
__host__ __device__ inline PrefillStage prefill_stage(int D, int bf16, int kda) {
    PrefillStage S;
    S.qkv_bytes = align_up((uint32_t)D * (bf16 ? 2u : 4u), 16);
    S.tok_bytes = 3 * S.qkv_bytes;
    S.dec_off = S.tok_bytes * kPfChunk;
    S.ba_off = S.dec_off + (kda ? (uint32_t)D * 4u * kPfChunk : 0u);
    S.bytes = align_up(S.ba_off + 8u * kPfChunk, 128);
    return S;
}

// barriers (0) | kq (64) | column partials k-side, q-side [WR][D] each | u [D]
// | compress scratch | two stages
template <int D, int BITS>
__host__ __device__ constexpr uint32_t prefill_fixed_smem() {
    return align_up(128u + 4u * (2u * FT<D>::WR * D + D), 128u) + group_smem_bytes<D, BITS>();
}

inline uint32_t prefill_smem_bytes(int D, int bits, const Flags &F) {
    uint32_t fixed;
    if (D == 128)
        fixed = bits == 8 ? prefill_fixed_smem<128, 8>() : prefill_fixed_smem<128, 4>();
    else
        fixed = bits == 8 ? prefill_fixed_smem<64, 8>() : prefill_fixed_smem<64, 4>();
    return fixed + 2u * prefill_stage(D, F.bf16_in, F.kda).bytes;
}

// n consecutive inputs (n = 8 or 4) in the input dtype, as floats
template <int N>
__device__ __forceinline__ void load_row_slice(const uint8_t *p, int bf16, float (&x)[N]) {
    if (bf16) {
        if constexpr (N == 8) {
            const uint4 w = *reinterpret_cast<const uint4 *>(p);
            const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                x[2 * i] = __uint_as_float(a[i] << 16);
                x[2 * i + 1] = __uint_as_float(a[i] & 0xFFFF0000u);
            }
        } else {
            const uint2 w = *reinterpret_cast<const uint2 *>(p);
            const uint32_t a[2] = {w.x, w.y};
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                x[2 * i] = __uint_as_float(a[i] << 16);
                x[2 * i + 1] = __uint_as_float(a[i] & 0xFFFF0000u);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const float4 f = *reinterpret_cast<const float4 *>(p + 4 * i);
            x[i] = f.x;
            x[i + 1] = f.y;
            x[i + 2] = f.z;
            x[i + 3] = f.w;
        }
    }
}

template <int D, int BITS, bool SLOTS>
__global__ void __launch_bounds__(kGroup, 2) prefill_kernel(PrefillArgs A) {
    constexpr int TI = FT<D>::TI, TJ = FT<D>::TJ, IP = FT<D>::IP, WR = FT<D>::WR;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Layout L = A.L;
    const Flags F = A.F;
    const int T = A.tokens;
    const PrefillStage SG = prefill_stage(D, F.bf16_in, F.kda);
    const int h = blockIdx.x;  // work item
    const int H = A.map.heads;
    const int row = h / H, hh = h - row * H;
    const int bi = SLOTS ? A.map.blob(h) : h;
    const Tile<D> tl(tid);
    const int i0 = tl.i0, j0 = tl.j0;

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);  // [2]
    float *s_kq = reinterpret_cast<float *>(smem + 64);
    float *s_pk = reinterpret_cast<float *>(smem + 128);  // [WR][D]
    float *s_pq = s_pk + WR * D;                          // [WR][D]
    float *s_u = s_pq + WR * D;                           // [D]
    uint8_t *scratch = smem + align_up(128u + 4u * (2u * WR * D + D), 128u);
    uint8_t *stages = scratch + group_smem_bytes<D, BITS>();

    pdl_wait();
    pdl_trigger();
    if (bi < 0) return;  // slot out of range: nothing to do (uniform over the CTA)
    uint8_t *blob = A.state + (size_t)bi * L.blob;
    int len = T;
    if (A.lengths) len = min(max(__ldcg(A.lengths + row), 0), T);
    const int n_chunks = (len + kPfChunk - 1) / kPfChunk;
    auto in_row = [&](int t) -> size_t { return ((size_t)row * T + t) * H + hh; };

    // thread 0: stage chunk c into stage c % 2
    auto issue = [&](int c) {
        const int s = c & 1, n = min(kPfChunk, len - c * kPfChunk);
        uint8_t *st = stages + (size_t)s * SG.bytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)n * (SG.tok_bytes + (F.kda ? (uint32_t)D * 4u : 0u)));
        for (int x = 0; x < n; ++x) {
            const size_t r = in_row(c * kPfChunk + x);
            uint8_t *dst = st + (size_t)x * SG.tok_bytes;
            bulk_g2s(dst, static_cast<const uint8_t *>(A.q) + r * SG.qkv_bytes, SG.qkv_bytes, &full[s]);
            bulk_g2s(dst + SG.qkv_bytes, static_cast<const uint8_t *>(A.k) + r * SG.qkv_bytes, SG.qkv_bytes,
                     &full[s]);
            bulk_g2s(dst + 2 * SG.qkv_bytes, static_cast<const uint8_t *>(A.v) + r * SG.qkv_bytes,
                     SG.qkv_bytes, &full[s]);
            if (F.kda) bulk_g2s(st + SG.dec_off + (size_t)x * D * 4, A.decay + r * D, (uint32_t)D * 4u, &full[s]);
        }
    };
    // threads < kPfChunk: beta and the GDN alpha of chunk c (registers)
    auto load_ba = [&](int c, float &b, float &a) {
        const int t = c * kPfChunk + tid;
        b = 0.f;
        a = 1.f;
        if (tid < kPfChunk && c < n_chunks && t < len) {
            const size_t r = in_row(t);
            b = A.beta[r];
            if (!F.kda) a = A.decay[r];
        }
    };

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        fence_mbar_init();
        for (int c = 0; c < 2 && c < n_chunks; ++c) issue(c);
    }
    float nb, na;
    load_ba(0, nb, na);
    if (tid < kPfChunk) {
        reinterpret_cast<float *>(stages + SG.ba_off)[tid] = nb;
        reinterpret_cast<float *>(stages + SG.ba_off)[kPfChunk + tid] = na;
    }

    // ---- the state tile: S0 or zero
    TileReg<D> P;
#pragma unroll
    for (int ip = 0; ip < IP; ++ip)
#pragma unroll
        for (int jj = 0; jj < TJ; ++jj) P[ip][jj] = f2(0.f, 0.f);
    if (A.S0) {
        const float *S0 = A.S0 + (size_t)h * D * D;
#pragma unroll
        for (int ip = 0; ip < IP; ++ip)
#pragma unroll
            for (int jj = 0; jj < TJ; jj += 4) {
                const float4 a = *reinterpret_cast<const float4 *>(S0 + (size_t)(i0 + 2 * ip) * D + j0 + jj);
                const float4 b = *reinterpret_cast<const float4 *>(S0 + (size_t)(i0 + 2 * ip + 1) * D + j0 + jj);
                P[ip][jj] = f2(a.x, b.x);
                P[ip][jj + 1] = f2(a.y, b.y);
                P[ip][jj + 2] = f2(a.z, b.z);
                P[ip][jj + 3] = f2(a.w, b.w);
            }
    }
    __syncthreads();

    int failed = -1;  // chunk whose copies never landed
    for (int c = 0; c < n_chunks; ++c) {
        const int s = c & 1;
        const uint8_t *st = stages + (size_t)s * SG.bytes;
        if (!gsync_and(mbar_wait_bounded(&full[s], (uint32_t)(c >> 1) & 1u))) {
            failed = c;
            break;
        }
        load_ba(c + 1, nb, na);  // beta / alpha of the next chunk, in flight during this one
        const float *ba = reinterpret_cast<const float *>(st + SG.ba_off);
        const int n = min(kPfChunk, len - c * kPfChunk);
        for (int x = 0; x < n; ++x) {
            const uint8_t *tok = st + (size_t)x * SG.tok_bytes;
            float kr[TI], qr[TI];
            load_row_slice<TI>(tok + SG.qkv_bytes + (size_t)i0 * (F.bf16_in ? 2 : 4), F.bf16_in, kr);
            load_row_slice<TI>(tok + (size_t)i0 * (F.bf16_in ? 2 : 4), F.bf16_in, qr);
            // decay: S' = diag(a) S
            float2 a2[IP];
            if (F.kda) {
                const float *dec = reinterpret_cast<const float *>(st + SG.dec_off + (size_t)x * D * 4) + i0;
#pragma unroll
                for (int ip = 0; ip < IP; ++ip) a2[ip] = f2(dec[2 * ip], dec[2 * ip + 1]);
            } else {
                const float al = ba[kPfChunk + x];
#pragma unroll
                for (int ip = 0; ip < IP; ++ip) a2[ip] = f2(al, al);
            }
            float ck[TJ], cq[TJ];
#pragma unroll
            for (int jj = 0; jj < TJ; ++jj) {
                float2 sk = f2(0.f, 0.f), sq = f2(0.f, 0.f);
#pragma unroll
                for (int ip = 0; ip < IP; ++ip) {
                    P[ip][jj] = __fmul2_rn(P[ip][jj], a2[ip]);
                    sk = __ffma2_rn(P[ip][jj], f2(kr[2 * ip], kr[2 * ip + 1]), sk);
                    sq = __ffma2_rn(P[ip][jj], f2(qr[2 * ip], qr[2 * ip + 1]), sq);
                }
                ck[jj] = sk.x + sk.y;
                cq[jj] = sq.x + sq.y;
            }
            store_col_partials<D, float, false>(ck, s_pk, tid);
            store_col_partials<D, float, false>(cq, s_pq, tid);
            if (warp == 0) {  // k . q
                float kq = 0.f;
                for (int i = lane; i < D; i += 32)
                    kq = fmaf(load_in(tok + SG.qkv_bytes, i, F.bf16_in), load_in(tok, i, F.bf16_in), kq);
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) kq += __shfl_xor_sync(0xFFFFFFFFu, kq, off);
                if (lane == 0) *s_kq = kq;
            }
            gsync();
            if (tid < D) {
                const int j = tid;
                float a = 0.f, b = 0.f;
#pragma unroll
                for (int w = 0; w < WR; ++w) {
                    a += s_pk[w * D + j];
                    b += s_pq[w * D + j];
                }
                const float u = ba[x] * (load_in(tok + 2 * SG.qkv_bytes, j, F.bf16_in) - a);
                s_u[j] = u;
                if (A.out) A.out[in_row(c * kPfChunk + x) * D + j] = fmaf(*s_kq, u, b);
            }
            gsync();
            // S = S' + k u^T
            float uj[TJ];
#pragma unroll
            for (int jj = 0; jj < TJ; jj += 4) {
                const float4 u4 = *reinterpret_cast<const float4 *>(s_u + j0 + jj);
                uj[jj] = u4.x;
                uj[jj + 1] = u4.y;
                uj[jj + 2] = u4.z;
                uj[jj + 3] = u4.w;
            }
#pragma unroll
            for (int ip = 0; ip < IP; ++ip)
#pragma unroll
                for (int jj = 0; jj < TJ; ++jj)
                    P[ip][jj] = __ffma2_rn(f2(kr[2 * ip], kr[2 * ip + 1]), f2(uj[jj], uj[jj]), P[ip][jj]);
        }
        gsync();  // stage s has been read
        if (tid < kPfChunk && c + 1 < n_chunks) {
            float *nba = reinterpret_cast<float *>(stages + (size_t)((c + 1) & 1) * SG.bytes + SG.ba_off);
            nba[tid] = nb;
            nba[kPfChunk + tid] = na;
        }
        if (tid == 0 && c + 2 < n_chunks) issue(c + 2);
    }
    if (failed >= 0) {
        if (tid == 0) {
            set_status(blob, LQ_DEV_TIMEOUT);
            // let the copies still in flight (this chunk and the next) land before the CTA leaves
            for (int c = failed; c < failed + 2 && c < n_chunks; ++c)
                mbar_wait_bounded(&full[c & 1], (uint32_t)(c >> 1) & 1u);
        }
        return;
    }
    // outputs of the tokens past this row's prompt length
    if (A.out)
        for (int t = len; t < T; ++t)
            if (tid < D) A.out[in_row(t) * D + tid] = 0.f;
    if (A.S_final) {
        float *So = A.S_final + (size_t)h * D * D;
#pragma unroll
        for (int ip = 0; ip < IP; ++ip)
#pragma unroll
            for (int jj = 0; jj < TJ; jj += 4) {
                *reinterpret_cast<float4 *>(So + (size_t)(i0 + 2 * ip) * D + j0 + jj) =
                    make_float4(P[ip][jj].x, P[ip][jj + 1].x, P[ip][jj + 2].x, P[ip][jj + 3].x);
                *reinterpret_cast<float4 *>(So + (size_t)(i0 + 2 * ip + 1) * D + j0 + jj) =
                    make_float4(P[ip][jj].y, P[ip][jj + 1].y, P[ip][jj + 2].y, P[ip][jj + 3].y);
            }
    }
    const int ncomp = compress_tile<D, BITS>(P, F, L, scratch, blob, tid);
    write_fresh_header<D>(blob, F, ncomp, true, tid);
}

}  // namespace lq
