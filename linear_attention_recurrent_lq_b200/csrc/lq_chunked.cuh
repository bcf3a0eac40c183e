// lq_chunked.cuh -- prompt handoff on the tensor cores: the chunkwise form of
// the delta rule (dk = dv = 128), then compression of the final state into a
// fresh LeapQuant blob in the same kernel (sm_100a, tcgen05).
//
// The pages have the state a prefill leaves enter the quantized cache before
// decode starts (news post "Linear attention has to move state every token it
// generates; LeapQuant compresses it to 8-bit without losing accuracy",
// per-window paragraph; "LeapQuant: Efficient Linear Attention with Accurate
// Recurrent State Quantization", abstract: Gated DeltaNet and Kimi Delta
// Attention heads).  The recurrence is that of decode,
//     S_t = D_t S_{t-1} + k_t u_t^T,  u_t = beta_t (v_t - (D_t S_{t-1})^T k_t),
//     o_t = S_t^T q_t,
// and over a chunk of n tokens it is solved in closed form.  The first token's
// gate is applied to the incoming state S (S' = D_{t0} S); with G_t the
// product of the gates of tokens t0+1 .. t (per key channel; G_{t0} = 1),
//     Kt = K . G, Qt = Q . G, Kh = K / G          (rows = tokens)
//     A  = strictly lower part of diag(beta) Kt Kh^T
//     U  = (I + A)^-1 diag(beta) (V - Kt S')     (the new u_t)
//     O  = Qt S' + (lower part of Qt Kh^T, diagonal included) U
//     S  = diag(G_last) S' + (K . G_last / G)^T U.
// A chunk ends before any token that would take a product G below 2^-40, so
// Kh stays in range whatever the gates (a gate of 0 starts a new chunk, where
// it scales the state); otherwise chunks are 64 tokens.
//
// Layout (one 256-thread CTA per (slot, head), one CTA per SM):
//  * tensor memory, 512 columns: S^T (lane = value channel, column = key
//    channel) in [0, 128); W^T | Y^T in [128, 256) with W = Kt S', Y = Qt S'
//    (O^T accumulates onto Y^T); [Kt; Qt] Kh^T in [256, 320); U^T in
//    [320, 384);
//  * the products are TF32 MMAs with FP32 accumulation (tcgen05.mma issued by
//    one thread, completion through an mbarrier): [Kt;Qt] Kh^T and
//    S'^T [Kt;Qt]^T (S' read from tensor memory as the A operand),
//    U^T = RHS^T Tinv^T, O^T += U^T P^T and S^T += U^T Kbar; the operand tiles
//    are K-major with the 128-byte swizzle in shared memory, values rounded
//    to TF32 to nearest;
//  * (I + A)^-1 on the CUDA cores in FP32: the 16 x 16 diagonal blocks by
//    forward substitution, then the off-diagonal blocks level by level;
//  * the chunk's q, k, v (and KDA decays) arrive by bulk copies
//    (cp.async.bulk, no multicast), beta and the GDN decays by plain loads.
// After the last chunk S goes from tensor memory to the flush's register tile
// and through compress_tile, as the token-recurrent prefill does.
#pragma once

#include "lq_prefill.cuh"
#include "lq_umma.cuh"

namespace lq {

constexpr int kChunk = 64;                 // tokens per chunk (at most)
constexpr float kMinChunkGate = 0x1p-40f;  // smallest gate product inside a chunk
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColW = 128, kColY = 192, kColA = 256, kColU = 320;

// Shared memory (from a 1024-aligned base): tile region X [64 KB] | tile
// region K [32 KB] | staging: q, k, v rows [kChunk][in bytes] each, KDA
// decay rows [kChunk][128] f32 (staged with bf16 inputs; with f32 inputs they
// would not fit and are read from global memory) | control.
struct ChunkSmem {
    uint32_t stage_q, stage_k, stage_v, stage_dec, ctl, total;
    int dec_staged;
};

__host__ __device__ inline ChunkSmem chunk_smem(int bf16, int kda) {
    constexpr uint32_t D = 128;
    ChunkSmem S;
    const uint32_t qkv = D * (bf16 ? 2u : 4u);
    S.dec_staged = kda && bf16;
    S.stage_q = 98304u;
    S.stage_k = S.stage_q + kChunk * qkv;
    S.stage_v = S.stage_k + kChunk * qkv;
    S.stage_dec = S.stage_v + kChunk * qkv;
    S.ctl = align_up(S.stage_dec + (S.dec_staged ? kChunk * D * 4u : 0u), 128u);
    // control: barriers [2] | tmem slot | n | beta [64] | alpha [64] | gate scale [128] | M [16][16]
    S.total = S.ctl + 64u + 4u * (2u * kChunk + 128u) + 1024u + 1024u;  // + alignment slack
    return S;
}

// (I + A)^-1 of a unit lower-triangular 64 x 64 matrix in FP32 (A strictly
// lower, row-major in Lb), into Tb (row-major); Mb: 16 x 16 scratch.  All 256
// threads.
__device__ __forceinline__ void unit_lower_inverse(const float *Lb, float *Tb, float *Mb, int tid) {
    for (int x = tid; x < kChunk * kChunk; x += kGroup) Tb[x] = 0.f;
    __syncthreads();
    // diagonal 16 x 16 blocks: column c of block b by forward substitution
    if (tid < 64) {
        const int b = tid >> 4, c = tid & 15, o = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = r == c ? 1.f : 0.f;
#pragma unroll
            for (int s = 0; s < r; ++s)
                if (s >= c) acc = fmaf(-Lb[(o + r) * kChunk + o + s], x[s], acc);
            x[r] = r < c ? 0.f : acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[(o + r) * kChunk + o + c] = x[r];
    }
    __syncthreads();
    // off-diagonal blocks, nearest the diagonal first:
    // T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj
    const int r = tid >> 4, c = tid & 15;
#pragma unroll 1
    for (int d = 1; d < 4; ++d)
#pragma unroll 1
        for (int bj = 0; bj + d < 4; ++bj) {
            const int bi = bj + d;
            float m = 0.f;
            for (int k = 16 * bj; k < 16 * bi; ++k) m = fmaf(Lb[(16 * bi + r) * kChunk + k], Tb[k * kChunk + 16 * bj + c], m);
            Mb[r * 16 + c] = m;
            __syncthreads();
            float t = 0.f;
#pragma unroll
            for (int s = 0; s < 16; ++s) t = fmaf(Tb[(16 * bi + r) * kChunk + 16 * bi + s], Mb[s * 16 + c], t);
            Tb[(16 * bi + r) * kChunk + 16 * bj + c] = -t;
            __syncthreads();
        }
}

template <int BITS, bool SLOTS>
__global__ void __launch_bounds__(kGroup, 1) chunk_prefill_kernel(PrefillArgs A) {
    constexpr int D = 128;
    constexpr int IP = FT<D>::IP, TJ = FT<D>::TJ;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Layout L = A.L;
    const Flags F = A.F;
    const int T = A.tokens;
    const ChunkSmem SM = chunk_smem(F.bf16_in, F.kda);
    const uint32_t qkv = (uint32_t)D * (F.bf16_in ? 2u : 4u);
    const int h = blockIdx.x;  // work item
    const int H = A.map.heads;
    const int row = h / H, hh = h - row * H;
    const int bi = SLOTS ? A.map.blob(h) : h;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *RX = smem, *RK = smem + 65536;
    uint64_t *bar_stage = reinterpret_cast<uint64_t *>(smem + SM.ctl);
    uint64_t *bar_mma = bar_stage + 1;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + SM.ctl + 16);
    int *s_n = reinterpret_cast<int *>(smem + SM.ctl + 20);
    float *s_beta = reinterpret_cast<float *>(smem + SM.ctl + 64);
    float *s_alpha = s_beta + kChunk;
    float *s_gs = s_alpha + kChunk;   // per key channel: the gate scale of the state
    float *s_M = s_gs + 128;          // 16 x 16 scratch
    const uint32_t rx = smem_u32(RX), rk = smem_u32(RK);

    pdl_wait();
    pdl_trigger();
    if (bi < 0) return;  // slot out of range: nothing to do (uniform over the CTA)
    uint8_t *blob = A.state + (size_t)bi * L.blob;
    int len = T;
    if (A.lengths) len = min(max(__ldcg(A.lengths + row), 0), T);
    auto in_row = [&](int t) -> size_t { return ((size_t)row * T + t) * H + hh; };
    auto gate = [&](int t, int i) -> float {  // gate of token t, key channel i (global)
        return F.kda ? A.decay[in_row(t) * D + i] : A.decay[in_row(t)];
    };

    if (tid == 0) {
        mbar_init(bar_stage, 1);
        mbar_init(bar_mma, 1);
        *s_n = kChunk;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(s_tmem, kTmemCols);
    // the first token's gate scales the incoming state
    if (tid < D) s_gs[tid] = len > 0 ? gate(0, tid) : 1.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    // lane j = 32 (warp % 4) + lane, columns [64 (warp / 4), +64)
    const int j = 32 * (warp & 3) + lane, chalf = warp >> 2;
    const uint32_t tlane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);

    // ---- S'^T into tensor memory: S^T[j][i] = gs_i S0[i][j]
    {
        const float *S0 = A.S0 ? A.S0 + (size_t)h * D * D : nullptr;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
            float v[16];
            const int ib = 64 * chalf + 16 * q;
#pragma unroll
            for (int x = 0; x < 16; ++x) v[x] = S0 ? s_gs[ib + x] * S0[(size_t)(ib + x) * D + j] : 0.f;
            tmem_st16(tlane + kColS + (uint32_t)ib, v);
        }
    }

    uint32_t mma_phase = 0, stage_phase = 0;
    bool failed = false;
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_bounded(bar_mma, mma_phase & 1u);
        ++mma_phase;
        tc_fence_after();
        return ok;
    };

#pragma unroll 1
    for (int t0 = 0; t0 < len;) {
        const int nt = min(kChunk, len - t0);  // tokens staged (the chunk may end earlier)
        // ---- stage q, k, v (and KDA decays) of tokens t0 .. t0 + nt; beta, alpha
        if (warp == 0) {
            if (lane == 0)
                mbar_arrive_expect_tx(bar_stage, (uint32_t)nt * (3u * qkv + (SM.dec_staged ? (uint32_t)D * 4u : 0u)));
            __syncwarp();
            for (int x = lane; x < nt; x += 32) {
                const size_t r = in_row(t0 + x);
                bulk_g2s(smem + SM.stage_q + (size_t)x * qkv, static_cast<const uint8_t *>(A.q) + r * qkv, qkv, bar_stage);
                bulk_g2s(smem + SM.stage_k + (size_t)x * qkv, static_cast<const uint8_t *>(A.k) + r * qkv, qkv, bar_stage);
                bulk_g2s(smem + SM.stage_v + (size_t)x * qkv, static_cast<const uint8_t *>(A.v) + r * qkv, qkv, bar_stage);
                if (SM.dec_staged)
                    bulk_g2s(smem + SM.stage_dec + (size_t)x * D * 4, A.decay + r * D, (uint32_t)D * 4u, bar_stage);
            }
        }
        if (tid < kChunk) {
            const bool in = tid < nt;
            s_beta[tid] = in ? A.beta[in_row(t0 + tid)] : 0.f;
            s_alpha[tid] = (in && !F.kda) ? A.decay[in_row(t0 + tid)] : 1.f;
        }
        const bool landed = mbar_wait_bounded(bar_stage, stage_phase & 1u);
        ++stage_phase;
        if (!__syncthreads_and(landed)) {
            failed = true;
            break;
        }
        const float *dec = reinterpret_cast<const float *>(smem + SM.stage_dec);
        auto a_of = [&](int x, int i) -> float {
            return F.kda ? (SM.dec_staged ? dec[x * D + i] : A.decay[in_row(t0 + x) * D + i]) : s_alpha[x];
        };
        auto in_of = [&](uint32_t base, int x, int i) -> float {
            return load_in(smem + base + (size_t)x * qkv, i, F.bf16_in);
        };

        // ---- pass 1: chunk length (the first token whose gate product falls
        // below the range ends the chunk)
        if (tid < D) {
            float g = 1.f;
            int viol = nt;
            for (int x = 1; x < nt; ++x) {
                g *= a_of(x, tid);
                if (!(g >= kMinChunkGate)) {
                    viol = x;
                    break;
                }
            }
            if (viol < kChunk) atomicMin(s_n, viol);
        }
        __syncthreads();
        const int n = min(*s_n, nt);

        // ---- pass 2: X = [Kt; Qt] (128 x 128) and Kh (64 x 128), K-major tiles
        {
            const int i = tid & 127;
            const bool kside = tid < 128;
            float g = 1.f;
#pragma unroll 1
            for (int x = 0; x < kChunk; ++x) {
                if (x > 0 && x < n) g *= a_of(x, i);
                if (kside) {
                    const float kv = x < n ? in_of(SM.stage_k, x, i) : 0.f;
                    *reinterpret_cast<float *>(RX + sw128_off(x, i, 128)) = to_tf32(kv * g);
                    *reinterpret_cast<float *>(RK + sw128_off(x, i, 64)) = to_tf32(kv * __frcp_rn(g));
                } else {
                    const float qv = x < n ? in_of(SM.stage_q, x, i) : 0.f;
                    *reinterpret_cast<float *>(RX + sw128_off(64 + x, i, 128)) = to_tf32(qv * g);
                }
            }
            // the state's scale at the chunk end: the last product, times the
            // next chunk's first gate (applied here, to S and to Kbar)
            if (kside) s_gs[i] = g * (t0 + n < len ? gate(t0 + n, i) : 1.f);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id1 = umma_idesc_tf32(128, 64), id3 = umma_idesc_tf32(128, 128);
#pragma unroll 1
            for (int ks = 0; ks < D / 8; ++ks)
                umma_ss(tmem + kColA, umma_kdesc(rx, 128, ks), umma_kdesc(rk, 64, ks), id1, ks > 0);
#pragma unroll 1
            for (int ks = 0; ks < D / 8; ++ks)
                umma_ts(tmem + kColW, tmem + kColS + (uint32_t)(8 * ks), umma_kdesc(rx, 128, ks), id3, ks > 0);
            umma_commit(bar_mma);
        }
        if (!__syncthreads_and(wait_mma())) {
            failed = true;
            break;
        }

        // ---- A (into Lb, plain) and the masked lower part of Qt Kh^T (P tile)
        float *Lb = reinterpret_cast<float *>(RK);          // [64][64]
        float *Tb = reinterpret_cast<float *>(RK + 16384);  // [64][64]
        {
            // lanes 0..63: rows of Kt Kh^T; lanes 64..127: rows of Qt Kh^T
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                float v[16];
                const int c0 = 32 * chalf + 16 * q;
                tmem_ld16(tlane + kColA + (uint32_t)c0, v);
                if (j < 64) {
                    const int t = j;
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const int s = c0 + x;
                        Lb[t * kChunk + s] = (s < t && t < n) ? s_beta[t] * v[x] : 0.f;
                    }
                } else {
                    const int t = j - 64;
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const int s = c0 + x;
                        *reinterpret_cast<float *>(RX + 49152 + sw128_off(t, s, 64)) =
                            to_tf32((s <= t && t < n) ? v[x] : 0.f);
                    }
                }
            }
        }
        __syncthreads();
        unit_lower_inverse(Lb, Tb, s_M, tid);
        // Tinv as the B operand of U^T = RHS^T Tinv^T (rows t, K = s)
        for (int x = tid; x < kChunk * kChunk; x += kGroup) {
            const int t = x >> 6, s = x & 63;
            *reinterpret_cast<float *>(RX + 32768 + sw128_off(t, s, 64)) = to_tf32(Tb[x]);
        }
        // RHS^T (rows j, K = s): beta_s (v_s[j] - W_s[j])
        {
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                float w[16];
                const int c0 = 32 * chalf + 16 * q;
                tmem_ld16(tlane + kColW + (uint32_t)c0, w);
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const int s = c0 + x;
                    const float r = s < n ? s_beta[s] * (in_of(SM.stage_v, s, j) - w[x]) : 0.f;
                    *reinterpret_cast<float *>(RX + sw128_off(j, s, 128)) = to_tf32(r);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idu = umma_idesc_tf32(128, 64);
#pragma unroll 1
            for (int ks = 0; ks < kChunk / 8; ++ks)
                umma_ss(tmem + kColU, umma_kdesc(rx, 128, ks), umma_kdesc(rx + 32768, 64, ks), idu, ks > 0);
            umma_commit(bar_mma);
        }
        // meanwhile: S'^T scaled by the chunk-end gate scale (column i)
        {
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                float v[16];
                const int ib = 64 * chalf + 16 * q;
                tmem_ld16(tlane + kColS + (uint32_t)ib, v);
#pragma unroll
                for (int x = 0; x < 16; ++x) v[x] *= s_gs[ib + x];
                tmem_st16(tlane + kColS + (uint32_t)ib, v);
            }
        }
        if (!__syncthreads_and(wait_mma())) {
            failed = true;
            break;
        }

        // ---- U^T (rows j, K = s) as the A operand; Kbar^T (rows i, K = s)
        {
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                float u[16];
                const int c0 = 32 * chalf + 16 * q;
                tmem_ld16(tlane + kColU + (uint32_t)c0, u);
#pragma unroll
                for (int x = 0; x < 16; ++x)
                    *reinterpret_cast<float *>(RK + sw128_off(j, c0 + x, 128)) = to_tf32(u[x]);
            }
            // Kbar[s][i] = k_s,i * (G_last,i / G_s,i) * (next gate): thread i
            // takes tokens [32 half, +32), its gate product recomputed
            const int i = tid & 127, s0 = 32 * (tid >> 7);
            float g = 1.f;
            for (int x = 1; x <= s0 && x < n; ++x) g *= a_of(x, i);
            const float gl = s_gs[i];
#pragma unroll 1
            for (int x = s0; x < s0 + 32; ++x) {
                if (x > s0 && x < n) g *= a_of(x, i);
                const float kb = x < n ? in_of(SM.stage_k, x, i) * (gl * __frcp_rn(g)) : 0.f;
                *reinterpret_cast<float *>(RX + sw128_off(i, x, 128)) = to_tf32(kb);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t ido = umma_idesc_tf32(128, 64), ids = umma_idesc_tf32(128, 128);
#pragma unroll 1
            for (int ks = 0; ks < kChunk / 8; ++ks)  // O^T += U^T P^T (onto Y^T)
                umma_ss(tmem + kColY, umma_kdesc(rk, 128, ks), umma_kdesc(rx + 49152, 64, ks), ido, 1u);
#pragma unroll 1
            for (int ks = 0; ks < kChunk / 8; ++ks)  // S^T += U^T Kbar
                umma_ss(tmem + kColS, umma_kdesc(rk, 128, ks), umma_kdesc(rx, 128, ks), ids, 1u);
            umma_commit(bar_mma);
        }
        if (!__syncthreads_and(wait_mma())) {
            failed = true;
            break;
        }
        // ---- outputs o_t[j] of this chunk
        if (A.out) {
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                float o[16];
                const int c0 = 32 * chalf + 16 * q;
                tmem_ld16(tlane + kColY + (uint32_t)c0, o);
#pragma unroll
                for (int x = 0; x < 16; ++x)
                    if (c0 + x < n) A.out[in_row(t0 + c0 + x) * D + j] = o[x];
            }
        }
        if (tid == 0) *s_n = kChunk;
        __syncthreads();  // the tiles and the staging are free for the next chunk
        t0 += n;
    }

    if (failed) {
        if (tid == 0) {
            set_status(blob, LQ_DEV_TIMEOUT);
            mbar_wait_bounded(bar_mma, mma_phase & 1u);  // let work in flight finish
            mbar_wait_bounded(bar_stage, stage_phase & 1u);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tmem, kTmemCols);
        return;
    }
    // outputs of the tokens past this row's prompt length
    if (A.out)
        for (int t = len; t < T; ++t)
            if (tid < D) A.out[in_row(t) * D + tid] = 0.f;

    // ---- S from tensor memory (S[i][j] = S^T[j][i]) into a plain array, then
    // the flush's register tile
    float *Sp = reinterpret_cast<float *>(RX);
    {
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
            float v[16];
            const int ib = 64 * chalf + 16 * q;
            tmem_ld16(tlane + kColS + (uint32_t)ib, v);
#pragma unroll
            for (int x = 0; x < 16; ++x) Sp[(ib + x) * D + j] = v[x];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    const Tile<D> tl(tid);
    TileReg<D> P;
#pragma unroll
    for (int ip = 0; ip < IP; ++ip)
#pragma unroll
        for (int jj = 0; jj < TJ; ++jj)
            P[ip][jj] = f2(Sp[(tl.i0 + 2 * ip) * D + tl.j0 + jj], Sp[(tl.i0 + 2 * ip + 1) * D + tl.j0 + jj]);
    if (A.S_final) {
        float *So = A.S_final + (size_t)h * D * D;
        for (int x = tid; x < D * D / 4; x += kGroup)
            reinterpret_cast<float4 *>(So)[x] = reinterpret_cast<const float4 *>(Sp)[x];
    }
    __syncthreads();  // the plain copy is read: its space serves the compression
    const int ncomp = compress_tile<D, BITS>(P, F, L, RK, blob, tid);
    write_fresh_header<D>(blob, F, ncomp, true, tid);
}

inline uint32_t chunk_prefill_smem_bytes(const Flags &F) { return chunk_smem(F.bf16_in, F.kda).total; }

}  // namespace lq
