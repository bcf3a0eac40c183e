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
// region K [32 KB] | gate products G [kChunk][128] f32 | staging: q, k rows
// [kChunk][in bytes], and with bf16 inputs also v rows and the KDA decay rows
// [kChunk][128] f32 (with f32 inputs those would not fit and are read from
// global memory) | control.
struct ChunkSmem {
    uint32_t gbuf, stage_q, stage_k, stage_v, stage_dec, ctl, total;
    int v_staged, dec_staged;
};

__host__ __device__ inline ChunkSmem chunk_smem(int bf16, int kda) {
    constexpr uint32_t D = 128;
    ChunkSmem S;
    const uint32_t qkv = D * (bf16 ? 2u : 4u);
    S.v_staged = bf16;
    S.dec_staged = kda && bf16;
    S.gbuf = 98304u;
    S.stage_q = S.gbuf + kChunk * D * 4u;
    S.stage_k = S.stage_q + kChunk * qkv;
    S.stage_v = S.stage_k + kChunk * qkv;
    S.stage_dec = S.stage_v + (S.v_staged ? kChunk * qkv : 0u);
    S.ctl = align_up(S.stage_dec + (S.dec_staged ? kChunk * D * 4u : 0u), 128u);
    // control: barriers [2] | tmem slot | n | beta [64] | alpha [64] | gate scale [128] | M [3][16][16]
    S.total = S.ctl + 64u + 4u * (2u * kChunk + 128u) + 3072u + 1024u;  // + alignment slack
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
            float lr[16];
#pragma unroll
            for (int s = 0; s < 16; s += 4) {
                const float4 w = *reinterpret_cast<const float4 *>(Lb + (o + r) * kChunk + o + s);
                lr[s] = w.x; lr[s + 1] = w.y; lr[s + 2] = w.z; lr[s + 3] = w.w;
            }
            float acc = r == c ? 1.f : 0.f;
#pragma unroll
            for (int s = 0; s < r; ++s)
                if (s >= c) acc = fmaf(-lr[s], x[s], acc);
            x[r] = r < c ? 0.f : acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[(o + r) * kChunk + o + c] = x[r];
    }
    __syncthreads();
    // off-diagonal blocks, nearest the diagonal first, the blocks of one
    // level at once: T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj  (Mb: [3][16][16])
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
        const int nb = 4 - d;
        for (int e = tid; e < nb * 256; e += kGroup) {
            const int bj = e >> 8, r = (e >> 4) & 15, c = e & 15, bi = bj + d;
            float m0 = 0.f, m1 = 0.f;
#pragma unroll 1
            for (int k0 = 16 * bj; k0 < 16 * bi; k0 += 16) {
                float lr[16], tc[16];
#pragma unroll
                for (int y = 0; y < 16; y += 4) {
                    const float4 w = *reinterpret_cast<const float4 *>(Lb + (16 * bi + r) * kChunk + k0 + y);
                    lr[y] = w.x; lr[y + 1] = w.y; lr[y + 2] = w.z; lr[y + 3] = w.w;
                }
#pragma unroll
                for (int y = 0; y < 16; ++y) tc[y] = Tb[(k0 + y) * kChunk + 16 * bj + c];
#pragma unroll
                for (int y = 0; y < 16; y += 2) {
                    m0 = fmaf(lr[y], tc[y], m0);
                    m1 = fmaf(lr[y + 1], tc[y + 1], m1);
                }
            }
            Mb[e] = m0 + m1;
        }
        __syncthreads();
        for (int e = tid; e < nb * 256; e += kGroup) {
            const int bj = e >> 8, r = (e >> 4) & 15, c = e & 15, bi = bj + d;
            float tr[16], mc[16];
#pragma unroll
            for (int y = 0; y < 16; y += 4) {
                const float4 w = *reinterpret_cast<const float4 *>(Tb + (16 * bi + r) * kChunk + 16 * bi + y);
                tr[y] = w.x; tr[y + 1] = w.y; tr[y + 2] = w.z; tr[y + 3] = w.w;
            }
#pragma unroll
            for (int y = 0; y < 16; ++y) mc[y] = Mb[(bj << 8) + y * 16 + c];
            float t0 = 0.f, t1 = 0.f;
#pragma unroll
            for (int y = 0; y < 16; y += 2) {
                t0 = fmaf(tr[y], mc[y], t0);
                t1 = fmaf(tr[y + 1], mc[y + 1], t1);
            }
            Tb[(16 * bi + r) * kChunk + 16 * bj + c] = -(t0 + t1);
        }
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
    float *s_M = s_gs + 128;          // [3][16][16] scratch
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
        float *G = reinterpret_cast<float *>(smem + SM.gbuf);  // [kChunk][D] gate products
        // ---- stage q, k (and v, KDA decays) of tokens t0 .. t0 + nt with
        // 16-byte loads by every thread; beta, alpha
        {
            const int cpr = (int)(qkv >> 4);  // 16-byte pieces per row
            const int nbuf = SM.v_staged ? 3 : 2;
#pragma unroll 4
            for (int x = tid; x < nbuf * nt * cpr; x += kGroup) {
                const int bsel = x / (nt * cpr), rem = x - bsel * nt * cpr, r = rem / cpr, c = rem - r * cpr;
                const void *src = bsel == 0 ? A.q : (bsel == 1 ? A.k : A.v);
                const uint32_t dst = bsel == 0 ? SM.stage_q : (bsel == 1 ? SM.stage_k : SM.stage_v);
                const uint4 w = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(src) + in_row(t0 + r) * qkv) + c);
                *reinterpret_cast<uint4 *>(smem + dst + (size_t)r * qkv + 16 * c) = w;
            }
            if (SM.dec_staged) {
#pragma unroll 4
                for (int x = tid; x < nt * (D / 4); x += kGroup) {
                    const int r = x / (D / 4), c = x - r * (D / 4);
                    const float4 w = __ldg(reinterpret_cast<const float4 *>(A.decay + in_row(t0 + r) * D) + c);
                    *reinterpret_cast<float4 *>(smem + SM.stage_dec + (size_t)r * D * 4 + 16 * c) = w;
                }
            }
            if (tid < kChunk) {
                const bool in = tid < nt;
                s_beta[tid] = in ? A.beta[in_row(t0 + tid)] : 0.f;
                s_alpha[tid] = (in && !F.kda) ? A.decay[in_row(t0 + tid)] : 1.f;
            }
        }
        __syncthreads();
        const float *dec = reinterpret_cast<const float *>(smem + SM.stage_dec);
        auto a_of = [&](int x, int i) -> float {
            return F.kda ? (SM.dec_staged ? dec[x * D + i] : A.decay[in_row(t0 + x) * D + i]) : s_alpha[x];
        };
        auto in_of = [&](uint32_t base, int x, int i) -> float {
            return load_in(smem + base + (size_t)x * qkv, i, F.bf16_in);
        };

        // ---- gate products G[x][i] (tokens t0+1 .. t0+x) and the chunk
        // length: the first token whose product falls below the range ends it
        if (tid < D) {
            float g = 1.f;
            int viol = nt;
            G[tid] = 1.f;
#pragma unroll 1
            for (int x0 = 1; x0 < nt; x0 += 8) {
                float av[8];
#pragma unroll
                for (int y = 0; y < 8; ++y) av[y] = x0 + y < nt ? a_of(x0 + y, tid) : 1.f;
#pragma unroll
                for (int y = 0; y < 8; ++y) {
                    g *= av[y];
                    if (x0 + y < nt) {
                        G[(x0 + y) * D + tid] = g;
                        if (viol == nt && !(g >= kMinChunkGate)) viol = x0 + y;
                    }
                }
            }
            if (viol < kChunk) atomicMin(s_n, viol);
        }
        __syncthreads();
        const int n = min(*s_n, nt);
        // the state's scale at the chunk end: the last product, times the next
        // chunk's first gate (applied to S and to Kbar)
        if (tid < D) s_gs[tid] = G[(n - 1) * D + tid] * (t0 + n < len ? gate(t0 + n, tid) : 1.f);
        // the next chunk's rows into L2 while this one runs (a prefetch moves
        // no data the kernel relies on); threads 128.. are free here
        if (tid >= D && tid < D + kChunk && t0 + n + (tid - D) < len) {
            const size_t r = in_row(t0 + n + (tid - D));
            bulk_prefetch_l2(static_cast<const uint8_t *>(A.q) + r * qkv, qkv);
            bulk_prefetch_l2(static_cast<const uint8_t *>(A.k) + r * qkv, qkv);
            bulk_prefetch_l2(static_cast<const uint8_t *>(A.v) + r * qkv, qkv);
            if (F.kda) bulk_prefetch_l2(A.decay + r * D, (uint32_t)D * 4u);
        }

        // ---- X = [Kt; Qt] (128 x 128) and Kh (64 x 128), K-major tiles; a
        // task is one row and four consecutive key channels
#pragma unroll 4
        for (int e = tid; e < 2 * kChunk * (D / 4); e += kGroup) {
            const int qside = e >= kChunk * (D / 4), ee = e - (qside ? kChunk * (D / 4) : 0);
            const int x = ee >> 5, i = 4 * (ee & 31);
            float4 g4 = make_float4(1.f, 1.f, 1.f, 1.f), v4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (x < n) {
                g4 = *reinterpret_cast<const float4 *>(G + x * D + i);
                const uint32_t base = qside ? SM.stage_q : SM.stage_k;
                v4 = make_float4(in_of(base, x, i), in_of(base, x, i + 1), in_of(base, x, i + 2), in_of(base, x, i + 3));
            }
            const float4 t4 = make_float4(to_tf32(v4.x * g4.x), to_tf32(v4.y * g4.y), to_tf32(v4.z * g4.z),
                                          to_tf32(v4.w * g4.w));
            *reinterpret_cast<float4 *>(RX + sw128_off(qside ? 64 + x : x, i, 128)) = t4;
            if (!qside)
                *reinterpret_cast<float4 *>(RK + sw128_off(x, i, 64)) =
                    make_float4(to_tf32(v4.x * __frcp_rn(g4.x)), to_tf32(v4.y * __frcp_rn(g4.y)),
                                to_tf32(v4.z * __frcp_rn(g4.z)), to_tf32(v4.w * __frcp_rn(g4.w)));
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
                const int t = j & 63;
                const float bt = s_beta[t];
#pragma unroll
                for (int x = 0; x < 16; x += 4) {
                    const int s0 = c0 + x;
                    float4 o;
                    if (j < 64) {
                        o.x = (s0 < t && t < n) ? bt * v[x] : 0.f;
                        o.y = (s0 + 1 < t && t < n) ? bt * v[x + 1] : 0.f;
                        o.z = (s0 + 2 < t && t < n) ? bt * v[x + 2] : 0.f;
                        o.w = (s0 + 3 < t && t < n) ? bt * v[x + 3] : 0.f;
                        *reinterpret_cast<float4 *>(Lb + t * kChunk + s0) = o;
                    } else {
                        o.x = to_tf32((s0 <= t && t < n) ? v[x] : 0.f);
                        o.y = to_tf32((s0 + 1 <= t && t < n) ? v[x + 1] : 0.f);
                        o.z = to_tf32((s0 + 2 <= t && t < n) ? v[x + 2] : 0.f);
                        o.w = to_tf32((s0 + 3 <= t && t < n) ? v[x + 3] : 0.f);
                        *reinterpret_cast<float4 *>(RX + 49152 + sw128_off(t, s0, 64)) = o;
                    }
                }
            }
        }
        __syncthreads();
        unit_lower_inverse(Lb, Tb, s_M, tid);
        // Tinv as the B operand of U^T = RHS^T Tinv^T (rows t, K = s)
        for (int e = tid; e < kChunk * kChunk / 4; e += kGroup) {
            const int t = e >> 4, s0 = 4 * (e & 15);
            const float4 w = *reinterpret_cast<const float4 *>(Tb + t * kChunk + s0);
            *reinterpret_cast<float4 *>(RX + 32768 + sw128_off(t, s0, 64)) =
                make_float4(to_tf32(w.x), to_tf32(w.y), to_tf32(w.z), to_tf32(w.w));
        }
        // RHS^T (rows j, K = s): beta_s (v_s[j] - W_s[j])
        {
            auto v_at = [&](int s_) -> float {
                return SM.v_staged ? in_of(SM.stage_v, s_, j) : load_in(A.v, in_row(t0 + s_) * D + j, F.bf16_in);
            };
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                float w[16];
                const int c0 = 32 * chalf + 16 * q;
                tmem_ld16(tlane + kColW + (uint32_t)c0, w);
#pragma unroll
                for (int x = 0; x < 16; x += 4) {
                    float r[4];
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        const int s_ = c0 + x + y;
                        r[y] = to_tf32(s_ < n ? s_beta[s_] * (v_at(s_) - w[x + y]) : 0.f);
                    }
                    *reinterpret_cast<float4 *>(RX + sw128_off(j, c0 + x, 128)) = make_float4(r[0], r[1], r[2], r[3]);
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
                for (int x = 0; x < 16; x += 4)
                    *reinterpret_cast<float4 *>(RK + sw128_off(j, c0 + x, 128)) =
                        make_float4(to_tf32(u[x]), to_tf32(u[x + 1]), to_tf32(u[x + 2]), to_tf32(u[x + 3]));
            }
            // Kbar[s][i] = k_s,i (G_last,i / G_s,i) (next gate); a task is one
            // key channel and four consecutive tokens
#pragma unroll 4
            for (int e = tid; e < D * (kChunk / 4); e += kGroup) {
                const int i = e & 127, s0 = 4 * (e >> 7);
                const float gl = s_gs[i];
                float r[4];
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const int s_ = s0 + y;
                    r[y] = to_tf32(s_ < n ? in_of(SM.stage_k, s_, i) * (gl * __frcp_rn(G[s_ * D + i])) : 0.f);
                }
                *reinterpret_cast<float4 *>(RX + sw128_off(i, s0, 128)) = make_float4(r[0], r[1], r[2], r[3]);
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
