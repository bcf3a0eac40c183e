// lq_multi.cuh -- T consecutive decode tokens per (slot, head) in one launch
// (sm_100a), the compact state read once.
//
// Sources: news post "Linear attention has to move state every token it
// generates; LeapQuant compresses it to 8-bit without losing accuracy",
// per-window paragraph (the window-start state is fixed and every token's
// update is an FP32 rank-one pair); the step itself is the one of the
// single-token kernel (lq_decode.cuh).
//
// Token t of a head needs a_t = S'_t^T k_t and b_t = S'_t^T q_t.  Of these,
// only the terms of the pairs that the launch's own earlier tokens append
// depend on earlier outputs (through u); the decay products, the
// window-frame keys khat_t and the decayed, quantized vectors x_t are known
// from the inputs alone.  So per head:
//  * the prep warp forms the vectors of all T tokens at once and writes each
//    token's khat into its pair slot in the stage;
//  * the consumers run the dot products of every (pair, token) and
//    (compensator column, token) combination as one batch of 8-lane jobs,
//    then the dual GEMV of each token against the codes held in registers
//    (one pass over the codes per token, no reload);
//  * thread j, which owns value column j, then adds the buffered pairs of
//    all tokens together (T independent FMA chains) and finally walks the
//    tokens in order, adding the launch's own pairs with the u of the
//    earlier tokens it computed itself, with no barrier between tokens.
// Every token runs the single-token kernel's arithmetic in the same order
// (chunk sums, quantization scale and column terms, row compensators, then
// the pairs in buffer order), so outputs and blob bytes equal those of T
// single-token launches.
//
// A decay product that leaves the window frame's range moves the frame
// (rebase_frame), which rescales the keys of the pairs already buffered:
// the prep warp then ends the batch before that token (a "segment"), waits
// until the consumers have committed it, moves the frame and goes on with a
// new segment.  A token with an invalid gate ends the head: the tokens
// before it commit, it and the later ones are skipped with the RANGE bit.
#pragma once

#include "lq_decode.cuh"

namespace lq {

// Prep buffer of one segment, sized by the launch's T:
//   info [16 words] | kq f32 [T] | row / column compensator lists u32 [16]
//   each | column -> column-compensator map int8 [D] | decay products after
//   the segment's last token f32 [D] | y f32 [T][2D] | x int16 [T][2D]
//   | chunk scales f32 [T][2 D/16]
struct MultiPrep {
    uint32_t kq, rowc, colc, colmap, g, y, X, sc, bytes;
};

__host__ __device__ inline MultiPrep multi_prep(int D, int T) {
    MultiPrep P;
    P.kq = 64;
    P.rowc = align_up(P.kq + 4u * (uint32_t)T, 16);
    P.colc = P.rowc + 64;
    P.colmap = P.colc + 64;
    P.g = align_up(P.colmap + (uint32_t)D, 16);
    P.y = P.g + 4u * (uint32_t)D;
    P.X = P.y + 8u * (uint32_t)D * (uint32_t)T;
    P.sc = P.X + 4u * (uint32_t)D * (uint32_t)T;
    P.bytes = align_up(P.sc + 8u * (uint32_t)(D / 16) * (uint32_t)T, 128);
    return P;
}

// info words of a segment
constexpr int kSegT0 = 0, kSegT1 = 1, kSegLast = 2, kSegCount = 3, kSegNrow = 4, kSegNcol = 5, kSegBits = 6;

// barriers (8 x 8) + control (128) | chunk sums float2 [D/16][D+1] | prep
// buffers [2] | pair dots float2 [T][kDotSlots] | column dots float2
// [T][kMaxComp] | copy-warp batch: blob and count [2][32], beta and gate
// [2][T][32]
__host__ __device__ inline uint32_t multi_fixed_smem(int D, int T) {
    return align_up(128u + 8u * (uint32_t)(D / 16) * (uint32_t)(D + 1) + 2u * multi_prep(D, T).bytes +
                        8u * (uint32_t)T * (uint32_t)(kDotSlots + kMaxComp) + 256u + 256u * (uint32_t)T,
                    128u);
}

inline uint32_t multi_smem_bytes(int D, const Layout &L, const Flags &F, int tokens) {
    return multi_fixed_smem(D, tokens) +
           (uint32_t)kDecodeStages * decode_stage(L, D, F.window, F.bf16_in, F.kda, tokens).bytes;
}

// NTM: the largest T the instance takes (4 or 8), which sizes the per-token
// register arrays of the consumers.
template <int D, int BITS, bool SLOTS, int NTM>
__global__ void __launch_bounds__(D + 64, 3) decode_tokens_kernel(DecodeArgs A) {
    static_assert(NTM <= kMaxTokens, "token bound");
    constexpr int NC = D;        // consumer threads
    constexpr int LPR = D / 16;  // threads per row, one 16-key chunk each
    constexpr int RPT = D / 16;  // rows per thread
    constexpr int GB = group_bytes<BITS>();
    constexpr int NCH = D / 16;
    constexpr int KPJ = D / 8;   // keys per lane in a dot-product job
    constexpr int PSTR = D + 1;
    constexpr int NJ = NC / 8;   // dot-product jobs per pass
    constexpr int KPL = D / 32;  // keys per lane of the prep warp
    constexpr int LPC = 16 / KPL;
    constexpr int BIAS = BITS == 8 ? 0 : (BITS == 6 ? 32 : 8);
    constexpr int COPY_WARP = NC / 32, PREP_WARP = NC / 32 + 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Layout L = A.L;
    const Flags F = A.F;
    const int T = A.tokens;
    const DecodeStage SG = decode_stage(L, D, F.window, F.bf16_in, F.kda, T);
    const MultiPrep MP = multi_prep(D, T);
    const int G = gridDim.x;
    const int n_mine = (A.num_heads - (int)blockIdx.x + G - 1) / G;
    auto blob_of = [](const SlotMap &m, int h) { return SLOTS ? m.blob(h) : h; };
    // input / output row of token t of work item h: ((h / H) T + t) H + h % H
    auto tok_row = [&](size_t h, int t) -> size_t {
        const int H = A.map.heads;
        return h + ((size_t)((int)h / H) * (size_t)(T - 1) + (size_t)t) * (size_t)H;
    };

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);  // [2] stage landed
    uint64_t *empty = full + 2;                           // [2] consumers done with the stage
    uint64_t *pfull = empty + 2;                          // [2] prep of the segment done
    uint64_t *pempty = pfull + 2;                         // [2] consumers done with the segment
    volatile uint32_t *s_abort = reinterpret_cast<volatile uint32_t *>(smem + 120);
    float2 *s_part = reinterpret_cast<float2 *>(smem + 128);  // chunk sums [LPR][PSTR]
    uint8_t *s_pb = reinterpret_cast<uint8_t *>(s_part + LPR * PSTR);
    float2 *s_dot = reinterpret_cast<float2 *>(s_pb + 2 * MP.bytes);  // [T][kDotSlots]
    float2 *s_cdot = s_dot + (size_t)T * kDotSlots;                   // [T][kMaxComp]
    uint32_t *s_cnt = reinterpret_cast<uint32_t *>(s_cdot + (size_t)T * kMaxComp);
    int *s_bidx = reinterpret_cast<int *>(s_cnt + 32);
    float *s_bbeta = reinterpret_cast<float *>(s_bidx + 32);  // [T][32]
    float *s_balpha = s_bbeta + 32 * T;                       // [T][32]
    uint8_t *stages = smem + multi_fixed_smem(D, T);

    if (tid == 0) {
        for (int s = 0; s < kDecodeStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NC / 32);
            mbar_init(&pfull[s], 32);
            mbar_init(&pempty[s], NC / 32);
        }
        *s_abort = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0 && !SLOTS) {
        // a prefetch changes no data: pull the first two blobs into L2 while
        // the previous kernel drains
        for (int it = 0; it < 2 && it < n_mine; ++it)
            bulk_prefetch_l2(A.state + ((size_t)blockIdx.x + (size_t)it * G) * L.blob, L.pairs_off);
    }
    pdl_wait();
    pdl_trigger();

    if (warp == COPY_WARP) {
        // ------------------------------------------------ copy warp
        for (int base = 0; base < n_mine; base += 32) {
            const int i = base + lane;
            if (i < n_mine) {
                const size_t h = blockIdx.x + (size_t)i * G;
                const int b = blob_of(A.map, (int)h);
                s_bidx[lane] = b;
                s_cnt[lane] = b >= 0 ? *reinterpret_cast<const uint32_t *>(A.state + b * L.blob + kHdrCount) : 0u;
                // beta and the GDN gate of every token, 32 heads at a time
                float bt[kMaxTokens], at[kMaxTokens];
#pragma unroll
                for (int t = 0; t < kMaxTokens; ++t)
                    if (t < T) {
                        const size_t r = tok_row(h, t);
                        bt[t] = A.beta[r];
                        at[t] = F.kda ? 1.f : A.decay[r];
                    }
#pragma unroll
                for (int t = 0; t < kMaxTokens; ++t)
                    if (t < T) {
                        s_bbeta[t * 32 + lane] = bt[t];
                        s_balpha[t * 32 + lane] = at[t];
                    }
            }
            __syncwarp();
            if (lane == 0) {
                const int nb = min(32, n_mine - base);
                for (int x = 0; x < nb && !*s_abort; ++x) {
                    const int it = base + x, s = it % kDecodeStages;
                    if (it >= kDecodeStages && !mbar_wait_bounded(&empty[s], ((it / kDecodeStages) - 1) & 1)) {
                        *s_abort = 1u;
                        break;
                    }
                    const size_t h = blockIdx.x + (size_t)it * G;
                    uint8_t *st = stages + (size_t)s * SG.bytes;
                    float *aux = reinterpret_cast<float *>(st + SG.aux_off);
                    for (int t = 0; t < T; ++t) {
                        aux[4 + t] = s_bbeta[t * 32 + x];
                        aux[4 + T + t] = s_balpha[t * 32 + x];
                    }
                    aux[0] = s_bidx[x] >= 0 ? 0.f : 1.f;  // 1: no blob for this work item
                    if (s_bidx[x] < 0) {
                        mbar_arrive_expect_tx(&full[s], 0u);
                        continue;
                    }
                    const uint8_t *blob = A.state + (size_t)s_bidx[x] * L.blob;
                    const uint32_t in_bytes = (uint32_t)T * (3 * SG.qkv_bytes + (F.kda ? (uint32_t)D * 4u : 0u));
                    const uint32_t cnt = s_cnt[x];
                    const uint32_t cc = cnt < (uint32_t)F.window ? cnt : 0u;
                    const uint32_t pbytes = cc * L.pair_bytes;
                    mbar_arrive_expect_tx(&full[s], L.codes_off + pbytes + in_bytes);
                    bulk_g2s(st, blob, L.codes_off, &full[s]);
                    if (pbytes) bulk_g2s(st + SG.pairs_at, blob + L.pairs_off, pbytes, &full[s]);
                    for (int t = 0; t < T; ++t) {
                        const size_t r = tok_row(h, t);
                        const size_t qo = r * (size_t)SG.qkv_bytes;
                        uint8_t *in = st + SG.in_off + (size_t)t * 3 * SG.qkv_bytes;
                        bulk_g2s(in, static_cast<const uint8_t *>(A.q) + qo, SG.qkv_bytes, &full[s]);
                        bulk_g2s(in + SG.qkv_bytes, static_cast<const uint8_t *>(A.k) + qo, SG.qkv_bytes, &full[s]);
                        bulk_g2s(in + 2 * SG.qkv_bytes, static_cast<const uint8_t *>(A.v) + qo, SG.qkv_bytes,
                                 &full[s]);
                        if (F.kda)
                            bulk_g2s(st + SG.dec_off + (size_t)t * D * 4, A.decay + r * D, (uint32_t)D * 4u, &full[s]);
                    }
                }
            }
            __syncwarp();
        }
        return;
    }

    if (warp == PREP_WARP) {
        // ------------------------------------------------ prep warp
        // Per head: header checks and compensator lists, then token by token
        // the decay product, y = g . k and g . q, khat = k / g (into the
        // token's pair slot of the stage), x = sm . y quantized per 16-key
        // chunk to int16, and k . q.  Lane l takes keys KPL*l .. +KPL-1.
        int step = 0;  // segments published so far
        const int i0 = KPL * lane;
        for (int it = 0; it < n_mine; ++it) {
            const int s = it % kDecodeStages;
            uint8_t *st = stages + (size_t)s * SG.bytes;
            if (!mbar_wait_bounded(&full[s], (uint32_t)(it / kDecodeStages) & 1u)) {
                if (lane == 0) *s_abort = 1u;
                return;  // the consumers time out on their own wait
            }
            const uint4 hdr = *reinterpret_cast<const uint4 *>(st);  // count, status, ncomp, magic
            const uint32_t ncomp = hdr.z;
            const bool inl = lane < (int)min(ncomp, (uint32_t)kMaxComp);
            const uint32_t m = inl ? reinterpret_cast<const uint32_t *>(st + kHdrMeta)[lane] : 0u;
            const bool iscol = inl && (m & kCompCol), isrow = inl && !(m & kCompCol);
            const unsigned colm = __ballot_sync(0xFFFFFFFFu, iscol);
            const unsigned rowm = __ballot_sync(0xFFFFFFFFu, isrow);
            const unsigned badm = __ballot_sync(0xFFFFFFFFu, inl && (m & 0x7FFFFFFFu) >= (uint32_t)D);
            const unsigned lt = (1u << lane) - 1u;
            uint32_t newbits = 0;
            if (hdr.w != kMagic || ncomp > (uint32_t)F.num_comp || hdr.x > (uint32_t)F.window || badm)
                newbits = LQ_DEV_CORRUPT;
            else if (hdr.y == 0 && hdr.x + (uint32_t)T > (uint32_t)F.window)
                newbits = LQ_DEV_WINDOW_FULL;  // the window has no room for the T pairs
            if (reinterpret_cast<const float *>(st + SG.aux_off)[0] != 0.f) newbits = kSkipItem;
            const bool run = hdr.y == 0 && newbits == 0;
            if (newbits == kSkipItem) newbits = 0;

            uint8_t *pb = nullptr;
            // a new segment: its buffer must be free (the consumers are done
            // with the segment two back), then the head's compensator lists
            auto open = [&]() -> bool {
                pb = s_pb + (size_t)(step & 1) * MP.bytes;
                if (step >= 2 && !mbar_wait_bounded(&pempty[step & 1], (uint32_t)((step - 2) >> 1) & 1u))
                    return false;
                int8_t *cmap = reinterpret_cast<int8_t *>(pb + MP.colmap);
                if (lane < D / 4) reinterpret_cast<uint32_t *>(cmap)[lane] = 0xFFFFFFFFu;
                __syncwarp();
                if (iscol) {
                    reinterpret_cast<uint32_t *>(pb + MP.colc)[__popc(colm & lt)] = (uint32_t)lane;
                    if ((m & 0x7FFFFFFFu) < (uint32_t)D) cmap[m & 0x7FFFFFFFu] = (int8_t)__popc(colm & lt);
                }
                if (isrow) reinterpret_cast<uint32_t *>(pb + MP.rowc)[__popc(rowm & lt)] = (uint32_t)lane;
                return true;
            };
            auto publish = [&](int t0, int t1, bool last, uint32_t bits) {
                if (lane == 0) {
                    uint32_t *info = reinterpret_cast<uint32_t *>(pb);
                    info[kSegT0] = (uint32_t)t0;
                    info[kSegT1] = (uint32_t)t1;
                    info[kSegLast] = last ? 1u : 0u;
                    info[kSegCount] = hdr.x + (uint32_t)t0;
                    info[kSegNrow] = (uint32_t)__popc(rowm);
                    info[kSegNcol] = (uint32_t)__popc(colm);
                    info[kSegBits] = bits;
                }
                __syncwarp();
                mbar_arrive(&pfull[step & 1]);
                ++step;
            };
            if (!open()) {
                if (lane == 0) *s_abort = 1u;
                return;
            }
            int t0 = 0, nrun = 0;
            uint32_t tokbits = 0;
            if (run) {
                const int bh = blob_of(A.map, (int)(blockIdx.x + (size_t)it * G));
                uint8_t *blob = A.state + (size_t)bh * L.blob;
                float gprev[KPL];
#pragma unroll
                for (int e = 0; e < KPL; ++e)
                    gprev[e] = F.kda ? reinterpret_cast<const float *>(st + L.g_off)[i0 + e]
                                     : *reinterpret_cast<const float *>(st + kHdrG);
                for (int t = 0; t < T; ++t) {
                    const uint8_t *in = st + SG.in_off + (size_t)t * 3 * SG.qkv_bytes;
                    float kv[KPL], qv[KPL], gn[KPL];
#pragma unroll
                    for (int e = 0; e < KPL; ++e) {
                        kv[e] = load_in(in + SG.qkv_bytes, i0 + e, F.bf16_in);
                        qv[e] = load_in(in, i0 + e, F.bf16_in);
                    }
                    if (F.kda) {
                        const float *dec = reinterpret_cast<const float *>(st + SG.dec_off + (size_t)t * D * 4);
#pragma unroll
                        for (int e = 0; e < KPL; ++e) gn[e] = gprev[e] * dec[i0 + e];
                    } else {
                        const float alpha = reinterpret_cast<const float *>(st + SG.aux_off)[4 + T + t];
#pragma unroll
                        for (int e = 0; e < KPL; ++e) gn[e] = gprev[e] * alpha;
                    }
                    bool small = false, invalid = false;
#pragma unroll
                    for (int e = 0; e < KPL; ++e) {
                        invalid |= !(gn[e] >= 0.f);
                        small |= gn[e] < kMinDecayProduct;
                    }
                    if (__any_sync(0xFFFFFFFFu, small) && !__any_sync(0xFFFFFFFFu, invalid)) {
                        // the earlier tokens' pairs take the new frame too: they
                        // must be committed (stage and blob) first
                        if (t > t0) {
                            publish(t0, t, false, 0u);
                            if (!mbar_wait_bounded(&pempty[(step - 1) & 1], (uint32_t)((step - 1) >> 1) & 1u) ||
                                !open()) {
                                if (lane == 0) *s_abort = 1u;
                                return;
                            }
                            t0 = t;
                        }
                        float f[KPL];
#pragma unroll
                        for (int e = 0; e < KPL; ++e) f[e] = (!F.kda || gn[e] < kMinDecayProduct) ? gn[e] : 1.f;
                        rebase_frame<D>(st, blob, L, SG.pairs_at, hdr.x + (uint32_t)t, hdr.z, F.f16_scale, f, lane);
#pragma unroll
                        for (int e = 0; e < KPL; ++e)
                            if (!F.kda || gn[e] < kMinDecayProduct) gn[e] = 1.f;
                    }
#pragma unroll
                    for (int e = 0; e < KPL; ++e) gprev[e] = gn[e];
                    bool bad = false;
                    float yk[KPL], yq[KPL], xk[KPL], xq[KPL];
                    float mk = 0.f, mq = 0.f, kq = 0.f;
#pragma unroll
                    for (int e = 0; e < KPL; ++e) {
                        bad |= !(gn[e] >= kMinDecayProduct);
                        yk[e] = gn[e] * kv[e];
                        yq[e] = gn[e] * qv[e];
                        const float smv = load_scale(st + L.sm_off, i0 + e, F.f16_scale);
                        xk[e] = smv * yk[e];
                        xq[e] = smv * yq[e];
                        mk = fmaxf(mk, fabsf(xk[e]));
                        mq = fmaxf(mq, fabsf(xq[e]));
                        kq = fmaf(kv[e], qv[e], kq);
                    }
                    if (__any_sync(0xFFFFFFFFu, bad)) {
                        tokbits = LQ_DEV_RANGE;  // this token and the later ones are skipped
                        break;
                    }
                    float *py = reinterpret_cast<float *>(pb + MP.y) + (size_t)t * 2 * D;
                    float *pkh = reinterpret_cast<float *>(st + SG.pairs_at + (hdr.x + (uint32_t)t) * L.pair_bytes);
                    float *pg = reinterpret_cast<float *>(pb + MP.g);
#pragma unroll
                    for (int e = 0; e < KPL; ++e) {
                        py[i0 + e] = yk[e];
                        py[D + i0 + e] = yq[e];
                        pkh[i0 + e] = __fdiv_rn(kv[e], gn[e]);  // window-start frame
                        pg[i0 + e] = gn[e];
                    }
#pragma unroll
                    for (int off = LPC / 2; off >= 1; off >>= 1) {
                        mk = fmaxf(mk, __shfl_xor_sync(0xFFFFFFFFu, mk, off));
                        mq = fmaxf(mq, __shfl_xor_sync(0xFFFFFFFFu, mq, off));
                    }
                    // int16 with scale ~32767 / (chunk max): rint(x * scale) by
                    // adding 1.5 * 2^23; chunks below 2^-100 contribute 0
                    float ik = 0.f, iq = 0.f;
                    if (mk >= 0x1p-100f) ik = mk < 0x1p100f ? 32767.f * rcp_approx(mk) : __fdiv_rn(32767.f, mk);
                    if (mq >= 0x1p-100f) iq = mq < 0x1p100f ? 32767.f * rcp_approx(mq) : __fdiv_rn(32767.f, mq);
                    int16_t *pX = reinterpret_cast<int16_t *>(pb + MP.X) + (size_t)t * 2 * D;
#pragma unroll
                    for (int e = 0; e < KPL; ++e) {
                        const float2 q2 = __ffma2_rn(make_float2(xk[e], xq[e]), make_float2(ik, iq),
                                                     make_float2(12582912.0f, 12582912.0f));
                        const int i = i0 + e, slot = (i & ~15) + xslot<BITS>(i & 15);
                        pX[slot] = (int16_t)(__float_as_uint(q2.x) & 0xFFFFu);
                        pX[D + slot] = (int16_t)(__float_as_uint(q2.y) & 0xFFFFu);
                    }
                    if (lane % LPC == 0) {
                        float *psc = reinterpret_cast<float *>(pb + MP.sc) + (size_t)t * 2 * NCH;
                        psc[lane / LPC] = ik > 0.f ? mk * (1.f / 32767.f) : 0.f;
                        psc[NCH + lane / LPC] = iq > 0.f ? mq * (1.f / 32767.f) : 0.f;
                    }
                    kq = warp_sum(kq);
                    if (lane == 0) reinterpret_cast<float *>(pb + MP.kq)[t] = kq;
                    nrun = t + 1;
                }
            }
            publish(t0, run ? nrun : 0, true, run ? tokbits : newbits);
        }
        return;
    }

    // ---------------------------------------------------- consumer threads
    // GEMV role: chunk c of rows RPT*rg + m (m < RPT); epilogue role: thread
    // j owns value column j; dot-product role: 8 lanes per job, lane kc takes
    // keys 4*kc + 32*e + (0..3).
    const int c = tid % LPR, rg = tid / LPR;
    const int kc = tid % 8, jslot = tid / 8;
    const int j = tid;
    const uint8_t *code_base = A.state + L.codes_off + c * GB;
    Group<BITS> cg[RPT];
    {
        const int b_first = n_mine > 0 ? blob_of(A.map, (int)blockIdx.x) : -1;
        if (b_first >= 0) {
            const uint8_t *cb = code_base + (size_t)b_first * L.blob;
#pragma unroll
            for (int m = 0; m < RPT; ++m) load_group<BITS>(cg[m], cb + (size_t)(RPT * rg + m) * L.row_bytes);
        }
    }
    int it = 0;
    for (int step = 0; it < n_mine; ++step) {
        const int s = it % kDecodeStages;
        uint8_t *st = stages + (size_t)s * SG.bytes;
        const uint8_t *pb = s_pb + (size_t)(step & 1) * MP.bytes;
        const size_t h = blockIdx.x + (size_t)it * G;
        const int bi = blob_of(A.map, (int)h);
        uint8_t *blob = A.state + (bi >= 0 ? (size_t)bi : 0) * L.blob;
        if (!consumer_sync_and(mbar_wait_bounded(&pfull[step & 1], (uint32_t)(step >> 1) & 1u), NC)) {
            if (tid == 0) {
                if (bi >= 0) set_status(blob, LQ_DEV_TIMEOUT);
                *s_abort = 1u;
            }
            for (int t = 0; t < T; ++t) A.out[tok_row(h, t) * D + tid] = 0.f;
            break;
        }
        const uint32_t *info = reinterpret_cast<const uint32_t *>(pb);
        const int t0 = (int)info[kSegT0], t1 = (int)info[kSegT1];
        const bool last = info[kSegLast] != 0u;
        const uint32_t count_s = info[kSegCount];
        const int nrow = (int)info[kSegNrow], ncol = (int)info[kSegNcol];
        const uint32_t newbits = info[kSegBits];
        // codes of the next work item, loaded during this one's last GEMV
        bool has_next = last && it + 1 < n_mine;
        const uint8_t *next_codes = code_base + (h + G) * (size_t)L.blob;
        if constexpr (SLOTS) {
            const int bn = has_next ? A.map.blob((int)h + G) : -1;
            has_next = bn >= 0;
            next_codes = code_base + (size_t)(has_next ? bn : 0) * L.blob;
        }

        if (t1 > t0) {
            const int nt = t1 - t0;
            const float *aux = reinterpret_cast<const float *>(st + SG.aux_off);
            float *pairs = reinterpret_cast<float *>(st + SG.pairs_at);
            const float *cvec = reinterpret_cast<const float *>(st + L.cvec_off);
            const uint32_t *meta = reinterpret_cast<const uint32_t *>(st + kHdrMeta);
            const uint32_t *colc = reinterpret_cast<const uint32_t *>(pb + MP.colc);
            const uint32_t *rowc = reinterpret_cast<const uint32_t *>(pb + MP.rowc);
            const float *py_all = reinterpret_cast<const float *>(pb + MP.y);

            // ---- dot products: token t0 + tt against the pairs m < count_s +
            // tt (its launch's earlier keys included), then the compensator
            // columns; tt (count_s + ncol) + tt (tt - 1) / 2 jobs come before
            // those of token t0 + tt
            const int nb = (int)count_s + ncol;
            const int J = nt * nb + nt * (nt - 1) / 2;
            for (int jb0 = 0; jb0 < J; jb0 += NJ) {
                const int jb = jb0 + jslot;
                const bool live = jb < J;
                int tt = 0;
#pragma unroll
                for (int x = 1; x < NTM; ++x)
                    if (x < nt && jb >= x * nb + x * (x - 1) / 2) tt = x;
                const int r = jb - (tt * nb + tt * (tt - 1) / 2);
                const int P = (int)count_s + tt;  // pair jobs of this token
                float2 ak2 = make_float2(0.f, 0.f), aq2 = make_float2(0.f, 0.f);
                if (live) {
                    const float *vec = r < P ? pairs + (size_t)r * 2 * D : cvec + (size_t)colc[r - P] * D;
                    const float *py = py_all + (size_t)(t0 + tt) * 2 * D;
#pragma unroll
                    for (int e = 0; e < KPJ / 4; ++e) {
                        const int o = 4 * kc + 32 * e;
                        const float4 x4 = *reinterpret_cast<const float4 *>(vec + o);
                        const float4 a4 = *reinterpret_cast<const float4 *>(py + o);
                        const float4 b4 = *reinterpret_cast<const float4 *>(py + D + o);
                        ak2 = __ffma2_rn(make_float2(x4.x, x4.y), make_float2(a4.x, a4.y), ak2);
                        ak2 = __ffma2_rn(make_float2(x4.z, x4.w), make_float2(a4.z, a4.w), ak2);
                        aq2 = __ffma2_rn(make_float2(x4.x, x4.y), make_float2(b4.x, b4.y), aq2);
                        aq2 = __ffma2_rn(make_float2(x4.z, x4.w), make_float2(b4.z, b4.w), aq2);
                    }
                }
                float dk_ = ak2.x + ak2.y, dq_ = aq2.x + aq2.y;
#pragma unroll
                for (int off = 4; off >= 1; off >>= 1) {
                    dk_ += __shfl_xor_sync(0xFFFFFFFFu, dk_, off);
                    dq_ += __shfl_xor_sync(0xFFFFFFFFu, dq_, off);
                }
                if (live && kc == 0) {
                    const int t = t0 + tt;
                    if (r < P) s_dot[(size_t)t * kDotSlots + r] = make_float2(dk_, dq_);
                    else s_cdot[(size_t)t * kMaxComp + (r - P)] = make_float2(dk_, dq_);
                }
            }

            consumer_sync(NC);  // every job's dot product is in place
            // ---- per token: dual GEMV over the codes in registers, then
            // thread j forms its column's sum up to the row compensators.
            // The chunk sums of rows 32w .. 32w + 31 all come from warp w,
            // which owns those rows in the epilogue: warp-level syncs suffice.
            const float qsj = load_scale(st + L.qs_off, j, F.f16_scale);
            const int cm = reinterpret_cast<const int8_t *>(pb + MP.colmap)[j];
            float2 abv[NTM];
#pragma unroll
            for (int x = 0; x < NTM; ++x) abv[x] = make_float2(0.f, 0.f);
            for (int tt = 0; tt < nt; ++tt) {
                const int t = t0 + tt;
                uint32_t Xk[8], Xq[8];
                {
                    const uint8_t *px = pb + MP.X + (size_t)t * 4 * D;
                    const uint4 *xk4 = reinterpret_cast<const uint4 *>(px + 32 * c);
                    const uint4 *xq4 = reinterpret_cast<const uint4 *>(px + 2 * D + 32 * c);
                    const uint4 a0 = xk4[0], a1 = xk4[1], b0 = xq4[0], b1 = xq4[1];
                    Xk[0] = a0.x; Xk[1] = a0.y; Xk[2] = a0.z; Xk[3] = a0.w;
                    Xk[4] = a1.x; Xk[5] = a1.y; Xk[6] = a1.z; Xk[7] = a1.w;
                    Xq[0] = b0.x; Xq[1] = b0.y; Xq[2] = b0.z; Xq[3] = b0.w;
                    Xq[4] = b1.x; Xq[5] = b1.y; Xq[6] = b1.z; Xq[7] = b1.w;
                }
                const float *psc = reinterpret_cast<const float *>(pb + MP.sc) + (size_t)t * 2 * NCH;
                const float2 sc2 = make_float2(psc[c], psc[NCH + c]);
                int biask = 0, biasq = 0;
                if constexpr (BIAS != 0) {
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        biask = dp2a_lo_ss(Xk[x], 0x00000101u, biask);
                        biasq = dp2a_lo_ss(Xq[x], 0x00000101u, biasq);
                    }
                    biask *= BIAS;
                    biasq *= BIAS;
                }
                const bool ld = has_next && tt == nt - 1;
#pragma unroll
                for (int m = 0; m < RPT; ++m) {
                    int ak = -biask, aq = -biasq;
                    group_dot<BITS>(cg[m], Xk, Xq, ak, aq);
                    if (ld) load_group<BITS>(cg[m], next_codes + (size_t)(RPT * rg + m) * L.row_bytes);
                    s_part[c * PSTR + RPT * rg + m] = __fmul2_rn(make_float2((float)ak, (float)aq), sc2);
                }
                __syncwarp();
                float2 ab = s_part[j];
#pragma unroll
                for (int x = 1; x < LPR; ++x) ab = __fadd2_rn(ab, s_part[x * PSTR + j]);
                const float2 ca = cm >= 0 ? s_cdot[(size_t)t * kMaxComp + cm] : make_float2(0.f, 0.f);
                ab = __ffma2_rn(ab, make_float2(qsj, qsj), ca);
                const float *py = py_all + (size_t)t * 2 * D;
                for (int r = 0; r < nrow; ++r) {
                    const uint32_t cc = rowc[r];
                    const float wj = cvec[(size_t)cc * D + j];
                    const int i0 = (int)(meta[cc] & 0x7FFFFFFFu);
                    ab = __ffma2_rn(make_float2(py[i0], py[D + i0]), make_float2(wj, wj), ab);
                }
#pragma unroll
                for (int x = 0; x < NTM; ++x)
                    if (x == tt) abv[x] = ab;
                __syncwarp();  // the warp's chunk sums are free again
            }

            // ---- the pairs buffered before the segment, every token at once
            for (uint32_t m = 0; m < count_s; ++m) {
                const float uj = pairs[(size_t)m * 2 * D + D + j];
#pragma unroll
                for (int x = 0; x < NTM; ++x)
                    if (x < nt) abv[x] = __ffma2_rn(s_dot[(size_t)(t0 + x) * kDotSlots + m], make_float2(uj, uj), abv[x]);
            }
            // ---- token by token: the segment's own pairs, u, o, the new pair
            float uv[NTM];
#pragma unroll
            for (int x = 0; x < NTM; ++x) {
                uv[x] = 0.f;
                if (x < nt) {
                    const int t = t0 + x;
                    float2 ab = abv[x];
#pragma unroll
                    for (int y = 0; y < x; ++y)
                        ab = __ffma2_rn(s_dot[(size_t)t * kDotSlots + count_s + y], make_float2(uv[y], uv[y]), ab);
                    const float u =
                        aux[4 + t] * (load_in(st + SG.in_off + ((size_t)t * 3 + 2) * SG.qkv_bytes, j, F.bf16_in) - ab.x);
                    const float kq = reinterpret_cast<const float *>(pb + MP.kq)[t];
                    A.out[tok_row(h, t) * D + j] = fmaf(kq, u, ab.y);
                    uv[x] = u;
                    const size_t m = count_s + (uint32_t)x;
                    float *sp = pairs + m * 2 * D;
                    float *bp = reinterpret_cast<float *>(blob + L.pairs_off + m * L.pair_bytes);
                    bp[D + j] = u;
                    bp[j] = sp[j];
                    sp[D + j] = u;  // a later segment of this head reads it
                }
            }
            const float *pg = reinterpret_cast<const float *>(pb + MP.g);
            if (F.kda) reinterpret_cast<float *>(blob + L.g_off)[j] = pg[j];
            if (tid == 0) {
                *reinterpret_cast<uint32_t *>(blob + kHdrCount) = count_s + (uint32_t)nt;
                if (!F.kda) *reinterpret_cast<float *>(blob + kHdrG) = pg[0];
            }
        } else if (has_next) {
#pragma unroll
            for (int m = 0; m < RPT; ++m) load_group<BITS>(cg[m], next_codes + (size_t)(RPT * rg + m) * L.row_bytes);
        }
        if (last) {
            for (int t = t1; t < T; ++t) A.out[tok_row(h, t) * D + tid] = 0.f;
            if (tid == 0 && newbits && bi >= 0) set_status(blob, newbits);
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&pempty[step & 1]);  // this warp is done with the segment
            if (last) mbar_arrive(&empty[s]);
        }
        if (last) ++it;
    }
}

}  // namespace lq
