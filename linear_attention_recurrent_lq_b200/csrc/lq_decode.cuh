// lq_decode.cuh -- one decode token of a LeapQuant low-bit state (sm_100a).
//
// Per (slot, head) the window-start state is fixed inside a window and every
// token's update is kept as an FP32 rank-one pair (news post "Linear
// attention has to move state every token it generates; LeapQuant compresses
// it to 8-bit without losing accuracy", per-window paragraph; "LeapQuant:
// Efficient Linear Attention with Accurate Recurrent State Quantization",
// abstract).  With g_t the decay product since the window start and
//     S'_t = diag(g_t) (S_base + sum_{m<t} khat_m u_m^T),
// the step needs a = S'^T k and b = S'^T q.  Both fold the decay into the
// vectors:  a = S_base^T (g_t . k) + sum_m (khat_m . (g_t . k)) u_m, likewise
// b with q.  The base part is a fused dequantize + dual GEMV over the codes
// (R_ij = sm_i qs_j C_ji, so R^T y = qs . (C (sm . y))); compensators (the
// outlier lines kept in FP32) and buffered pairs add rank-one terms.  Then
//     u_t = beta (v - a),   o_t = b + (k . q) u_t,
// and the pair (khat_t = k / g_t, u_t) is appended.
//
// Persistent kernel, one CTA = D consumer threads + a copy warp + a prep
// warp, each CTA walking a strided list of (slot, head) blobs:
//  * the copy warp bulk-copies each blob's small, variable-size parts
//    (header, decay product, scales, compensators, the buffered pairs) and the
//    token's q, k, v into a two-stage shared-memory ring (mbarrier-tracked);
//  * the prep warp, one head ahead, checks the header and forms the decayed
//    and quantized vectors of the head (and moves the window frame when a
//    decay product leaves its range);
//  * the codes (the bulk of the state) go straight from global memory into
//    registers: a consumer thread holds its D/16 16-code groups of the current
//    blob and, as it consumes group m, issues the load of group m of the next
//    blob, so code traffic is always in flight;
//  * the GEMV runs on the integer pipe: x_k, x_q are quantized per 16-key
//    chunk to int16 with the chunk's own scale (error <= 2^-16 of the chunk's
//    largest entry) and dp2a multiplies two int16 entries by two int8 codes,
//    accumulating exactly in int32;
//  * a row is split over D/16 threads (one chunk each); the chunk sums meet in
//    shared memory, where thread j adds up row j and then the compensator and
//    pair terms before forming u_j and o_j.  Waits on the ring sleep on the
//    mbarrier and give up after a bounded time; a consumer warp hands the
//    stage back as soon as it is done with it.
#pragma once

#include "lq_common.cuh"

namespace lq {

struct DecodeArgs {
    uint8_t *state;
    Layout L;
    Flags F;
    const void *q, *k, *v;
    const float *beta, *decay;
    float *out;
    int num_heads;  // work items: N * H, or active rows * H with a slot map
    SlotMap map;    // heads = H always; slots only in the slot-list instance
    int tokens;     // T consecutive tokens per work item (multi-token instance)
    uint32_t flags; // kEarlyState (plain rows only)
};

// Call flag of the plain decode: the kernel enqueued just before this one on
// the stream does not write the state (it may still be running).  The
// decode then stages its first blob and loads its codes before it waits for
// that kernel; the token's inputs are still read only after the wait.
constexpr uint32_t kEarlyState = 0x1u;
// Heads a CTA stages before that wait.  One, not both stages: every CTA
// requests at once, and the head scalars read after the wait (beta, gates,
// window counts) queue behind that burst; a burst of one head per CTA lets
// the first head start sooner (measured 14.2 against 14.4 us per launch at
// B = 64, H = 32).
constexpr int kEarlyHeads = 1;

constexpr int kDotSlots = kMaxWindow + kMaxComp;
constexpr int kMaxTokens = 8;  // tokens per work item in one multi-token launch

// One ring stage: [blob prefix up to the codes][buffered pairs][q k v per
// token][KDA decay per token][aux].  aux: f32 [0] 1 = the work item has no
// blob, [4 + t] beta of token t, [4 + T + t] GDN alpha of token t.
struct DecodeStage {
    uint32_t pairs_at, in_off, qkv_bytes, dec_off, aux_off, bytes;
};

__host__ __device__ inline DecodeStage decode_stage(const Layout &L, int D, int window, int bf16,
                                                    int kda, int tokens = 1) {
    DecodeStage S;
    S.pairs_at = L.codes_off;  // the prefix [0, codes_off) is copied as is
    // pairs buffered before the launch plus those its tokens append: at most
    // W - 1 for one token; a multi-token launch also stages its last key
    S.in_off = align_up(S.pairs_at + (uint32_t)(tokens > 1 ? window : window - 1) * L.pair_bytes, 128);
    S.qkv_bytes = align_up((uint32_t)D * (bf16 ? 2u : 4u), 16);
    S.dec_off = S.in_off + 3u * S.qkv_bytes * (uint32_t)tokens;
    S.aux_off = align_up(S.dec_off + (kda ? (uint32_t)D * 4u * (uint32_t)tokens : 0u), 16);
    S.bytes = align_up(S.aux_off + 16 + 8 * (uint32_t)tokens, 128);
    return S;
}

// Per-head scratch written by the prep warp one head ahead of the consumers
// (two of them, by head parity):
//   y [2D] f32 | X [2D] int16 | chunk scales [2*D/16] | khat [D] | g [D]
//   | column terms float2 [D] | row / column compensator lists [2*16] | info [8]
// Move the window frame of one head to the current token.  Within a window
// the state is diag(g)(S_base + sum_m khat_m u_m^T); when the decay product
// g_i of key channel i falls below kMinDecayProduct, channel i's factor
// f_i = g_i goes into what is stored instead: the smoothing scale sm_i (the
// base row i, rounded to the scale's storage format), the compensator
// entries of row i, and khat_m[i] of every buffered pair; g_i restarts at 1.
// Exact algebra up to one rounding per stored value; the base part taken
// along is below 2^-96 of its size at the window start.  Runs in the prep
// warp: lane l scales keys KPL*l .., f[e] its factors (1: channel kept).  The
// stage and the blob get the same values.
template <int D>
__device__ __noinline__ void rebase_frame(uint8_t *st, uint8_t *blob, const Layout &L, uint32_t pairs_at,
                                          uint32_t count, uint32_t ncomp, int f16, const float (&f)[D / 32],
                                          int lane) {
    constexpr int KPL = D / 32;
    const int i0 = KPL * lane;
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
        const int i = i0 + e;
        const float v = load_scale(st + L.sm_off, i, f16) * f[e];
        if (f16) {
            const __half hv = __float2half_rn(v);
            reinterpret_cast<__half *>(st + L.sm_off)[i] = hv;
            reinterpret_cast<__half *>(blob + L.sm_off)[i] = hv;
        } else {
            reinterpret_cast<float *>(st + L.sm_off)[i] = v;
            reinterpret_cast<float *>(blob + L.sm_off)[i] = v;
        }
    }
    for (uint32_t m = 0; m < count; ++m) {
        float *ks = reinterpret_cast<float *>(st + pairs_at + (size_t)m * L.pair_bytes);
        float *kb = reinterpret_cast<float *>(blob + L.pairs_off + (size_t)m * L.pair_bytes);
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            const float v = ks[i0 + e] * f[e];
            ks[i0 + e] = v;
            kb[i0 + e] = v;
        }
    }
    const uint32_t *meta = reinterpret_cast<const uint32_t *>(st + kHdrMeta);
    for (uint32_t c = 0; c < ncomp && c < (uint32_t)kMaxComp; ++c) {
        float *vs = reinterpret_cast<float *>(st + L.cvec_off) + (size_t)c * D;
        float *vb = reinterpret_cast<float *>(blob + L.cvec_off) + (size_t)c * D;
        const uint32_t m = meta[c];
        if (m & kCompCol) {  // a value column over the keys: entry i takes f_i
#pragma unroll
            for (int e = 0; e < KPL; ++e) {
                const float v = vs[i0 + e] * f[e];
                vs[i0 + e] = v;
                vb[i0 + e] = v;
            }
        } else {  // key row r over the values: every entry takes f_r
            const int r = (int)(m & 0x7FFFFFFFu) % D;
            float fr = 1.f;
#pragma unroll
            for (int e = 0; e < KPL; ++e)
                if (r % KPL == e) fr = f[e];
            fr = __shfl_sync(0xFFFFFFFFu, fr, r / KPL);
            for (int j = lane; j < D; j += 32) {
                const float v = vs[j] * fr;
                vs[j] = v;
                vb[j] = v;
            }
        }
    }
    __syncwarp();
}

template <int D>
struct PrepBuf {
    static constexpr uint32_t y = 0, X = 8 * D, sc = 12 * D, kh = sc + 8 * (D / 16), g = kh + 4 * D,
                              cadd = g + 4 * D, rowc = cadd + 8 * D, colc = rowc + 64, info = colc + 64,
                              bytes = info + 32;
};
// info words
constexpr int kInfoRun = 0, kInfoCount = 1, kInfoNrow = 2, kInfoNcol = 3, kInfoBits = 4, kInfoKq = 5;

template <int D>
__host__ __device__ constexpr uint32_t decode_fixed_smem() {
    // barriers (6 x 8 at 0) + control (128) | chunk sums float2 [D/16][D+1] | prep buffers [2]
    // | dots float2 [kDotSlots] | producer batch [4*32]
    return align_up(128u + 8u * (D / 16) * (D + 1) + 2u * PrepBuf<D>::bytes + 8u * kDotSlots + 4u * 32u * 4u,
                    128u);
}

constexpr int kDecodeStages = 2;
// Prep-warp marker of a work item whose slot is out of range (never a status bit).
constexpr uint32_t kSkipItem = 0xFFFFFFFFu;

inline uint32_t decode_smem_bytes(int D, const Layout &L, const Flags &F, int tokens = 1) {
    const uint32_t fixed = D == 128 ? decode_fixed_smem<128>() : decode_fixed_smem<64>();
    return fixed + (uint32_t)kDecodeStages * decode_stage(L, D, F.window, F.bf16_in, F.kda, tokens).bytes;
}

__device__ __forceinline__ void consumer_sync(int n) {
    asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory");
}

__device__ __forceinline__ bool consumer_sync_or(bool pred, int n) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ bool consumer_sync_and(bool pred, int n) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ int dp2a_lo_ss(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp2a.lo.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_hi_ss(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp2a.hi.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_lo_su(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_hi_su(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Position of key (i mod 16) inside its chunk's int16 array, so that the
// int16 pairs line up with the bytes dp2a reads: natural order for 8 and 6
// bits; for 4 bits a word's low nibbles hold the even codes of 8 keys and
// its high nibbles the odd ones.
template <int BITS>
__host__ __device__ constexpr int xslot(int r) {
    if (BITS != 4) return r;
    const int q = r >> 3, w = r & 7;
    return 8 * q + ((w & 1) ? 4 + (w >> 1) : (w >> 1));
}

// One 16-code group as raw words (4 words for 8 bits, 3 for 6 bits, 2 for 4).
template <int BITS>
struct Group {
    uint32_t w[BITS == 8 ? 4 : (BITS == 6 ? 3 : 2)];
};

template <int BITS>
__device__ __forceinline__ void load_group(Group<BITS> &g, const uint8_t *p) {
    if constexpr (BITS == 8) {
        const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(p));
        g.w[0] = v.x; g.w[1] = v.y; g.w[2] = v.z; g.w[3] = v.w;
    } else if constexpr (BITS == 4) {
        const uint2 v = __ldcs(reinterpret_cast<const uint2 *>(p));
        g.w[0] = v.x; g.w[1] = v.y;
    } else {
        const uint32_t *q = reinterpret_cast<const uint32_t *>(p);
        g.w[0] = __ldcs(q); g.w[1] = __ldcs(q + 1); g.w[2] = __ldcs(q + 2);
    }
}

// Integer dot products of one 16-code group with the int16 chunk of x_k
// (Xk, 8 words) and x_q (Xq).  For 4 and 6 bits the codes are read as
// unsigned offset values (code + 8, code + 32); the caller removes
// bias * sum(X).
template <int BITS>
__device__ __forceinline__ void group_dot(const Group<BITS> &g, const uint32_t (&Xk)[8],
                                          const uint32_t (&Xq)[8], int &ak, int &aq) {
    if constexpr (BITS == 8) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            ak = dp2a_lo_ss(Xk[2 * q], g.w[q], ak);
            ak = dp2a_hi_ss(Xk[2 * q + 1], g.w[q], ak);
            aq = dp2a_lo_ss(Xq[2 * q], g.w[q], aq);
            aq = dp2a_hi_ss(Xq[2 * q + 1], g.w[q], aq);
        }
    } else if constexpr (BITS == 4) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint32_t lo = (g.w[q] & 0x0F0F0F0Fu) ^ 0x08080808u;         // codes 8q + 0,2,4,6
            const uint32_t hi = ((g.w[q] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;  // codes 8q + 1,3,5,7
            ak = dp2a_lo_su(Xk[4 * q], lo, ak);
            ak = dp2a_hi_su(Xk[4 * q + 1], lo, ak);
            ak = dp2a_lo_su(Xk[4 * q + 2], hi, ak);
            ak = dp2a_hi_su(Xk[4 * q + 3], hi, ak);
            aq = dp2a_lo_su(Xq[4 * q], lo, aq);
            aq = dp2a_hi_su(Xq[4 * q + 1], lo, aq);
            aq = dp2a_lo_su(Xq[4 * q + 2], hi, aq);
            aq = dp2a_hi_su(Xq[4 * q + 3], hi, aq);
        }
    } else {
        const uint32_t w0 = g.w[0], w1 = g.w[1], w2 = g.w[2];
        const uint32_t l[4] = {(w0 & 0x3F3F3F3Fu) ^ 0x20202020u, (w1 & 0x3F3F3F3Fu) ^ 0x20202020u,
                               (w2 & 0x3F3F3F3Fu) ^ 0x20202020u,
                               (((w0 >> 6) & 0x03030303u) | ((w1 >> 4) & 0x0C0C0C0Cu) |
                                ((w2 >> 2) & 0x30303030u)) ^ 0x20202020u};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            ak = dp2a_lo_su(Xk[2 * q], l[q], ak);
            ak = dp2a_hi_su(Xk[2 * q + 1], l[q], ak);
            aq = dp2a_lo_su(Xq[2 * q], l[q], aq);
            aq = dp2a_hi_su(Xq[2 * q + 1], l[q], aq);
        }
    }
}

// Approximate reciprocal (one MUFU op, relative error below 2^-22 for
// normal x; subnormal results flush to zero).
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, off);
    return x;
}

// SLOTS: work items reach their blobs through A.map.  EARLY (plain rows
// only, kEarlyState): the first blob's state is staged before the wait on
// the previous kernel.  Separate instances, so the plain path carries
// none of this.  (Several tokens per work item: decode_tokens_kernel.)
template <int D, int BITS, bool SLOTS, bool EARLY>
__global__ void __launch_bounds__(D + 64, SLOTS ? 3 : 0) decode_kernel(DecodeArgs A) {
    static_assert(!(EARLY && SLOTS), "early staging is for plain rows");
    constexpr int NC = D;            // consumer threads
    constexpr int LPR = D / 16;      // threads per row, one 16-key chunk each
    constexpr int RPT = D / 16;      // rows per thread (16 row groups)
    constexpr int GB = group_bytes<BITS>();
    constexpr int NCH = D / 16;      // chunks per row
    constexpr int KPJ = D / 8;       // keys per lane in the dot-product phase
    constexpr int PSTR = D + 1;      // padded row of the chunk-sum array (spreads the banks)
    constexpr int NJ = NC / 8;       // dot-product jobs per pass
    constexpr int KPL = D / 32;      // keys per lane of the prep warp
    constexpr int LPC = 16 / KPL;    // prep lanes per 16-key chunk
    constexpr int BIAS = BITS == 8 ? 0 : (BITS == 6 ? 32 : 8);
    constexpr int COPY_WARP = NC / 32, PREP_WARP = NC / 32 + 1;
    using PB = PrepBuf<D>;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Layout L = A.L;
    const Flags F = A.F;
    const DecodeStage SG = decode_stage(L, D, F.window, F.bf16_in, F.kda);
    const int G = gridDim.x;
    const int n_mine = (A.num_heads - (int)blockIdx.x + G - 1) / G;
    auto blob_of = [](const SlotMap &m, int h) { return SLOTS ? m.blob(h) : h; };

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);  // [2] stage landed
    uint64_t *empty = full + 2;                           // [2] consumers done with the stage
    uint64_t *pfull = empty + 2;                          // [2] prep of the step done
    volatile uint32_t *s_abort = reinterpret_cast<volatile uint32_t *>(smem + 120);
    float2 *s_part = reinterpret_cast<float2 *>(smem + 128);            // chunk sums [LPR][PSTR]
    uint8_t *s_pb = reinterpret_cast<uint8_t *>(s_part + LPR * PSTR);    // PrepBuf [2]
    float2 *s_dot = reinterpret_cast<float2 *>(s_pb + 2 * PB::bytes);    // (k-side, q-side) [kDotSlots]
    uint32_t *s_cnt = reinterpret_cast<uint32_t *>(s_dot + kDotSlots);  // copy-warp batch [32]
    float *s_pbeta = reinterpret_cast<float *>(s_cnt + 32);
    float *s_palpha = s_pbeta + 32;
    int *s_bidx = reinterpret_cast<int *>(s_palpha + 32);  // blob of each batch item, -1: none
    uint8_t *stages = smem + decode_fixed_smem<D>();

    if (tid == 0) {
        for (int s = 0; s < kDecodeStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NC / 32);  // one arrival per consumer warp
            mbar_init(&pfull[s], 32);       // every lane of the prep warp
        }
        *s_abort = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    // consumer roles (see below); the codes of the first head are loaded
    // before the wait in the EARLY instance
    const int c = tid % LPR, rg = tid / LPR;
    const uint8_t *code_base = A.state + L.codes_off + c * GB;
    Group<BITS> cg[RPT];
    const int b_first = n_mine > 0 ? blob_of(A.map, (int)blockIdx.x) : -1;
    if (EARLY) {
        // The previous kernel does not write this state: stage the compact
        // state and buffered pairs of the first head (count, then bulk copies
        // on the stage's barrier, without arriving) and load its codes while
        // that kernel drains.
        if (warp == COPY_WARP) {
            if (lane < kEarlyHeads && lane < n_mine)
                s_cnt[lane] = *reinterpret_cast<const uint32_t *>(A.state + ((size_t)blockIdx.x + (size_t)lane * G) *
                                                                                 L.blob + kHdrCount);
            __syncwarp();
            if (lane == 0)
                for (int x = 0; x < kEarlyHeads && x < n_mine; ++x) {
                    const uint8_t *blob = A.state + ((size_t)blockIdx.x + (size_t)x * G) * L.blob;
                    uint8_t *st = stages + (size_t)x * SG.bytes;
                    const uint32_t cc = s_cnt[x] < (uint32_t)F.window ? s_cnt[x] : 0u;
                    mbar_expect_tx(&full[x], L.codes_off + cc * L.pair_bytes);
                    bulk_g2s(st, blob, L.codes_off, &full[x]);
                    if (cc) bulk_g2s(st + SG.pairs_at, blob + L.pairs_off, cc * L.pair_bytes, &full[x]);
                }
            __syncwarp();
        } else if (warp < COPY_WARP && b_first >= 0) {
            const uint8_t *cb = code_base + (size_t)b_first * L.blob;
#pragma unroll
            for (int m = 0; m < RPT; ++m) load_group<BITS>(cg[m], cb + (size_t)(RPT * rg + m) * L.row_bytes);
        }
    } else if (tid == 0 && !SLOTS) {
        // While the previous kernel on the stream drains, start pulling this
        // CTA's first two blobs (compact state and codes) into L2.  A prefetch
        // changes no data, so it is safe whatever that kernel writes.  Not
        // through a slot list: the list would have to be read first, and that
        // read measured slower than no prefetch at all.
        for (int it = 0; it < 2 && it < n_mine; ++it)
            bulk_prefetch_l2(A.state + ((size_t)blockIdx.x + (size_t)it * G) * L.blob, L.pairs_off);
    }
    pdl_wait();
    pdl_trigger();

    if (warp == COPY_WARP) {
        // ------------------------------------------------ copy warp
        // Early instance: the token's inputs of the staged heads go out at
        // once, so their latency overlaps the reads of the window counts,
        // beta and the decays below (the stages complete with the arrivals
        // in the loop).
        if (EARLY && lane == 0)
            for (int x = 0; x < kEarlyHeads && x < n_mine; ++x) {
                const size_t h = blockIdx.x + (size_t)x * G;
                uint8_t *st = stages + (size_t)x * SG.bytes;
                mbar_expect_tx(&full[x], 3 * SG.qkv_bytes + (F.kda ? (uint32_t)D * 4u : 0u));
                const size_t qo = h * (size_t)SG.qkv_bytes;
                bulk_g2s(st + SG.in_off, static_cast<const uint8_t *>(A.q) + qo, SG.qkv_bytes, &full[x]);
                bulk_g2s(st + SG.in_off + SG.qkv_bytes, static_cast<const uint8_t *>(A.k) + qo, SG.qkv_bytes, &full[x]);
                bulk_g2s(st + SG.in_off + 2 * SG.qkv_bytes, static_cast<const uint8_t *>(A.v) + qo, SG.qkv_bytes,
                         &full[x]);
                if (F.kda) bulk_g2s(st + SG.dec_off, A.decay + h * D, (uint32_t)D * 4u, &full[x]);
            }
        for (int base = 0; base < n_mine; base += 32) {
            const int i = base + lane;
            if (i < n_mine) {
                const size_t h = blockIdx.x + (size_t)i * G;
                const int b = blob_of(A.map, (int)h);
                s_bidx[lane] = (int)b;
                s_cnt[lane] = b >= 0 ? *reinterpret_cast<const uint32_t *>(A.state + b * L.blob + kHdrCount) : 0u;
                s_pbeta[lane] = A.beta[h];
                s_palpha[lane] = F.kda ? 1.f : A.decay[h];
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
                    aux[4] = s_pbeta[x];
                    aux[5] = s_palpha[x];
                    aux[0] = s_bidx[x] >= 0 ? 0.f : 1.f;  // 1: no blob for this work item
                    if (s_bidx[x] < 0) {
                        mbar_arrive_expect_tx(&full[s], 0u);  // nothing is staged
                        continue;
                    }
                    const uint8_t *blob = A.state + (size_t)s_bidx[x] * L.blob;
                    const uint32_t in_bytes = 3 * SG.qkv_bytes + (F.kda ? (uint32_t)D * 4u : 0u);
                    if (EARLY && it < kEarlyHeads) {
                        mbar_arrive(&full[s]);  // state and inputs are on their way already
                        continue;
                    } else {
                        const uint32_t cnt = s_cnt[x];
                        const uint32_t cc = cnt < (uint32_t)F.window ? cnt : 0u;
                        const uint32_t pb = cc * L.pair_bytes;
                        mbar_arrive_expect_tx(&full[s], L.codes_off + pb + in_bytes);
                        bulk_g2s(st, blob, L.codes_off, &full[s]);
                        if (pb) bulk_g2s(st + SG.pairs_at, blob + L.pairs_off, pb, &full[s]);
                    }
                    const size_t qo = h * (size_t)SG.qkv_bytes;
                    uint8_t *in = st + SG.in_off;
                    bulk_g2s(in, static_cast<const uint8_t *>(A.q) + qo, SG.qkv_bytes, &full[s]);
                    bulk_g2s(in + SG.qkv_bytes, static_cast<const uint8_t *>(A.k) + qo, SG.qkv_bytes, &full[s]);
                    bulk_g2s(in + 2 * SG.qkv_bytes, static_cast<const uint8_t *>(A.v) + qo, SG.qkv_bytes, &full[s]);
                    if (F.kda) bulk_g2s(st + SG.dec_off, A.decay + h * D, (uint32_t)D * 4u, &full[s]);
                }
            }
            __syncwarp();
        }
        return;
    }

    if (warp == PREP_WARP) {
        // ------------------------------------------------ prep warp
        // Per head, as soon as its stage lands: header checks, compensator
        // lists, the new decay product, y = g . k and g . q, the new key in
        // the window-start frame, x = sm . y quantized per 16-key chunk to
        // int16, and k . q.  Lane l takes keys KPL*l .. KPL*l + KPL - 1.
        for (int it = 0; it < n_mine; ++it) {
            const int s = it % kDecodeStages;
            const uint8_t *st = stages + (size_t)s * SG.bytes;
            uint8_t *pb = s_pb + (it & 1) * PB::bytes;
            uint32_t *info = reinterpret_cast<uint32_t *>(pb + PB::info);
            if (!mbar_wait_bounded(&full[s], (uint32_t)(it / kDecodeStages) & 1u)) {
                if (lane == 0) *s_abort = 1u;
                break;  // the consumers time out on their own wait
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
            if (iscol) reinterpret_cast<uint32_t *>(pb + PB::colc)[__popc(colm & lt)] = (uint32_t)lane;
            if (isrow) reinterpret_cast<uint32_t *>(pb + PB::rowc)[__popc(rowm & lt)] = (uint32_t)lane;
            uint32_t newbits = 0;
            if (hdr.w != kMagic || ncomp > (uint32_t)F.num_comp || hdr.x > (uint32_t)F.window || badm)
                newbits = LQ_DEV_CORRUPT;
            else if (hdr.y == 0 && hdr.x >= (uint32_t)F.window)
                newbits = LQ_DEV_WINDOW_FULL;  // the window has no room for the pair
            // a work item without a blob: the stage holds stale bytes, skip it
            if (reinterpret_cast<const float *>(st + SG.aux_off)[0] != 0.f) newbits = kSkipItem;
            bool run = hdr.y == 0 && newbits == 0;
            if (newbits == kSkipItem) newbits = 0;
            float kq = 0.f;
            if (run) {
                const int i0 = KPL * lane;
                const uint8_t *in = st + SG.in_off;
                float kv[KPL], qv[KPL], gn[KPL];
#pragma unroll
                for (int e = 0; e < KPL; ++e) {
                    kv[e] = load_in(in + SG.qkv_bytes, i0 + e, F.bf16_in);
                    qv[e] = load_in(in, i0 + e, F.bf16_in);
                }
                float gprev[KPL];
#pragma unroll
                for (int e = 0; e < KPL; ++e)
                    gprev[e] = F.kda ? reinterpret_cast<const float *>(st + L.g_off)[i0 + e]
                                     : *reinterpret_cast<const float *>(st + kHdrG);
                if (F.kda) {
                    const float *dec = reinterpret_cast<const float *>(st + SG.dec_off);
#pragma unroll
                    for (int e = 0; e < KPL; ++e) gn[e] = gprev[e] * dec[i0 + e];
                } else {
                    const float alpha = reinterpret_cast<const float *>(st + SG.aux_off)[5];
#pragma unroll
                    for (int e = 0; e < KPL; ++e) gn[e] = gprev[e] * alpha;
                }
                // A decay product below the window frame's range moves the frame
                // (rebase_frame): the stored parts take the factor and the
                // product of those channels restarts at 1.  A negative or NaN
                // gate is an input error (RANGE below).
                bool small = false, invalid = false;
#pragma unroll
                for (int e = 0; e < KPL; ++e) {
                    invalid |= !(gn[e] >= 0.f);
                    small |= gn[e] < kMinDecayProduct;
                }
                if (__any_sync(0xFFFFFFFFu, small) && !__any_sync(0xFFFFFFFFu, invalid)) {
                    float f[KPL];
#pragma unroll
                    for (int e = 0; e < KPL; ++e) f[e] = (!F.kda || gn[e] < kMinDecayProduct) ? gn[e] : 1.f;
                    const int bh = blob_of(A.map, (int)(blockIdx.x + (size_t)it * G));
                    rebase_frame<D>(const_cast<uint8_t *>(st), A.state + (size_t)bh * L.blob, L, SG.pairs_at, hdr.x,
                                    hdr.z, F.f16_scale, f, lane);
#pragma unroll
                    for (int e = 0; e < KPL; ++e)
                        if (!F.kda || gn[e] < kMinDecayProduct) gn[e] = 1.f;
                }
                bool bad = false;
                float yk[KPL], yq[KPL], kh[KPL], xk[KPL], xq[KPL];
                float mk = 0.f, mq = 0.f;
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
                bad = __any_sync(0xFFFFFFFFu, bad);
#pragma unroll
                for (int e = 0; e < KPL; ++e) kh[e] = bad ? 0.f : __fdiv_rn(kv[e], gn[e]);  // window-start frame
                float *py = reinterpret_cast<float *>(pb + PB::y);
                float *pkh = reinterpret_cast<float *>(pb + PB::kh);
                float *pg = reinterpret_cast<float *>(pb + PB::g);
                float2 *pcadd = reinterpret_cast<float2 *>(pb + PB::cadd);
                if constexpr (KPL == 4) {
                    *reinterpret_cast<float4 *>(py + i0) = make_float4(yk[0], yk[1], yk[2], yk[3]);
                    *reinterpret_cast<float4 *>(py + D + i0) = make_float4(yq[0], yq[1], yq[2], yq[3]);
                    *reinterpret_cast<float4 *>(pkh + i0) = make_float4(kh[0], kh[1], kh[2], kh[3]);
                    *reinterpret_cast<float4 *>(pg + i0) = make_float4(gn[0], gn[1], gn[2], gn[3]);
                } else {
#pragma unroll
                    for (int e = 0; e < KPL; ++e) {
                        py[i0 + e] = yk[e];
                        py[D + i0 + e] = yq[e];
                        pkh[i0 + e] = kh[e];
                        pg[i0 + e] = gn[e];
                    }
                }
#pragma unroll
                for (int e = 0; e < KPL; ++e) pcadd[i0 + e] = make_float2(0.f, 0.f);
                // chunk maxima over the LPC lanes of a chunk
#pragma unroll
                for (int off = LPC / 2; off >= 1; off >>= 1) {
                    mk = fmaxf(mk, __shfl_xor_sync(0xFFFFFFFFu, mk, off));
                    mq = fmaxf(mq, __shfl_xor_sync(0xFFFFFFFFu, mq, off));
                }
                // int16 with scale ~32767 / (chunk max): rint(x * scale) by adding
                // 1.5 * 2^23 (the result stays below 2^22); chunks below 2^-100
                // are dropped (they contribute 0)
                float ik = 0.f, iq = 0.f;
                if (mk >= 0x1p-100f) ik = mk < 0x1p100f ? 32767.f * rcp_approx(mk) : __fdiv_rn(32767.f, mk);
                if (mq >= 0x1p-100f) iq = mq < 0x1p100f ? 32767.f * rcp_approx(mq) : __fdiv_rn(32767.f, mq);
                int16_t *pX = reinterpret_cast<int16_t *>(pb + PB::X);
#pragma unroll
                for (int e = 0; e < KPL; ++e) {
                    const float2 t = __ffma2_rn(make_float2(xk[e], xq[e]), make_float2(ik, iq),
                                                make_float2(12582912.0f, 12582912.0f));
                    const int i = i0 + e, slot = (i & ~15) + xslot<BITS>(i & 15);
                    pX[slot] = (int16_t)(__float_as_uint(t.x) & 0xFFFFu);
                    pX[D + slot] = (int16_t)(__float_as_uint(t.y) & 0xFFFFu);
                }
                if (lane % LPC == 0) {
                    float *psc = reinterpret_cast<float *>(pb + PB::sc);
                    psc[lane / LPC] = ik > 0.f ? mk * (1.f / 32767.f) : 0.f;
                    psc[NCH + lane / LPC] = iq > 0.f ? mq * (1.f / 32767.f) : 0.f;
                }
                kq = warp_sum(kq);
                if (bad) {
                    run = false;
                    newbits = LQ_DEV_RANGE;
                }
            }
            if (lane == 0) {
                info[kInfoRun] = run ? 1u : 0u;
                info[kInfoCount] = hdr.x;
                info[kInfoNrow] = (uint32_t)__popc(rowm);
                info[kInfoNcol] = (uint32_t)__popc(colm);
                info[kInfoBits] = newbits;
                info[kInfoKq] = __float_as_uint(kq);
            }
            __syncwarp();
            mbar_arrive(&pfull[it & 1]);
        }
        return;
    }

    // ---------------------------------------------------- consumer threads
    // GEMV role: chunk c of rows RPT*rg + m (m < RPT); the per-chunk sums go
    // to shared memory and thread j then owns row j in the epilogue.
    // dot-product role: 8 lanes per job, lane kc takes keys 4*kc + 32*e + (0..3)
    const int kc = tid % 8, jslot = tid / 8;
    if (!EARLY && b_first >= 0) {
        const uint8_t *cb = code_base + (size_t)b_first * L.blob;
#pragma unroll
        for (int m = 0; m < RPT; ++m) load_group<BITS>(cg[m], cb + (size_t)(RPT * rg + m) * L.row_bytes);
    }

    // Every iteration starts with a barrier over all consumers (the wait on
    // the prep of the head), so the chunk sums and dot products of the
    // previous head are free by then; the stage goes back to the copy warp
    // when every consumer warp has arrived on its "empty" barrier.
    for (int it = 0; it < n_mine; ++it) {
        const int s = it % kDecodeStages;
        const uint32_t ph = (uint32_t)(it >> 1) & 1u;  // phase of this head's prep barrier
        const uint8_t *st = stages + (size_t)s * SG.bytes;
        const uint8_t *pb = s_pb + (it & 1) * PB::bytes;
        const size_t h = blockIdx.x + (size_t)it * G;
        const size_t orow = h;  // input / output row of this work item
        const int bi = blob_of(A.map, (int)h);
        uint8_t *blob = A.state + (bi >= 0 ? (size_t)bi : 0) * L.blob;
        // codes of the next work item to load (through a slot map: if it has
        // a blob)
        bool has_next = it + 1 < n_mine;
        const uint8_t *next_codes = code_base + (h + G) * (size_t)L.blob;
        if constexpr (SLOTS) {
            const int bn = has_next ? A.map.blob((int)h + G) : -1;
            has_next = bn >= 0;
            next_codes = code_base + (size_t)(has_next ? bn : 0) * L.blob;
        }
        if (!consumer_sync_and(mbar_wait_bounded(&pfull[it & 1], ph), NC)) {
            // the data never arrived: record it on this blob and stop this CTA
            if (tid == 0) {
                if (bi >= 0) set_status(blob, LQ_DEV_TIMEOUT);
                *s_abort = 1u;
            }
            A.out[orow * D + tid] = 0.f;
            break;
        }
        const uint32_t *info = reinterpret_cast<const uint32_t *>(pb + PB::info);
        const bool run = info[kInfoRun] != 0u;
        const uint32_t count = info[kInfoCount];
        const int nrow = (int)info[kInfoNrow], ncol = (int)info[kInfoNcol];
        const uint32_t newbits = info[kInfoBits];
        const float *py = reinterpret_cast<const float *>(pb + PB::y);

        if (run) {
            const float *aux = reinterpret_cast<const float *>(st + SG.aux_off);
            const float *pairs = reinterpret_cast<const float *>(st + SG.pairs_at);
            const float *cvec = reinterpret_cast<const float *>(st + L.cvec_off);
            const uint32_t *meta = reinterpret_cast<const uint32_t *>(st + kHdrMeta);
            const uint32_t *colc = reinterpret_cast<const uint32_t *>(pb + PB::colc);
            const uint32_t *rowc = reinterpret_cast<const uint32_t *>(pb + PB::rowc);
            float2 *cadd = reinterpret_cast<float2 *>(const_cast<uint8_t *>(pb) + PB::cadd);
            // ---- dot products of buffered keys / compensator columns with y
            const int jobs = (int)count + ncol;
            for (int jb0 = 0; jb0 < jobs; jb0 += NJ) {
                const int jb = jb0 + jslot;
                const bool live = jb < jobs;
                float2 ak2 = make_float2(0.f, 0.f), aq2 = make_float2(0.f, 0.f);
                if (live) {
                    const float *vec = jb < (int)count ? pairs + (size_t)jb * 2 * D
                                                       : cvec + (size_t)colc[jb - count] * D;
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
                    if (jb < (int)count) s_dot[jb] = make_float2(dk_, dq_);
                    else cadd[meta[colc[jb - count]] & 0x7FFFFFFFu] = make_float2(dk_, dq_);
                }
            }

            // ---- fused dequantize + dual GEMV over the codes (integer pipe)
            uint32_t Xk[8], Xq[8];
            {
                const uint4 *xk4 = reinterpret_cast<const uint4 *>(pb + PB::X + 32 * c);
                const uint4 *xq4 = reinterpret_cast<const uint4 *>(pb + PB::X + 2 * D + 32 * c);
                const uint4 a0 = xk4[0], a1 = xk4[1], b0 = xq4[0], b1 = xq4[1];
                Xk[0] = a0.x; Xk[1] = a0.y; Xk[2] = a0.z; Xk[3] = a0.w;
                Xk[4] = a1.x; Xk[5] = a1.y; Xk[6] = a1.z; Xk[7] = a1.w;
                Xq[0] = b0.x; Xq[1] = b0.y; Xq[2] = b0.z; Xq[3] = b0.w;
                Xq[4] = b1.x; Xq[5] = b1.y; Xq[6] = b1.z; Xq[7] = b1.w;
            }
            const float *psc = reinterpret_cast<const float *>(pb + PB::sc);
            const float2 sc2 = make_float2(psc[c], psc[NCH + c]);
            int biask = 0, biasq = 0;
            if constexpr (BIAS != 0) {
#pragma unroll
                for (int x = 0; x < 8; ++x) {  // sum of the chunk's 16 entries
                    biask = dp2a_lo_ss(Xk[x], 0x00000101u, biask);
                    biasq = dp2a_lo_ss(Xq[x], 0x00000101u, biasq);
                }
                biask *= BIAS;
                biasq *= BIAS;
            }
#pragma unroll
            for (int m = 0; m < RPT; ++m) {
                int ak = -biask, aq = -biasq;
                group_dot<BITS>(cg[m], Xk, Xq, ak, aq);
                if (has_next) load_group<BITS>(cg[m], next_codes + (size_t)(RPT * rg + m) * L.row_bytes);
                s_part[c * PSTR + RPT * rg + m] = __fmul2_rn(make_float2((float)ak, (float)aq), sc2);
            }
            consumer_sync(NC);

            // ---- epilogue: thread j owns (a_j, b_j) of row j
            const int j = tid;
            float2 ab = s_part[j];
#pragma unroll
            for (int x = 1; x < LPR; ++x) ab = __fadd2_rn(ab, s_part[x * PSTR + j]);
            const float qsj = load_scale(st + L.qs_off, j, F.f16_scale);
            ab = __ffma2_rn(ab, make_float2(qsj, qsj), cadd[j]);
            for (int r = 0; r < nrow; ++r) {
                const uint32_t cc = rowc[r];
                const float wj = cvec[(size_t)cc * D + j];
                const int i0 = (int)(meta[cc] & 0x7FFFFFFFu);
                ab = __ffma2_rn(make_float2(py[i0], py[D + i0]), make_float2(wj, wj), ab);
            }
            const float *up = pairs + D + j;
#pragma unroll 4
            for (uint32_t m = 0; m < count; ++m) {
                const float uj = up[(size_t)m * 2 * D];
                ab = __ffma2_rn(s_dot[m], make_float2(uj, uj), ab);
            }
            const float u = aux[4] * (load_in(st + SG.in_off + 2 * SG.qkv_bytes, j, F.bf16_in) - ab.x);
            const float kq = __uint_as_float(info[kInfoKq]);
            A.out[orow * D + j] = fmaf(kq, u, ab.y);
            const float *pkh = reinterpret_cast<const float *>(pb + PB::kh);
            const float *pg = reinterpret_cast<const float *>(pb + PB::g);
            float *pair = reinterpret_cast<float *>(blob + L.pairs_off + (size_t)count * L.pair_bytes);
            pair[D + j] = u;
            pair[tid] = pkh[tid];
            if (F.kda) reinterpret_cast<float *>(blob + L.g_off)[tid] = pg[tid];
            if (tid == 0) {
                *reinterpret_cast<uint32_t *>(blob + kHdrCount) = count + 1;
                if (!F.kda) *reinterpret_cast<float *>(blob + kHdrG) = pg[0];
            }
        } else {
            // skipped: still move on to the next blob's codes
            if (has_next) {
#pragma unroll
                for (int m = 0; m < RPT; ++m) load_group<BITS>(cg[m], next_codes + (size_t)(RPT * rg + m) * L.row_bytes);
            }
            A.out[orow * D + tid] = 0.f;
            if (tid == 0 && newbits) set_status(blob, newbits);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with stage s
    }
}

}  // namespace lq
