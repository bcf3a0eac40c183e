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
// One CTA per (slot, head), 2*D threads.  Thread 0 starts two bulk copies
// into shared memory (scales + compensators + codes at once, then the buffered
// pairs once the header says how many), while all threads load q, k, v and
// build the decay-folded vectors.  The GEMV reads 16-code groups from shared
// memory (conflict-free for 8, 6 and 4 bits), turns codes into exact floats
// with byte permutes instead of int->float conversions, and reduces over the
// D/16 threads of a row with a reduce-scatter shuffle tree.
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
};

constexpr int kDotSlots = kMaxWindow + kMaxComp;

template <int D>
__host__ __device__ constexpr uint32_t decode_fixed_smem() {
    // barriers + header (128), y/x/gemv (6D floats), dots (2*kDotSlots), reduce (32)
    return align_up(128u + (6u * D + 2u * kDotSlots + 32u) * 4u, 128u);
}

inline uint32_t decode_smem_bytes(int D, const Layout &L, int window) {
    const uint32_t fixed = D == 128 ? decode_fixed_smem<128>() : decode_fixed_smem<64>();
    return fixed + align_up(L.compact_bytes, 128) + (uint32_t)(window - 1) * L.pair_bytes;
}

// Reduce-scatter of N values over the N consecutive lanes of an aligned
// group (N a power of two <= 32): afterwards lane l holds the group sum of
// value (l mod N) in v[0].
template <int N>
__device__ __forceinline__ void reduce_scatter_group(float (&v)[N], int lane) {
#pragma unroll
    for (int off = N / 2; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = upper ? v[i] : v[i + off];
            const float keep = upper ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
        }
    }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, off);
    return x;
}

template <int D, int BITS>
__global__ void __launch_bounds__(2 * D) decode_kernel(DecodeArgs A) {
    constexpr int NT = 2 * D, CPR = D / 16, MR = D / 32, E = D / 32;
    constexpr int GB = group_bytes<BITS>();
    static_assert(2 * MR == CPR, "one value per lane after the reduce-scatter");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t head = blockIdx.x;
    const Layout &L = A.L;
    const Flags &F = A.F;
    uint8_t *blob = A.state + head * L.blob;

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
    uint32_t *s_hdr = reinterpret_cast<uint32_t *>(smem + 16);  // count, status, ncomp, skip, g, newbits
    uint32_t *s_meta = reinterpret_cast<uint32_t *>(smem + 64);
    float *s_y = reinterpret_cast<float *>(smem + 128);  // y_k [D] | y_q [D]
    float *s_x = s_y + 2 * D;                            // x_k [D] | x_q [D]
    float *s_gemv = s_x + 2 * D;                         // R^T y_k [D] | R^T y_q [D] (before qs)
    float *s_dot = s_gemv + 2 * D;                       // k-side [kDotSlots] | q-side
    float *s_red = s_dot + 2 * kDotSlots;                // [32]
    uint8_t *s_cmp = smem + decode_fixed_smem<D>();      // qs | sm | comp_vec | codes
    float *s_pairs = reinterpret_cast<float *>(s_cmp + align_up(L.compact_bytes, 128));
    const uint8_t *s_qs = s_cmp;
    const uint8_t *s_sm = s_cmp + (L.sm_off - L.qs_off);
    const float *s_cvec = reinterpret_cast<const float *>(s_cmp + (L.cvec_off - L.qs_off));
    const uint8_t *s_codes = s_cmp + (L.codes_off - L.qs_off);

    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar[0], L.compact_bytes);
        bulk_g2s(s_cmp, blob + L.qs_off, L.compact_bytes, &bar[0]);
        const uint4 h = *reinterpret_cast<const uint4 *>(blob);  // count, status, ncomp, magic
        const uint32_t g_bits = *reinterpret_cast<const uint32_t *>(blob + kHdrG);
        const uint4 *gm = reinterpret_cast<const uint4 *>(blob + kHdrMeta);
        uint4 *sm4 = reinterpret_cast<uint4 *>(s_meta);
#pragma unroll
        for (int x = 0; x < 4; ++x) sm4[x] = gm[x];
        bool meta_ok = true;
        for (uint32_t cc = 0; cc < h.z && cc < (uint32_t)kMaxComp; ++cc)
            meta_ok &= (s_meta[cc] & 0x7FFFFFFFu) < (uint32_t)D;
        uint32_t newbits = 0;
        if (h.w != kMagic || h.z > (uint32_t)F.num_comp || h.x > (uint32_t)F.window || !meta_ok)
            newbits = LQ_DEV_CORRUPT;
        else if (h.y == 0 && h.x >= (uint32_t)F.window)
            newbits = LQ_DEV_WINDOW_FULL;
        const bool run = h.y == 0 && newbits == 0;
        const uint32_t pbytes = run ? h.x * L.pair_bytes : 0u;
        mbar_arrive_expect_tx(&bar[1], pbytes);
        if (pbytes) bulk_g2s(s_pairs, blob + L.pairs_off, pbytes, &bar[1]);
        s_hdr[0] = h.x;
        s_hdr[1] = h.y;
        s_hdr[2] = h.z;
        s_hdr[3] = run ? 0u : 1u;
        s_hdr[4] = g_bits;
        s_hdr[5] = newbits;
    }

    // inputs of this token (independent of the state)
    float kv = 0.f, qv = 0.f, vv = 0.f, av = 1.f, gold = 1.f;
    if (tid < D) {
        const size_t o = head * D + tid;
        kv = load_in(A.k, o, F.bf16_in);
        qv = load_in(A.q, o, F.bf16_in);
        vv = load_in(A.v, o, F.bf16_in);
        if (F.kda) {
            av = A.decay[o];
            gold = reinterpret_cast<const float *>(blob + L.g_off)[tid];
        }
    }
    const float bt = A.beta[head];
    const float alpha = F.kda ? 1.f : A.decay[head];
    __syncthreads();

    uint32_t skip = s_hdr[3];
    const uint32_t count = s_hdr[0], ncomp = s_hdr[2];
    if (!F.kda) {
        gold = __uint_as_float(s_hdr[4]);
        av = alpha;
    }
    const float gnew = gold * av;
    const bool bad = (tid < D) && !(gnew >= kMinDecayProduct);
    const int any_bad = __syncthreads_or(bad);
    uint32_t newbits = s_hdr[5];
    if (!skip && any_bad) {
        skip = 1;
        newbits = LQ_DEV_RANGE;
    }

    bool ok = true;
    if (!skip) {
        if (tid < D) {
            s_y[tid] = gnew * kv;
            s_y[D + tid] = gnew * qv;
        }
        float kq = (tid < D) ? kv * qv : 0.f;
        kq = warp_sum(kq);
        if (lane == 0) s_red[warp] = kq;
        ok = __syncthreads_and(mbar_wait_bounded(&bar[0], 0));
        if (ok) {
            if (tid < D) {
                const float smv = load_scale(s_sm, tid, F.f16_scale);
                s_x[tid] = smv * s_y[tid];
                s_x[D + tid] = smv * s_y[D + tid];
            }
            __syncthreads();

            // ---- fused dequantize + dual GEMV over the codes
            const int c = tid % CPR, rg = tid / CPR;
            float xk[16], xq[16];
#pragma unroll
            for (int x = 0; x < 16; x += 4) {
                const float4 a4 = *reinterpret_cast<const float4 *>(s_x + 16 * c + x);
                const float4 b4 = *reinterpret_cast<const float4 *>(s_x + D + 16 * c + x);
                xk[x] = a4.x; xk[x + 1] = a4.y; xk[x + 2] = a4.z; xk[x + 3] = a4.w;
                xq[x] = b4.x; xq[x + 1] = b4.y; xq[x + 2] = b4.z; xq[x + 3] = b4.w;
            }
            float acc[2 * MR];
#pragma unroll
            for (int m = 0; m < MR; ++m) {
                const int j = rg + 32 * m;
                float cf[16];
                unpack16<BITS>(s_codes + (size_t)j * L.row_bytes + c * GB, cf);
                float ak = 0.f, aq = 0.f;
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    ak = fmaf(cf[x], xk[x], ak);
                    aq = fmaf(cf[x], xq[x], aq);
                }
                acc[m] = ak;
                acc[MR + m] = aq;
            }
            reduce_scatter_group<CPR>(acc, lane);
            {
                const int idx = lane & (CPR - 1);
                const int side = idx / MR, m = idx % MR;
                s_gemv[side * D + rg + 32 * m] = acc[0];
            }
            ok = __syncthreads_and(mbar_wait_bounded(&bar[1], 0));
        }
        if (ok) {
            // ---- dot products of buffered keys and compensator columns with y
            float yk[E], yq[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                yk[e] = s_y[lane * E + e];
                yq[e] = s_y[D + lane * E + e];
            }
            const int jobs = (int)(count + ncomp);
            for (int jb = warp; jb < jobs; jb += NT / 32) {
                const float *vec;
                if (jb < (int)count) {
                    vec = s_pairs + (size_t)jb * 2 * D;
                } else {
                    const uint32_t meta = s_meta[jb - count];
                    if (!(meta & kCompCol)) continue;  // key-row lines need no dot
                    vec = s_cvec + (size_t)(jb - count) * D;
                }
                float dk_ = 0.f, dq_ = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float x = vec[lane * E + e];
                    dk_ = fmaf(x, yk[e], dk_);
                    dq_ = fmaf(x, yq[e], dq_);
                }
                dk_ = warp_sum(dk_);
                dq_ = warp_sum(dq_);
                if (lane == 0) {
                    s_dot[jb] = dk_;
                    s_dot[kDotSlots + jb] = dq_;
                }
            }
            __syncthreads();

            // ---- combine, delta update, output, append the pair
            if (tid < D) {
                const int j = tid;
                float kq = 0.f;
#pragma unroll
                for (int w = 0; w < D / 32; ++w) kq += s_red[w];
                const float qsj = load_scale(s_qs, j, F.f16_scale);
                float a = qsj * s_gemv[j];
                float b = qsj * s_gemv[D + j];
                for (uint32_t cc = 0; cc < ncomp; ++cc) {
                    const uint32_t meta = s_meta[cc];
                    if (meta & kCompCol) {
                        if ((int)(meta & 0x7FFFFFFFu) == j) {
                            a += s_dot[count + cc];
                            b += s_dot[kDotSlots + count + cc];
                        }
                    } else {
                        const float wj = s_cvec[(size_t)cc * D + j];
                        a = fmaf(s_y[meta], wj, a);
                        b = fmaf(s_y[D + meta], wj, b);
                    }
                }
                for (uint32_t m = 0; m < count; ++m) {
                    const float uj = s_pairs[(size_t)m * 2 * D + D + j];
                    a = fmaf(s_dot[m], uj, a);
                    b = fmaf(s_dot[kDotSlots + m], uj, b);
                }
                const float u = bt * (vv - a);
                A.out[head * D + j] = fmaf(kq, u, b);
                float *pair = reinterpret_cast<float *>(blob + L.pairs_off + (size_t)count * L.pair_bytes);
                pair[j] = __fdiv_rn(kv, gnew);  // key j in the window-start frame
                pair[D + j] = u;
                if (F.kda) reinterpret_cast<float *>(blob + L.g_off)[j] = gnew;
            }
            if (tid == 0) {
                *reinterpret_cast<uint32_t *>(blob + kHdrCount) = count + 1;
                if (!F.kda) *reinterpret_cast<float *>(blob + kHdrG) = gnew;
            }
            return;
        }
        newbits = LQ_DEV_TIMEOUT;
    }

    // skipped (or a copy wait timed out): zero output, record, drain copies
    if (tid < D) A.out[head * D + tid] = 0.f;
    if (tid == 0) {
        if (newbits) set_status(blob, newbits);
        mbar_wait_bounded(&bar[0], 0);
        mbar_wait_bounded(&bar[1], 0);
    }
}

}  // namespace lq
