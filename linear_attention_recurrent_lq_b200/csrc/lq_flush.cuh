// lq_flush.cuh -- window boundary (flush), sequence entry (init) and dense
// read-back (dequant) of LeapQuant states on sm_100a.
//
// Sources: news post "Linear attention has to move state every token it
// generates; LeapQuant compresses it to 8-bit without losing accuracy":
// per-window paragraph (quantize once at the end of the window), Compensator
// Tokens paragraph (the largest outliers leave the state as a few FP32
// rank-one pairs, the residual is quantized), residual smoothing paragraph
// (rows of the residual are balanced before quantizing; the scales are fixed
// within the window and refreshed at its boundary).
//
// Rules fixed by this library where the pages are silent:
//  * rebuild, in FP32 and in this order:
//      S_ij = g_i * ( ((qs_j * C_ji) * sm_i)  + compensators in round order
//                     + fma-chain over the buffered pairs in buffer order )
//  * compensators: r greedy rounds, each takes the key row or value column of
//    largest residual L2 energy (ties: row before column, lower index), keeps
//    it in FP32 and zeroes it in the residual;
//  * smoothing: sm_i = smallest power of two >= max_j |R_ij| (1 for a zero
//    row), clamped to the storage dtype's normal range; R' = R / sm is exact;
//  * quantization per value column: qs_j = fl32(max_i |R'_ij| / Qmax) (then
//    rounded to f16 when stored so), C_ji = clamp(rint(fl32(R'_ij / qs_j))),
//    ties to even.
//
// 4*D consumer threads per (slot, head), each owning a TI x 4 tile of the
// state (TI = D/16, layout below) in registers through every stage; row and
// column reductions go through warp shuffles, then across warps through
// shared memory.  Line energies for the compensator choice are kept in FP64
// (exact squares), so taking a line can update the other side's energies in
// place without cancellation trouble.  Every entry
// of the rebuild follows the rule's operation order exactly (packed FP32x2
// instructions round each lane like the scalar ones), so the flush compresses
// the same FP32 matrix lq_dequant_state returns.  The flush kernel is
// persistent: a producer warp double-buffers each blob (compact state and
// buffered pairs) into shared memory with bulk async copies, the consumers
// rebuild from shared memory, release the stage, then compress from registers
// and write the new compact state straight to global memory.
#pragma once

#include "lq_common.cuh"

namespace lq {

// Thread tiling of a D x D state (NT = 4D threads): warp w owns a
// (4*TI) x 32 block, rows 4*TI*wi.., columns 32*wj.. (wi = w % WR,
// wj = w / WR); lane (li = lane % 4, lj = lane / 4) owns rows
// i0 = 4*TI*wi + TI*li .. +TI and columns j0 = 32*wj + 4*lj .. +4.  Lanes
// with the same li read the same key slice of a buffered pair and lanes
// with the same lj the same value slice, so the rebuild's shared loads are
// broadcasts.
template <int D>
struct FT {
    static constexpr int NT = 4 * D, TI = D / 16, NW = NT / 32;
    static constexpr int WR = D / (4 * TI), WC = D / 32;  // warp grid (rows x cols)
    static_assert(WR * WC == NW, "warp tiling");
};

template <int D>
struct Tile {
    int li, lj, wi, wj, i0, j0;
    __device__ __forceinline__ explicit Tile(int tid) {
        const int lane = tid & 31, w = tid >> 5;
        li = lane & 3;
        lj = lane >> 2;
        wi = w % FT<D>::WR;
        wj = w / FT<D>::WR;
        i0 = 4 * FT<D>::TI * wi + FT<D>::TI * li;
        j0 = 32 * wj + 4 * lj;
    }
};

// compress scratch: rowE [D] f64 | colE [D] f64 | dred [WC][D] f64 | dredc [WR][D] f64
// | red [WC][D] | redc [WR][D] | rowv [D] | colv [D] | sm [D] | qs [D] | pick [16] | ctl [16]
template <int D>
__host__ __device__ constexpr uint32_t compress_scratch_bytes() {
    return align_up(8u * (2u * D + FT<D>::WC * D + FT<D>::WR * D) +
                        (FT<D>::WC * D + FT<D>::WR * D + 4u * D + 32u) * 4u, 128u);
}

// One flush stage: the blob prefix through W buffered pairs.
__host__ __device__ inline uint32_t flush_stage_bytes(const Layout &L, int window) {
    return align_up(L.pairs_off + (uint32_t)window * L.pair_bytes, 128);
}

constexpr int kFlushStages = 2;

template <int D>
__host__ __device__ constexpr uint32_t flush_fixed_smem() {
    return 256u + compress_scratch_bytes<D>();
}

inline uint32_t flush_smem_bytes(int D, int bits, const Layout &L, int window) {
    const uint32_t fixed = D == 128 ? flush_fixed_smem<128>() : flush_fixed_smem<64>();
    return fixed + (bits != 8 ? (uint32_t)D * D : 0u) + kFlushStages * flush_stage_bytes(L, window);
}

// init / dequant: one blob per CTA
inline uint32_t boundary_smem_bytes(int D, int bits, const Layout &L, int window) {
    const uint32_t fixed = D == 128 ? flush_fixed_smem<128>() : flush_fixed_smem<64>();
    return fixed + (bits != 8 ? (uint32_t)D * D : 0u) + flush_stage_bytes(L, window);
}

struct FlushArgs {
    uint8_t *state;
    const float *S0;  // init only
    float *S_out;     // dequant only
    Layout L;
    Flags F;
    int num_heads;
};

__device__ __forceinline__ void cons_sync(int n) { asm volatile("bar.sync 2, %0;" ::"r"(n) : "memory"); }

__device__ __forceinline__ bool cons_sync_and(bool pred, int n) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 2, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

template <typename T, bool MAX>
__device__ __forceinline__ T rop(T a, T b) { return MAX ? (a > b ? a : b) : a + b; }

// Sum (or max) of per-thread row partials r[ii] over the 8 lanes sharing li
// (lane bits 2..4): reduce-scatter, then lane lj holds the total of row
// ii = lj * TI / 8 (TI = 8: every lj; TI = 4: lj = 2*ii and 2*ii + 1 both hold it).
template <int TI, typename T, bool MAX>
__device__ __forceinline__ T warp_rows(const T (&r)[TI], int lane) {
    T v[TI];
#pragma unroll
    for (int i = 0; i < TI; ++i) v[i] = r[i];
    int n = TI;
#pragma unroll
    for (int off = 16; off >= 4; off >>= 1) {
        if (n > 1) {
            const bool up = lane & off;
#pragma unroll
            for (int i = 0; i < TI / 2; ++i) {
                if (i < n / 2) {
                    const T send = up ? v[i] : v[i + n / 2];
                    const T keep = up ? v[i + n / 2] : v[i];
                    v[i] = rop<T, MAX>(keep, __shfl_xor_sync(0xFFFFFFFFu, send, off));
                }
            }
            n >>= 1;
        } else {
            v[0] = rop<T, MAX>(v[0], __shfl_xor_sync(0xFFFFFFFFu, v[0], off));
        }
    }
    return v[0];
}

// Sum (or max) of per-thread column partials c[jj] over the 4 lanes sharing
// lj (lane bits 0..1): lane li holds the total of column jj = li.
template <typename T, bool MAX>
__device__ __forceinline__ T warp_cols(const T (&c)[4], int lane) {
    T v[4] = {c[0], c[1], c[2], c[3]};
    {
        const bool up = lane & 2;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const T send = up ? v[i] : v[i + 2];
            const T keep = up ? v[i + 2] : v[i];
            v[i] = rop<T, MAX>(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 2));
        }
    }
    const bool up = lane & 1;
    const T send = up ? v[0] : v[1];
    const T keep = up ? v[1] : v[0];
    return rop<T, MAX>(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 1));
}

// Row totals (over j) into rowv and column totals (over i) into colv for
// float partials; two consumer barriers.
template <int D, bool MAX>
__device__ __forceinline__ void reduce_rows_cols(const float (&r)[FT<D>::TI], const float (&c)[4],
                                                 float *red, float *redc, float *rowv, float *colv,
                                                 int tid, bool rows, bool cols) {
    constexpr int TI = FT<D>::TI, NT = FT<D>::NT, WR = FT<D>::WR, WC = FT<D>::WC;
    const Tile<D> t(tid);
    const int lane = tid & 31;
    if (rows) {
        const float v = warp_rows<TI, float, MAX>(r, lane);
        if (TI == 8 || (t.lj & 1) == 0) red[t.wj * D + t.i0 + t.lj * TI / 8] = v;
    }
    if (cols) {
        const float v = warp_cols<float, MAX>(c, lane);
        redc[t.wi * D + t.j0 + t.li] = v;
    }
    cons_sync(NT);
    if (rows && tid < D) {
        float a = red[tid];
#pragma unroll
        for (int w = 1; w < WC; ++w) a = rop<float, MAX>(a, red[w * D + tid]);
        rowv[tid] = a;
    }
    if (cols && tid >= D && tid < 2 * D) {
        const int j = tid - D;
        float a = redc[j];
#pragma unroll
        for (int w = 1; w < WR; ++w) a = rop<float, MAX>(a, redc[w * D + j]);
        colv[j] = a;
    }
    cons_sync(NT);
}

// The FP32 state of a blob, in the rule's order (see the file comment).
// codes8: rows of D signed 8-bit codes (value-major).
template <int D>
__device__ __forceinline__ void reconstruct_tile(float (&R)[FT<D>::TI][4], const uint8_t *qs_p,
                                                 const uint8_t *sm_p, const float *cvec,
                                                 const int8_t *codes8, const float *pairs,
                                                 const float *gvec, float gsc, const uint32_t *meta,
                                                 int ncomp, int count, int f16, int tid) {
    constexpr int TI = FT<D>::TI;
    const Tile<D> t(tid);
    const int i0 = t.i0, j0 = t.j0;
    float qsj[4], smi[TI], gi[TI];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) qsj[jj] = load_scale(qs_p, j0 + jj, f16);
#pragma unroll
    for (int ii = 0; ii < TI; ++ii) {
        smi[ii] = load_scale(sm_p, i0 + ii, f16);
        gi[ii] = gvec ? gvec[i0 + ii] : gsc;
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const int8_t *row = codes8 + (size_t)(j0 + jj) * D + i0;
        uint32_t w[TI / 4];
        if constexpr (TI == 8) {
            const uint2 v = *reinterpret_cast<const uint2 *>(row);
            w[0] = v.x ^ 0x80808080u;
            w[1] = v.y ^ 0x80808080u;
        } else {
            w[0] = *reinterpret_cast<const uint32_t *>(row) ^ 0x80808080u;
        }
#pragma unroll
        for (int ii = 0; ii < TI; ii += 2) {
            float2 cf = f2(byte_to_float(w[ii >> 2], ii & 3), byte_to_float(w[ii >> 2], (ii & 3) + 1));
            cf = __fadd2_rn(cf, f2(-8388736.0f, -8388736.0f));  // exact codes
            float2 b = __fmul2_rn(cf, f2(qsj[jj], qsj[jj]));
            b = __fmul2_rn(b, f2(smi[ii], smi[ii + 1]));
            R[ii][jj] = b.x;
            R[ii + 1][jj] = b.y;
        }
    }
    for (int cc = 0; cc < ncomp; ++cc) {
        const uint32_t m = meta[cc];
        const float *w = cvec + (size_t)cc * D;
        const int idx = (int)(m & 0x7FFFFFFFu);
        if (m & kCompCol) {
            if (idx >= j0 && idx < j0 + 4) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    if (j0 + jj == idx)
#pragma unroll
                        for (int ii = 0; ii < TI; ++ii) R[ii][jj] = __fadd_rn(R[ii][jj], w[i0 + ii]);
            }
        } else if (idx >= i0 && idx < i0 + TI) {
#pragma unroll
            for (int ii = 0; ii < TI; ++ii)
                if (i0 + ii == idx)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) R[ii][jj] = __fadd_rn(R[ii][jj], w[j0 + jj]);
        }
    }
    for (int m = 0; m < count; ++m) {
        const float *p = pairs + (size_t)m * 2 * D;
        float kh[TI];
#pragma unroll
        for (int ii = 0; ii < TI; ii += 4) {
            const float4 k4 = *reinterpret_cast<const float4 *>(p + i0 + ii);
            kh[ii] = k4.x; kh[ii + 1] = k4.y; kh[ii + 2] = k4.z; kh[ii + 3] = k4.w;
        }
        const float4 u4 = *reinterpret_cast<const float4 *>(p + D + j0);
        const float uu[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
        for (int ii = 0; ii < TI; ii += 2) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const float2 r = __ffma2_rn(f2(kh[ii], kh[ii + 1]), f2(uu[jj], uu[jj]),
                                            f2(R[ii][jj], R[ii + 1][jj]));
                R[ii][jj] = r.x;
                R[ii + 1][jj] = r.y;
            }
        }
    }
#pragma unroll
    for (int ii = 0; ii < TI; ii += 2)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const float2 r = __fmul2_rn(f2(gi[ii], gi[ii + 1]), f2(R[ii][jj], R[ii + 1][jj]));
            R[ii][jj] = r.x;
            R[ii + 1][jj] = r.y;
        }
}

// smallest power of two >= m (m > 0 finite), clamped to [lo, hi]
__device__ __forceinline__ float pow2_ceil_clamped(float m, float lo, float hi) {
    const uint32_t b = __float_as_uint(m);
    float s;
    if ((b >> 23) == 0) {
        s = lo;  // subnormal: below every allowed scale
    } else if ((b & 0x7FFFFFu) == 0) {
        s = m;   // already a power of two
    } else {
        const uint32_t e = (b >> 23) + 1;
        s = e >= 255 ? hi : __uint_as_float(e << 23);
    }
    return fminf(fmaxf(s, lo), hi);
}

// exact 1/s for a power of two s in [2^-126, 2^127]
__device__ __forceinline__ float pow2_recip(float s) {
    const uint32_t e = __float_as_uint(s) >> 23;  // biased exponent, 1..254
    return e <= 253u ? __uint_as_float((254u - e) << 23) : 0x1p-127f;
}

// Compress the register tile R (rules in the file comment) and write the new
// compact state into `blob`: compensator lines, smoothing and quantization
// scales, codes, compensator meta.  `scratch` is compress_scratch_bytes<D>()
// of shared memory; codes8 (packed formats only) D*D bytes.  Returns the
// number of compensators taken.  Every consumer thread must call it.
template <int D, int BITS>
__device__ int compress_tile(float (&R)[FT<D>::TI][4], const Flags &F, const Layout &L,
                             uint8_t *scratch, int8_t *codes8, uint8_t *blob, int tid) {
    constexpr int TI = FT<D>::TI, NT = FT<D>::NT, WR = FT<D>::WR, WC = FT<D>::WC;
    constexpr int QMAX = (1 << (BITS - 1)) - 1;
    const Tile<D> t(tid);
    const int lane = tid & 31, i0 = t.i0, j0 = t.j0;
    double *rowE = reinterpret_cast<double *>(scratch);
    double *colE = rowE + D;
    double *dred = colE + D;         // [WC][D]
    double *dredc = dred + WC * D;   // [WR][D]
    float *red = reinterpret_cast<float *>(dredc + WR * D);
    float *redc = red + WC * D;
    float *rowv = redc + WR * D, *colv = rowv + D, *smv = colv + D, *qsv = smv + D;
    uint32_t *pick = reinterpret_cast<uint32_t *>(qsv + D);
    float *cvec_out = reinterpret_cast<float *>(blob + L.cvec_off);

    // ---- line energies in FP64 (exact squares), then greedy one-hot extraction;
    // taking a line only lowers the other side's energies, updated in place
    if (F.num_comp > 0) {
        double er[TI], ec[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
        for (int ii = 0; ii < TI; ++ii) {
            er[ii] = 0.0;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const double x = (double)R[ii][jj];
                er[ii] = fma(x, x, er[ii]);
                ec[jj] = fma(x, x, ec[jj]);
            }
        }
        {
            const double v = warp_rows<TI, double, false>(er, lane);
            if (TI == 8 || (t.lj & 1) == 0) dred[t.wj * D + i0 + t.lj * TI / 8] = v;
            const double w = warp_cols<double, false>(ec, lane);
            dredc[t.wi * D + j0 + t.li] = w;
        }
        cons_sync(NT);
        if (tid < D) {
            double a = dred[tid];
#pragma unroll
            for (int w = 1; w < WC; ++w) a += dred[w * D + tid];
            rowE[tid] = a;
        } else if (tid < 2 * D) {
            const int j = tid - D;
            double a = dredc[j];
#pragma unroll
            for (int w = 1; w < WR; ++w) a += dredc[w * D + j];
            colE[j] = a;
        }
        cons_sync(NT);
    }
    int ncomp = 0;
    for (int cc = 0; cc < F.num_comp; ++cc) {
        if (tid < 32) {
            double best = -1.0;
            int key = 0x7FFFFFFF;
#pragma unroll
            for (int x = 0; x < 2 * D / 32; ++x) {
                const int k = lane + 32 * x;
                const double e = k < D ? rowE[k] : colE[k - D];
                if (e > best) { best = e; key = k; }  // ascending keys: ties keep the lower key
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                const double ob = __shfl_xor_sync(0xFFFFFFFFu, best, off);
                const int ok = __shfl_xor_sync(0xFFFFFFFFu, key, off);
                if (ob > best || (ob == best && ok < key)) { best = ob; key = ok; }
            }
            if (lane == 0) {
                uint32_t p = kCompNone;
                if (best > 0.0) {
                    p = key < D ? (uint32_t)key : (kCompCol | (uint32_t)(key - D));
                    if (key < D) rowE[key] = 0.0; else colE[key - D] = 0.0;
                }
                pick[cc] = p;
            }
        }
        cons_sync(NT);
        const uint32_t p = pick[cc];
        if (p == kCompNone) break;
        float *w = cvec_out + (size_t)cc * D;
        const int idx = (int)(p & 0x7FFFFFFFu);
        if (p & kCompCol) {
            if (idx >= j0 && idx < j0 + 4) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    if (j0 + jj == idx) {
#pragma unroll
                        for (int ii = 0; ii < TI; ++ii) {
                            const float x = R[ii][jj];
                            w[i0 + ii] = x;
                            rowE[i0 + ii] -= (double)x * (double)x;
                            R[ii][jj] = 0.f;
                        }
                    }
            }
        } else if (idx >= i0 && idx < i0 + TI) {
#pragma unroll
            for (int ii = 0; ii < TI; ++ii)
                if (i0 + ii == idx) {
                    *reinterpret_cast<float4 *>(w + j0) = make_float4(R[ii][0], R[ii][1], R[ii][2], R[ii][3]);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        colE[j0 + jj] -= (double)R[ii][jj] * (double)R[ii][jj];
                        R[ii][jj] = 0.f;
                    }
                }
        }
        ++ncomp;
        cons_sync(NT);
    }
    for (int cc = ncomp; cc < F.num_comp; ++cc)
        for (int x = tid; x < D; x += NT) cvec_out[(size_t)cc * D + x] = 0.f;

    // ---- residual smoothing: one power of two per key row
    const float sm_lo = F.f16_scale ? 0x1p-14f : 0x1p-126f;
    const float sm_hi = F.f16_scale ? 0x1p15f : 0x1p127f;
    {
        float mr[TI], dummy[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ii = 0; ii < TI; ++ii)
            mr[ii] = fmaxf(fmaxf(fabsf(R[ii][0]), fabsf(R[ii][1])), fmaxf(fabsf(R[ii][2]), fabsf(R[ii][3])));
        reduce_rows_cols<D, true>(mr, dummy, red, redc, rowv, colv, tid, true, false);
        if (tid < D) {
            const float m = rowv[tid];
            const float s = (F.smoothing && m > 0.f) ? pow2_ceil_clamped(m, sm_lo, sm_hi) : 1.f;
            smv[tid] = s;
            if (F.f16_scale) reinterpret_cast<__half *>(blob + L.sm_off)[tid] = __float2half_rn(s);
            else reinterpret_cast<float *>(blob + L.sm_off)[tid] = s;
        }
        cons_sync(NT);
    }
    float cm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ii = 0; ii < TI; ii += 2) {
        const float2 inv = f2(pow2_recip(smv[i0 + ii]), pow2_recip(smv[i0 + ii + 1]));
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const float2 r = __fmul2_rn(f2(R[ii][jj], R[ii + 1][jj]), inv);  // exact
            R[ii][jj] = r.x;
            R[ii + 1][jj] = r.y;
            cm[jj] = fmaxf(cm[jj], fmaxf(fabsf(r.x), fabsf(r.y)));
        }
    }

    // ---- symmetric scale per value column
    {
        float dummy[TI];
#pragma unroll
        for (int ii = 0; ii < TI; ++ii) dummy[ii] = 0.f;
        reduce_rows_cols<D, true>(dummy, cm, red, redc, rowv, colv, tid, false, true);
    }
    if (tid < D) {
        const float m = colv[tid];
        float s = __fdiv_rn(m, (float)QMAX);
        if (F.f16_scale) {
            s = __half2float(__float2half_rn(s));
            if (m > 0.f && s == 0.f) s = 0x1p-24f;
            reinterpret_cast<__half *>(blob + L.qs_off)[tid] = __float2half_rn(s);
        } else {
            if (m > 0.f && s == 0.f) s = 0x1p-149f;
            reinterpret_cast<float *>(blob + L.qs_off)[tid] = s;
        }
        qsv[tid] = s;
    }
    cons_sync(NT);

    // ---- codes: rint of the correctly rounded FP32 quotient, ties to even.
    // Fast path: multiply by the rounded reciprocal (within 1.5 ulp of the
    // quotient) and round by adding 1.5*2^23.  A thread with any entry within
    // 2e-5 of a half-integer, or with a column scale so small that the
    // quotient may leave [-Qmax, Qmax], redoes its entries by division.
    int8_t *dst8 = BITS == 8 ? reinterpret_cast<int8_t *>(blob + L.codes_off) : codes8;
    const uint32_t dst_row = BITS == 8 ? L.row_bytes : (uint32_t)D;
    const float min_fast = F.f16_scale ? 0x1p-14f : 0x1p-100f;
    float sj[4], inv[4];
    bool slow = false;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        sj[jj] = qsv[j0 + jj];
        inv[jj] = __frcp_rn(sj[jj]);
        slow |= (sj[jj] != 0.f) && !(sj[jj] >= min_fast);
    }
    uint32_t nb[TI][4];
    float dmax = 0.f;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
        for (int ii = 0; ii < TI; ii += 2) {
            const float2 tq = __fmul2_rn(f2(R[ii][jj], R[ii + 1][jj]), f2(inv[jj], inv[jj]));
            const float2 nf = __fadd2_rn(tq, f2(12582912.0f, 12582912.0f));  // 1.5 * 2^23
            const float2 back = __fadd2_rn(nf, f2(-12582912.0f, -12582912.0f));
            const float2 d = __fadd2_rn(tq, f2(-back.x, -back.y));
            dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
            nb[ii][jj] = sj[jj] != 0.f ? __float_as_uint(nf.x) : 0x4B400000u;
            nb[ii + 1][jj] = sj[jj] != 0.f ? __float_as_uint(nf.y) : 0x4B400000u;
        }
    }
    if (slow || dmax > 0.49998f) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
#pragma unroll
            for (int ii = 0; ii < TI; ++ii) {
                if (sj[jj] == 0.f) continue;
                float tq = __fdiv_rn(R[ii][jj], sj[jj]);
                tq = fminf(fmaxf(tq, -(float)QMAX), (float)QMAX);
                nb[ii][jj] = __float_as_uint(__fadd_rn(tq, 12582912.0f));
            }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        int8_t *row = dst8 + (size_t)(j0 + jj) * dst_row + i0;
        const uint32_t w0 = __byte_perm(__byte_perm(nb[0][jj], nb[1][jj], 0x0040),
                                        __byte_perm(nb[2][jj], nb[3][jj], 0x0040), 0x5410);
        if constexpr (TI == 8) {
            const uint32_t w1 = __byte_perm(__byte_perm(nb[4][jj], nb[5][jj], 0x0040),
                                            __byte_perm(nb[6][jj], nb[7][jj], 0x0040), 0x5410);
            *reinterpret_cast<uint2 *>(row) = make_uint2(w0, w1);
        } else {
            *reinterpret_cast<uint32_t *>(row) = w0;
        }
    }
    if constexpr (BITS != 8) {
        cons_sync(NT);
        constexpr int GB = group_bytes<BITS>(), GPR = D / 16;
        for (int gi = tid; gi < D * GPR; gi += NT) {
            const int j = gi / GPR, grp = gi % GPR;
            const uint4 w = *reinterpret_cast<const uint4 *>(codes8 + (size_t)j * D + 16 * grp);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
            int8_t c[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) c[x] = (int8_t)(ws[x >> 2] >> (8 * (x & 3)));
            pack16<BITS>(c, blob + L.codes_off + (size_t)j * L.row_bytes + grp * GB);
        }
    }
    if (tid < 16) {
        const uint32_t m = tid < ncomp ? pick[tid] : kCompNone;
        reinterpret_cast<uint32_t *>(blob + kHdrMeta)[tid] = m;
    }
    cons_sync(NT);  // scratch free for the next blob
    return ncomp;
}

// Unpack a blob's packed codes (shared memory) to int8 rows of D codes.
template <int D, int BITS>
__device__ __forceinline__ void unpack_all(const uint8_t *codes, uint32_t row_bytes, int8_t *codes8,
                                           int tid) {
    constexpr int GB = group_bytes<BITS>(), GPR = D / 16, NT = FT<D>::NT;
    for (int g = tid; g < D * GPR; g += NT) {
        const int j = g / GPR, grp = g % GPR;
        float cf[16];
        unpack16<BITS>(codes + (size_t)j * row_bytes + grp * GB, cf);
        uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int x = 0; x < 16; ++x) w[x >> 2] |= ((uint32_t)(int)cf[x] & 0xFFu) << (8 * (x & 3));
        *reinterpret_cast<uint4 *>(codes8 + (size_t)j * D + 16 * grp) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Header fields a consumer needs, parsed from a staged blob prefix.
struct StagedHeader {
    uint32_t count, status, ncomp;
    bool ok;
    float g;
};

template <int D>
__device__ __forceinline__ StagedHeader parse_staged(const uint8_t *st, const Flags &F) {
    StagedHeader H;
    const uint4 h = *reinterpret_cast<const uint4 *>(st);
    H.count = h.x;
    H.status = h.y;
    H.ncomp = h.z;
    H.g = *reinterpret_cast<const float *>(st + kHdrG);
    bool ok = h.w == kMagic && h.z <= (uint32_t)F.num_comp && h.x <= (uint32_t)F.window;
    const uint32_t *meta = reinterpret_cast<const uint32_t *>(st + kHdrMeta);
    for (uint32_t cc = 0; ok && cc < h.z; ++cc) ok = (meta[cc] & 0x7FFFFFFFu) < (uint32_t)D;
    H.ok = ok;
    return H;
}

template <int D>
__device__ __forceinline__ void write_fresh_header(uint8_t *blob, const Flags &F, int ncomp,
                                                   bool reset_status, int tid) {
    if (F.kda)
        for (int x = tid; x < D; x += FT<D>::NT) reinterpret_cast<float *>(blob + kHdrBytes)[x] = 1.f;
    if (tid == 0) {
        uint32_t *h = reinterpret_cast<uint32_t *>(blob);
        h[0] = 0u;                  // count
        if (reset_status) h[1] = 0u;
        h[2] = (uint32_t)ncomp;
        h[3] = kMagic;
        *reinterpret_cast<float *>(blob + kHdrG) = 1.f;
    }
}

// ---------------------------------------------------------------- flush
template <int D, int BITS>
__global__ void __launch_bounds__(4 * D + 32, 1) flush_kernel(FlushArgs A) {
    constexpr int NT = FT<D>::NT, TI = FT<D>::TI;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Layout L = A.L;
    const Flags F = A.F;
    const uint32_t SB = flush_stage_bytes(L, F.window);
    const int G = gridDim.x;
    const int n_mine = (A.num_heads - (int)blockIdx.x + G - 1) / G;

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + kFlushStages;
    volatile uint32_t *s_abort = reinterpret_cast<volatile uint32_t *>(smem + 60);
    uint32_t *s_cnt = reinterpret_cast<uint32_t *>(smem + 64);  // producer batch [32]
    uint8_t *scratch = smem + 256;
    int8_t *codes8 = reinterpret_cast<int8_t *>(scratch + compress_scratch_bytes<D>());
    uint8_t *stages = reinterpret_cast<uint8_t *>(codes8) + (BITS != 8 ? D * D : 0);

    if (tid == 0) {
        for (int s = 0; s < kFlushStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        *s_abort = 0u;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == NT / 32) {
        // producer: copy each blob's prefix and its buffered pairs; the
        // window counts of up to 32 blobs are read at once
        for (int base = 0; base < n_mine && !*s_abort; base += 32) {
            if (base + lane < n_mine)
                s_cnt[lane] = *reinterpret_cast<const uint32_t *>(
                    A.state + ((size_t)blockIdx.x + (size_t)(base + lane) * G) * L.blob + kHdrCount);
            __syncwarp();
            if (lane == 0) {
                for (int x = 0; x < 32 && base + x < n_mine; ++x) {
                    const int it = base + x, s = it % kFlushStages;
                    if (it >= kFlushStages && !mbar_wait_bounded(&empty[s], ((it / kFlushStages) - 1) & 1)) {
                        *s_abort = 1u;
                        break;
                    }
                    const uint8_t *blob = A.state + ((size_t)blockIdx.x + (size_t)it * G) * L.blob;
                    const uint32_t c = s_cnt[x];
                    const uint32_t bytes = L.pairs_off + (c <= (uint32_t)F.window ? c : 0u) * L.pair_bytes;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    bulk_g2s(stages + (size_t)s * SB, blob, bytes, &full[s]);
                }
            }
            __syncwarp();
        }
        return;
    }

    for (int it = 0; it < n_mine; ++it) {
        const int s = it % kFlushStages;
        const uint8_t *st = stages + (size_t)s * SB;
        uint8_t *blob = A.state + ((size_t)blockIdx.x + (size_t)it * G) * L.blob;
        if (!cons_sync_and(mbar_wait_bounded(&full[s], (uint32_t)(it / kFlushStages) & 1u), NT)) {
            if (tid == 0) {
                set_status(blob, LQ_DEV_TIMEOUT);
                *s_abort = 1u;
            }
            break;
        }
        const StagedHeader H = parse_staged<D>(st, F);
        // flush only a valid blob with a non-empty window and no error flag
        const bool run = H.ok && H.status == 0 && H.count > 0;
        if (!H.ok && tid == 0) set_status(blob, LQ_DEV_CORRUPT);
        float R[TI][4];
        if (run) {
            const int8_t *c8 = reinterpret_cast<const int8_t *>(st + L.codes_off);
            if constexpr (BITS != 8) {
                unpack_all<D, BITS>(st + L.codes_off, L.row_bytes, codes8, tid);
                cons_sync(NT);
                c8 = codes8;
            }
            reconstruct_tile<D>(R, st + L.qs_off, st + L.sm_off,
                                reinterpret_cast<const float *>(st + L.cvec_off), c8,
                                reinterpret_cast<const float *>(st + L.pairs_off),
                                F.kda ? reinterpret_cast<const float *>(st + L.g_off) : nullptr, H.g,
                                reinterpret_cast<const uint32_t *>(st + kHdrMeta), (int)H.ncomp,
                                (int)H.count, F.f16_scale, tid);
        }
        cons_sync(NT);  // the stage has been read
        if (tid == 0) mbar_arrive(&empty[s]);
        if (run) {
            const int ncomp = compress_tile<D, BITS>(R, F, L, scratch, codes8, blob, tid);
            write_fresh_header<D>(blob, F, ncomp, false, tid);
        }
    }
}

// ------------------------------------------------- init (MODE 1), dequant (MODE 2)
template <int D, int BITS, int MODE>
__global__ void __launch_bounds__(4 * D) boundary_kernel(FlushArgs A) {
    constexpr int NT = FT<D>::NT, TI = FT<D>::TI;
    const int tid = threadIdx.x;
    const size_t head = blockIdx.x;
    const Layout L = A.L;
    const Flags F = A.F;
    uint8_t *blob = A.state + head * L.blob;
    const Tile<D> tl(tid);
    const int i0 = tl.i0, j0 = tl.j0;

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
    uint32_t *s_hdr = reinterpret_cast<uint32_t *>(smem + 16);
    uint8_t *scratch = smem + 256;
    int8_t *codes8 = reinterpret_cast<int8_t *>(scratch + compress_scratch_bytes<D>());
    uint8_t *st = reinterpret_cast<uint8_t *>(codes8) + (BITS != 8 ? D * D : 0);

    float R[TI][4];
    if constexpr (MODE == 1) {
        const float *S0 = A.S0 + head * (size_t)D * D;
#pragma unroll
        for (int ii = 0; ii < TI; ++ii) {
            const float4 r4 = *reinterpret_cast<const float4 *>(S0 + (size_t)(i0 + ii) * D + j0);
            R[ii][0] = r4.x; R[ii][1] = r4.y; R[ii][2] = r4.z; R[ii][3] = r4.w;
        }
        const int ncomp = compress_tile<D, BITS>(R, F, L, scratch, codes8, blob, tid);
        write_fresh_header<D>(blob, F, ncomp, true, tid);
    } else {
        if (tid == 0) {
            const uint4 h = *reinterpret_cast<const uint4 *>(blob);
            bool ok = h.w == kMagic && h.z <= (uint32_t)F.num_comp && h.x <= (uint32_t)F.window;
            const uint32_t *meta = reinterpret_cast<const uint32_t *>(blob + kHdrMeta);
            for (uint32_t cc = 0; ok && cc < h.z; ++cc) ok = (meta[cc] & 0x7FFFFFFFu) < (uint32_t)D;
            s_hdr[0] = ok ? 1u : 0u;
            if (ok) {
                const uint32_t bytes = L.pairs_off + h.x * L.pair_bytes;
                mbar_init(&bar[0], 1);
                fence_mbar_init();
                mbar_arrive_expect_tx(&bar[0], bytes);
                bulk_g2s(st, blob, bytes, &bar[0]);
            }
        }
        __syncthreads();
        float *So = A.S_out + head * (size_t)D * D;
        if (!s_hdr[0]) {  // unreadable blob: zeros
#pragma unroll
            for (int ii = 0; ii < TI; ++ii)
                *reinterpret_cast<float4 *>(So + (size_t)(i0 + ii) * D + j0) = make_float4(0.f, 0.f, 0.f, 0.f);
            return;
        }
        if (!__syncthreads_and(mbar_wait_bounded(&bar[0], 0))) {
            if (tid == 0) {
                set_status(blob, LQ_DEV_TIMEOUT);
                mbar_wait_bounded(&bar[0], 0);
            }
            return;
        }
        const StagedHeader H = parse_staged<D>(st, F);
        const int8_t *c8 = reinterpret_cast<const int8_t *>(st + L.codes_off);
        if constexpr (BITS != 8) {
            unpack_all<D, BITS>(st + L.codes_off, L.row_bytes, codes8, tid);
            __syncthreads();
            c8 = codes8;
        }
        reconstruct_tile<D>(R, st + L.qs_off, st + L.sm_off,
                            reinterpret_cast<const float *>(st + L.cvec_off), c8,
                            reinterpret_cast<const float *>(st + L.pairs_off),
                            F.kda ? reinterpret_cast<const float *>(st + L.g_off) : nullptr, H.g,
                            reinterpret_cast<const uint32_t *>(st + kHdrMeta), (int)H.ncomp,
                            (int)H.count, F.f16_scale, tid);
#pragma unroll
        for (int ii = 0; ii < TI; ++ii)
            *reinterpret_cast<float4 *>(So + (size_t)(i0 + ii) * D + j0) =
                make_float4(R[ii][0], R[ii][1], R[ii][2], R[ii][3]);
    }
}

}  // namespace lq
