// lq_common.cuh -- blob layout and device helpers shared by the LeapQuant
// kernels (sm_100a).  Everything here is internal to libleapquant.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "leapquant.h"

namespace lq {

constexpr uint32_t kMagic = 0x4C515354u;     // "LQST"
constexpr uint32_t kCompCol = 0x80000000u;   // compensator kind bit: value column
constexpr uint32_t kCompNone = 0xFFFFFFFFu;
constexpr int kMaxComp = 16;
constexpr int kMaxWindow = 64;
// Decay products below this leave the window-start frame's safe range: the
// keys are stored divided by the product, so it must stay far from FP32
// underflow.  The decode moves the frame (rebase_frame) when a product
// falls below it.
constexpr float kMinDecayProduct = 0x1p-96f;
// Bounded waits on on-chip copies: give up after this long (ns).
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// Header field offsets (bytes) inside a blob.
constexpr int kHdrCount = 0, kHdrStatus = 4, kHdrNcomp = 8, kHdrMagic = 12, kHdrG = 16;
constexpr int kHdrMeta = 64, kHdrBytes = 128;

// Byte offsets of one (slot, head) blob; identical on host and device.
struct Layout {
    uint32_t blob;           // bytes per blob (multiple of 256)
    uint32_t g_off;          // KDA decay-product vector (0 when GDN)
    uint32_t qs_off, sm_off, cvec_off, codes_off, pairs_off;
    uint32_t row_bytes;      // packed code bytes per value row
    uint32_t compact_bytes;  // [qs_off, pairs_off): scales, compensators, codes
    uint32_t pair_bytes;     // (dk + dv) * 4
    uint32_t scale_bytes;    // 4 (f32) or 2 (f16)
};

__host__ __device__ constexpr uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

inline Layout make_layout(const lq_config &c) {
    Layout L{};
    const uint32_t dk = c.dk, dv = c.dv, maxd = dk > dv ? dk : dv;
    if (c.bits == 32) {
        L.qs_off = L.sm_off = L.cvec_off = L.codes_off = kHdrBytes;  // S[dk][dv] at 128
        L.pairs_off = kHdrBytes + dk * dv * 4;
        L.blob = align_up(L.pairs_off, 256);
        return L;
    }
    if (c.per_step) {
        // BF16: S[dk][dv] bf16 at 128.  FP8: scale[dv] f32 at 128, codes[dk][dv] after it.
        L.qs_off = L.sm_off = L.cvec_off = kHdrBytes;
        L.codes_off = c.bits == 16 ? kHdrBytes : kHdrBytes + align_up(dv * 4, 128);
        L.pairs_off = L.codes_off + dk * dv * (c.bits == 16 ? 2u : 1u);
        L.blob = align_up(L.pairs_off, 256);
        return L;
    }
    L.scale_bytes = c.scale_dtype ? 2 : 4;
    L.row_bytes = dk * (uint32_t)c.bits / 8;
    L.pair_bytes = (dk + dv) * 4;
    uint32_t off = kHdrBytes;
    if (c.decay_kind == 1) { L.g_off = off; off += align_up(dk * 4, 128); }
    L.qs_off = off;    off += align_up(dv * L.scale_bytes, 128);
    L.sm_off = off;    off += align_up(dk * L.scale_bytes, 128);
    L.cvec_off = off;  off += align_up((uint32_t)c.num_comp * maxd * 4, 128);
    L.codes_off = off; off += align_up(dv * L.row_bytes, 128);
    L.pairs_off = off; off += (uint32_t)c.window * L.pair_bytes;
    L.compact_bytes = L.pairs_off - L.qs_off;
    L.blob = align_up(off, 256);
    return L;
}

// Serving-side slot indirection.  Work item h (0 <= h < rows * H) is head
// h % H of active row h / H, and its blob is that head of slot
// slots[h / H] of the state buffer.  Without a slot array the work item is
// the blob itself.  A slot index outside [0, num_slots) maps to -1: the work
// item is skipped and no blob is touched.
struct SlotMap {
    const int32_t *slots;  // device, one per active row; null = identity
    int heads;             // H
    int num_slots;         // slots in the state buffer
    // blob index of work item h (< 2^31, checked on the host), -1: none.
    // The list is read through L2 only (never a possibly stale L1 line: a
    // kernel may read it before its wait on the kernel that writes it).
    __device__ __forceinline__ int blob(int h) const {
        if (!slots) return h;
        const int row = h / heads;
        const int s = __ldcg(slots + row);
        return (s >= 0 && s < num_slots) ? s * heads + (h - row * heads) : -1;
    }
};

// Runtime switches that do not change a kernel's shape.
struct Flags {
    int kda;        // per-key-channel decay
    int f16_scale;  // qs / sm stored as f16
    int bf16_in;    // q, k, v as bf16
    int smoothing;
    int window;
    int num_comp;
};

// ---------------------------------------------------------------- PTX bits

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the asynchronous (bulk copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes) : "memory");
}

// Expect `bytes` more of transaction on the current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Test for completion of phase `phase`; the thread may sleep in the barrier
// for up to ~1 ms (suspend-time hint) while the phase is still open.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase), "r"(1000000u)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Wait for phase `phase` of `bar`, giving up after kWaitLimitNs.  Returns
// false on timeout (the caller records it and returns; it never spins on).
__device__ __noinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t phase) {
    if (mbar_try_wait(bar, phase)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        if (mbar_try_wait(bar, phase)) return true;
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
}

// One bulk copy global -> this CTA's shared memory (no multicast), completing
// `bytes` of transaction on `bar`.  Addresses 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Bulk prefetch of global memory into L2 (no shared memory, no completion
// tracking, no effect on the data seen later: L2 stays coherent with any
// writer).  Address 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_prefetch_l2(const void *gmem, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gmem), "r"(bytes) : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel on the stream finishes;
// pdl_wait() blocks until that kernel has completed and its memory is
// visible (a no-op for an ordinary launch), so every global access comes
// after it.  pdl_trigger() lets the next such kernel start its own launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void set_status(uint8_t *blob, uint32_t bits) {
    atomicOr(reinterpret_cast<unsigned int *>(blob + kHdrStatus), bits);
}

__device__ __forceinline__ float load_in(const void *p, size_t idx, int bf16) {
    if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[idx]);
    return reinterpret_cast<const float *>(p)[idx];
}

__device__ __forceinline__ float load_scale(const uint8_t *base, int idx, int f16) {
    if (f16) return __half2float(reinterpret_cast<const __half *>(base)[idx]);
    return reinterpret_cast<const float *>(base)[idx];
}

// --------------------------------------------------------- code unpacking
// Codes become exact floats without an int->float conversion instruction:
// a byte b placed in the low mantissa bits of 2^23 gives the float 2^23 + b,
// and subtracting 2^23 + bias recovers the signed code exactly.

__device__ __forceinline__ float byte_to_float(uint32_t word, uint32_t sel_lo) {
    // result bytes: [byte sel_lo of word, 0x00, 0x00, 0x4B]
    return __uint_as_float(__byte_perm(word, 0x4B000000u, 0x7540u | sel_lo));
}

// 16 codes of one group, as exact floats c[0..15] (key index ascending).
template <int BITS>
__device__ __forceinline__ void unpack16(const uint8_t *src, float (&c)[16]) {
    if constexpr (BITS == 8) {
        const uint4 w = *reinterpret_cast<const uint4 *>(src);
        const uint32_t ws[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u, w.z ^ 0x80808080u,
                                w.w ^ 0x80808080u};
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int b = 0; b < 4; ++b) c[4 * q + b] = byte_to_float(ws[q], b) - 8388736.0f;  // 2^23+128
    } else if constexpr (BITS == 4) {
        const uint2 w = *reinterpret_cast<const uint2 *>(src);
        const uint32_t ws[2] = {w.x, w.y};
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint32_t lo = (ws[q] & 0x0F0F0F0Fu) ^ 0x08080808u;         // codes 8q + 2b
            const uint32_t hi = ((ws[q] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;  // codes 8q + 2b + 1
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                c[8 * q + 2 * b] = byte_to_float(lo, b) - 8388616.0f;  // 2^23 + 8
                c[8 * q + 2 * b + 1] = byte_to_float(hi, b) - 8388616.0f;
            }
        }
    } else {  // 6-bit
        const uint32_t *s32 = reinterpret_cast<const uint32_t *>(src);
        const uint32_t w0 = s32[0], w1 = s32[1], w2 = s32[2];
        const uint32_t l0 = (w0 & 0x3F3F3F3Fu) ^ 0x20202020u;
        const uint32_t l1 = (w1 & 0x3F3F3F3Fu) ^ 0x20202020u;
        const uint32_t l2 = (w2 & 0x3F3F3F3Fu) ^ 0x20202020u;
        const uint32_t h = (((w0 >> 6) & 0x03030303u) | ((w1 >> 4) & 0x0C0C0C0Cu) |
                            ((w2 >> 2) & 0x30303030u)) ^ 0x20202020u;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            c[b] = byte_to_float(l0, b) - 8388640.0f;  // 2^23 + 32
            c[4 + b] = byte_to_float(l1, b) - 8388640.0f;
            c[8 + b] = byte_to_float(l2, b) - 8388640.0f;
            c[12 + b] = byte_to_float(h, b) - 8388640.0f;
        }
    }
}

template <int BITS>
__host__ __device__ constexpr int group_bytes() { return 16 * BITS / 8; }

// Pack 16 signed codes (|c| <= Qmax) into one group of the row format.
template <int BITS>
__device__ __forceinline__ void pack16(const int8_t (&c)[16], uint8_t *dst) {
    if constexpr (BITS == 8) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            w[q] = (uint32_t)(uint8_t)c[4 * q] | ((uint32_t)(uint8_t)c[4 * q + 1] << 8) |
                   ((uint32_t)(uint8_t)c[4 * q + 2] << 16) | ((uint32_t)(uint8_t)c[4 * q + 3] << 24);
        *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    } else if constexpr (BITS == 4) {
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int x = 0; x < 16; ++x) w[x >> 3] |= ((uint32_t)c[x] & 0xFu) << (4 * (x & 7));
        *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
    } else {
        uint32_t w[3] = {0u, 0u, 0u};
#pragma unroll
        for (int q = 0; q < 3; ++q)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t lo = (uint32_t)c[4 * q + b] & 0x3Fu;
                const uint32_t hi = (((uint32_t)c[12 + b] & 0x3Fu) >> (2 * q)) & 0x3u;
                w[q] |= (lo | (hi << 6)) << (8 * b);
            }
        uint32_t *d = reinterpret_cast<uint32_t *>(dst);
        d[0] = w[0]; d[1] = w[1]; d[2] = w[2];
    }
}

}  // namespace lq
