// leapquant.cu -- host side of the C ABI declared in include/leapquant.h:
// argument checks, blob layout, and launches of the sm_100a kernels.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>
#include <vector>

#include "leapquant.h"
#include "lq_common.cuh"
#include "lq_decode.cuh"
#include "lq_multi.cuh"
#include "lq_dense.cuh"
#include "lq_flush.cuh"
#include "lq_fp32.cuh"
#include "lq_perstep.cuh"
#include "lq_prefill.cuh"
#include "lq_chunked.cuh"

using namespace lq;

namespace {

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

lq_status check_config(const lq_config *c) {
    if (!c) return LQ_ERR_INVALID_ARG;
    if (c->num_slots <= 0 || c->num_heads <= 0 || c->dk <= 0 || c->dv <= 0 || c->window <= 0 ||
        c->num_comp < 0)
        return LQ_ERR_INVALID_ARG;
    if ((c->decay_kind | c->scale_dtype | c->smoothing | c->in_dtype | c->per_step) & ~1)
        return LQ_ERR_INVALID_ARG;
    if (c->per_step ? (c->bits != 8 && c->bits != 16)
                    : (c->bits != 4 && c->bits != 6 && c->bits != 8 && c->bits != 32))
        return LQ_ERR_INVALID_ARG;
    if ((int64_t)c->num_slots * c->num_heads > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED;
    if (c->dk != c->dv || (c->dk != 64 && c->dk != 128)) return LQ_ERR_UNSUPPORTED;
    if (c->window > kMaxWindow || c->num_comp > kMaxComp) return LQ_ERR_UNSUPPORTED;
    return LQ_OK;
}

Flags make_flags(const lq_config &c) {
    return Flags{c.decay_kind, c.scale_dtype, c.in_dtype, c.smoothing, c.window, c.num_comp};
}

// Allow a kernel more than 48 KB of dynamic shared memory (once per kernel
// and device).
struct SmemGrant {
    int dev;
    const void *fn;
    uint32_t bytes;
};

template <typename K>
cudaError_t allow_smem(K kernel, uint32_t bytes) {
    static std::mutex mu;
    static std::vector<SmemGrant> done;
    if (bytes <= 48u * 1024u) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const void *fn = reinterpret_cast<const void *>(kernel);
    std::lock_guard<std::mutex> lock(mu);
    for (const SmemGrant &g : done)
        if (g.dev == dev && g.fn == fn && g.bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done.push_back({dev, fn, bytes});
    return e;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream drains; it waits for that kernel's
// completion (pdl_wait) before its first global-memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int threads, uint32_t smem, cudaStream_t s,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

lq_status launched(cudaError_t e) {
    if (e != cudaSuccess) return LQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? LQ_OK : LQ_ERR_CUDA;
}

// Persistent grid: as many CTAs as fit on the device at once, each walking
// a strided list of (slot, head) blobs.
template <typename K>
int persistent_grid(K kernel, int threads, uint32_t smem, int work) {
    static std::mutex mu;
    static std::vector<std::pair<std::pair<const void *, uint32_t>, int>> cache;
    const void *fn = reinterpret_cast<const void *>(kernel);
    int per_sm = 0, sms = 0, dev = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (auto &e : cache)
            if (e.first.first == fn && e.first.second == smem) per_sm = e.second;
    }
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return -1;
    if (per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess)
            return -1;
        if (per_sm < 1) per_sm = 1;
        std::lock_guard<std::mutex> lock(mu);
        cache.push_back({{fn, smem}, per_sm});
    }
    const long cap = (long)sms * per_sm;
    return (int)(work < cap ? work : cap);
}

// Largest dynamic shared memory a block of this device may opt into.
int smem_optin_limit() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return -1;
    return v;
}

template <int D, int BITS>
lq_status launch_decode(const lq_config &c, const DecodeArgs &a, cudaStream_t s) {
    const bool multi = a.tokens > 1;
    const uint32_t smem = multi ? multi_smem_bytes(D, a.L, a.F, a.tokens) : decode_smem_bytes(D, a.L, a.F, 1);
    const bool t4 = a.tokens <= 4;
    auto k = a.map.slots ? (multi ? (t4 ? decode_tokens_kernel<D, BITS, true, 4> : decode_tokens_kernel<D, BITS, true, 8>)
                                  : decode_kernel<D, BITS, true, false>)
                         : (multi ? (t4 ? decode_tokens_kernel<D, BITS, false, 4> : decode_tokens_kernel<D, BITS, false, 8>)
                                  : ((a.flags & kEarlyState) ? decode_kernel<D, BITS, false, true>
                                                             : decode_kernel<D, BITS, false, false>));
    const int lim = smem_optin_limit();
    if (lim < 0) return LQ_ERR_CUDA;
    if (smem > (uint32_t)lim) return LQ_ERR_UNSUPPORTED;
    cudaError_t e = allow_smem(k, smem);
    if (e != cudaSuccess) return LQ_ERR_CUDA;
    const int threads = D + 64;
    const int grid = persistent_grid(k, threads, smem, a.num_heads);
    if (grid <= 0) return LQ_ERR_CUDA;
    return launched(launch_pdl(k, grid, threads, smem, s, a));
}

template <int D, int BITS, int MODE>
lq_status launch_boundary(const lq_config &c, const FlushArgs &a, cudaStream_t s) {
    if (MODE == 0) {  // persistent flush
        const uint32_t smem = flush_smem_bytes(D, BITS, a.L, c.window);
        auto k = a.map.slots ? flush_kernel<D, BITS, true> : flush_kernel<D, BITS, false>;
        cudaError_t e = allow_smem(k, smem);
        if (e != cudaSuccess) return LQ_ERR_CUDA;
        const int threads = kGroup;
        const int grid = persistent_grid(k, threads, smem, a.num_heads);
        if (grid <= 0) return LQ_ERR_CUDA;
        return launched(launch_pdl(k, grid, threads, smem, s, a));
    }
    const uint32_t smem = boundary_smem_bytes(D, BITS, a.L, c.window);
    auto k = boundary_kernel<D, BITS, MODE == 0 ? 1 : MODE>;
    cudaError_t e = allow_smem(k, smem);
    if (e != cudaSuccess) return LQ_ERR_CUDA;
    k<<<(unsigned)a.num_heads, kGroup, smem, s>>>(a);
    return launched(cudaSuccess);
}

template <int MODE>
lq_status dispatch_boundary(const lq_config &c, const FlushArgs &a, cudaStream_t s) {
    switch (c.dk * 100 + c.bits) {
        case 12808: return launch_boundary<128, 8, MODE>(c, a, s);
        case 12806: return launch_boundary<128, 6, MODE>(c, a, s);
        case 12804: return launch_boundary<128, 4, MODE>(c, a, s);
        case 6408: return launch_boundary<64, 8, MODE>(c, a, s);
        case 6406: return launch_boundary<64, 6, MODE>(c, a, s);
        case 6404: return launch_boundary<64, 4, MODE>(c, a, s);
        default: return LQ_ERR_UNSUPPORTED;
    }
}

lq_status dispatch_decode(const lq_config &c, const DecodeArgs &a, cudaStream_t s) {
    switch (c.dk * 100 + c.bits) {
        case 12808: return launch_decode<128, 8>(c, a, s);
        case 12806: return launch_decode<128, 6>(c, a, s);
        case 12804: return launch_decode<128, 4>(c, a, s);
        case 6408: return launch_decode<64, 8>(c, a, s);
        case 6406: return launch_decode<64, 6>(c, a, s);
        case 6404: return launch_decode<64, 4>(c, a, s);
        default: return LQ_ERR_UNSUPPORTED;
    }
}

// The dense decode step (FP32 state, or a per-step BF16 / FP8 state):
// persistent, one CTA per SM (the stage ring takes most of shared memory).
template <int D, int FMT>
lq_status launch_dense_step(const DenseArgs &a, cudaStream_t s) {
    const uint32_t smem = dense_smem_bytes(D, FMT, a.F.bf16_in, a.F.kda);
    auto k = dense_step_kernel<D, FMT>;
    if (allow_smem(k, smem) != cudaSuccess) return LQ_ERR_CUDA;
    const int grid = persistent_grid(k, DenseShape<D>::NT, smem, a.num_heads);
    if (grid <= 0) return LQ_ERR_CUDA;
    return launched(launch_pdl(k, grid, DenseShape<D>::NT, smem, s, a));
}

lq_status dispatch_dense_step(const lq_config &c, const DenseArgs &a, cudaStream_t s) {
    const int fmt = c.per_step ? c.bits : 32;
    switch (c.dk * 100 + fmt) {
        case 12832: return launch_dense_step<128, 32>(a, s);
        case 12816: return launch_dense_step<128, 16>(a, s);
        case 12808: return launch_dense_step<128, 8>(a, s);
        case 6432: return launch_dense_step<64, 32>(a, s);
        case 6416: return launch_dense_step<64, 16>(a, s);
        case 6408: return launch_dense_step<64, 8>(a, s);
        default: return LQ_ERR_UNSUPPORTED;
    }
}

// The per-step baselines: one 128-thread CTA per (slot, head) and 64-column
// block.  MODE 0 decode step, 1 store S0, 2 read back.
template <int MODE>
lq_status dispatch_perstep(const lq_config &c, const Fp32Args &a, cudaStream_t s) {
    const int grid = a.num_heads * (c.dk / kPsCols);
    cudaError_t e;
    switch (c.dk * 100 + c.bits) {
        case 12816: e = launch_pdl(perstep_kernel<128, 16, MODE>, grid, kFp32Threads, 0u, s, a); break;
        case 12808: e = launch_pdl(perstep_kernel<128, 8, MODE>, grid, kFp32Threads, 0u, s, a); break;
        case 6416: e = launch_pdl(perstep_kernel<64, 16, MODE>, grid, kFp32Threads, 0u, s, a); break;
        case 6408: e = launch_pdl(perstep_kernel<64, 8, MODE>, grid, kFp32Threads, 0u, s, a); break;
        default: return LQ_ERR_UNSUPPORTED;
    }
    return launched(e);
}

// Blob copy between two state buffers: CTA x moves blob x % H of pair x / H
// with 16-byte loads and stores (a blob is a multiple of 256 bytes).  A pair
// with either slot out of range is skipped.
__global__ void __launch_bounds__(256) copy_slots_kernel(uint8_t *dst, int dst_slots_n, const int32_t *dst_slots,
                                                         const uint8_t *src, int src_slots_n,
                                                         const int32_t *src_slots, int heads, uint32_t blob) {
    const int pair = blockIdx.x / heads, h = blockIdx.x % heads;
    const int sd = __ldg(dst_slots + pair), ss = __ldg(src_slots + pair);
    if (sd < 0 || sd >= dst_slots_n || ss < 0 || ss >= src_slots_n) return;
    const uint4 *from = reinterpret_cast<const uint4 *>(src + ((size_t)ss * heads + h) * blob);
    uint4 *to = reinterpret_cast<uint4 *>(dst + ((size_t)sd * heads + h) * blob);
    for (uint32_t x = threadIdx.x; x < blob / 16u; x += 256u) to[x] = __ldg(from + x);
}

// Diagnostic: one thread waits, through the same bounded wait every kernel
// uses, on a barrier that nothing arrives on; when the wait gives up it
// records LQ_DEV_TIMEOUT in *status (0 if the wait ever succeeded).
__global__ void selftest_wait_kernel(uint32_t *status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    *status = mbar_wait_bounded(&bar, 0u) ? 0u : LQ_DEV_TIMEOUT;
}

// Checks shared by the entry points that take a slot list.
lq_status check_slots(const lq_config *cfg, const void *state, const int32_t *slots, int n_active) {
    lq_status st = check_config(cfg);
    if (st != LQ_OK) return st;
    if (!state || n_active < 0 || (n_active > 0 && !slots)) return LQ_ERR_INVALID_ARG;
    if (cfg->bits == 32 || cfg->per_step) return LQ_ERR_UNSUPPORTED;
    if ((int64_t)n_active * cfg->num_heads > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED;
    if (!aligned(state, 256) || !aligned(slots, 4)) return LQ_ERR_MISALIGNED;
    return LQ_OK;
}

template <int D, int BITS>
lq_status launch_prefill(const PrefillArgs &a, cudaStream_t s) {
    if constexpr (D == 128) {  // the chunkwise form on the tensor cores
        const uint32_t smem = chunk_prefill_smem_bytes(a.F);
        auto k = a.map.slots ? chunk_prefill_kernel<BITS, true> : chunk_prefill_kernel<BITS, false>;
        if (allow_smem(k, smem) != cudaSuccess) return LQ_ERR_CUDA;
        return launched(launch_pdl(k, a.num_heads, kGroup, smem, s, a));
    }
    const uint32_t smem = prefill_smem_bytes(D, BITS, a.F);
    auto k = a.map.slots ? prefill_kernel<D, BITS, true> : prefill_kernel<D, BITS, false>;
    if (allow_smem(k, smem) != cudaSuccess) return LQ_ERR_CUDA;
    return launched(launch_pdl(k, a.num_heads, kGroup, smem, s, a));
}

lq_status prefill_rows(const lq_config *cfg, void *state, const int32_t *slots, int rows, int tokens,
                       const int32_t *lengths, const float *S0, const void *q, const void *k, const void *v,
                       const float *beta, const float *decay, float *out, float *S_final, lq_stream_t stream) {
    const lq_config &c = *cfg;
    if (tokens < 0) return LQ_ERR_INVALID_ARG;
    if (c.bits == 32 || c.per_step) return LQ_ERR_UNSUPPORTED;
    if ((int64_t)rows * (tokens > 0 ? tokens : 1) * c.num_heads > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED;
    if (rows > 0 && tokens > 0 && (!q || !k || !v || !beta || !decay)) return LQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(beta, 4) ||
        !aligned(decay, c.decay_kind ? 16 : 4) || !aligned(out, 4) || !aligned(S0, 16) ||
        !aligned(S_final, 16) || !aligned(lengths, 4))
        return LQ_ERR_MISALIGNED;
    if (rows == 0) return LQ_OK;
    PrefillArgs a{static_cast<uint8_t *>(state), make_layout(c), make_flags(c), S0, q, k, v, beta, decay,
                  lengths, tokens > 0 ? out : nullptr, S_final, tokens, rows * c.num_heads,
                  SlotMap{slots, c.num_heads, c.num_slots}};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (c.dk * 100 + c.bits) {
        case 12808: return launch_prefill<128, 8>(a, s);
        case 12806: return launch_prefill<128, 6>(a, s);
        case 12804: return launch_prefill<128, 4>(a, s);
        case 6408: return launch_prefill<64, 8>(a, s);
        case 6406: return launch_prefill<64, 6>(a, s);
        case 6404: return launch_prefill<64, 4>(a, s);
        default: return LQ_ERR_UNSUPPORTED;
    }
}

template <int MODE>
lq_status launch_fp32_copy(const lq_config &c, const Fp32Args &a, cudaStream_t s) {
    const unsigned grid = (unsigned)(c.num_slots * c.num_heads);
    if (c.dk == 128)
        fp32_copy_kernel<128, MODE><<<grid, 256, 0, s>>>(a);
    else
        fp32_copy_kernel<64, MODE><<<grid, 256, 0, s>>>(a);
    return launched(cudaSuccess);
}

}  // namespace

extern "C" {

lq_status lq_validate_config(const lq_config *cfg) { return check_config(cfg); }

size_t lq_state_bytes(const lq_config *cfg) {
    if (check_config(cfg) != LQ_OK) return 0;
    return make_layout(*cfg).blob;
}

lq_status lq_state_init(const lq_config *cfg, void *state, const float *S0, lq_stream_t stream) {
    lq_status st = check_config(cfg);
    if (st != LQ_OK) return st;
    if (!state || !S0) return LQ_ERR_INVALID_ARG;
    if (!aligned(state, 256) || !aligned(S0, 16)) return LQ_ERR_MISALIGNED;
    const lq_config &c = *cfg;
    const Layout L = make_layout(c);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (c.per_step) {
        Fp32Args a{};
        a.state = static_cast<uint8_t *>(state);
        a.S0 = S0;
        a.L = L;
        a.F = make_flags(c);
        a.num_heads = c.num_slots * c.num_heads;
        return dispatch_perstep<1>(c, a, s);
    }
    if (c.bits == 32) {
        Fp32Args a{};
        a.state = static_cast<uint8_t *>(state);
        a.S0 = S0;
        a.L = L;
        return launch_fp32_copy<1>(c, a, s);
    }
    FlushArgs a{static_cast<uint8_t *>(state), S0, nullptr, L, make_flags(c), c.num_slots * c.num_heads};
    return dispatch_boundary<1>(c, a, s);
}

lq_status lq_decode_step_ex(const lq_config *cfg, void *state, const void *q, const void *k,
                            const void *v, const float *beta, const float *decay, float *out, uint32_t flags,
                            lq_stream_t stream) {
    lq_status st = check_config(cfg);
    if (flags & ~kEarlyState) return LQ_ERR_INVALID_ARG;
    if (st != LQ_OK) return st;
    if (!state || !q || !k || !v || !beta || !decay || !out) return LQ_ERR_INVALID_ARG;
    if (!aligned(state, 256) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) ||
        !aligned(beta, 4) || !aligned(decay, cfg->decay_kind ? 16 : 4) || !aligned(out, 4))
        return LQ_ERR_MISALIGNED;
    const lq_config &c = *cfg;
    const Layout L = make_layout(c);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (c.per_step || c.bits == 32) {
        DenseArgs a{static_cast<uint8_t *>(state), L, make_flags(c), q, k, v, beta, decay, out,
                    c.num_slots * c.num_heads, flags};
        return dispatch_dense_step(c, a, s);
    }
    DecodeArgs a{static_cast<uint8_t *>(state), L, make_flags(c), q, k, v, beta, decay, out,
                 c.num_slots * c.num_heads, SlotMap{nullptr, c.num_heads, c.num_slots}, 1, flags};
    return dispatch_decode(c, a, s);
}

lq_status lq_decode_step(const lq_config *cfg, void *state, const void *q, const void *k,
                         const void *v, const float *beta, const float *decay, float *out,
                         lq_stream_t stream) {
    return lq_decode_step_ex(cfg, state, q, k, v, beta, decay, out, 0u, stream);
}

lq_status lq_window_flush(const lq_config *cfg, void *state, lq_stream_t stream) {
    lq_status st = check_config(cfg);
    if (st != LQ_OK) return st;
    if (!state) return LQ_ERR_INVALID_ARG;
    if (!aligned(state, 256)) return LQ_ERR_MISALIGNED;
    const lq_config &c = *cfg;
    if (c.bits == 32 || c.per_step) return LQ_OK;
    FlushArgs a{static_cast<uint8_t *>(state), nullptr, nullptr, make_layout(c), make_flags(c),
                c.num_slots * c.num_heads};
    return dispatch_boundary<0>(c, a, reinterpret_cast<cudaStream_t>(stream));
}

lq_status lq_dequant_state(const lq_config *cfg, const void *state, float *S_out, lq_stream_t stream) {
    lq_status st = check_config(cfg);
    if (st != LQ_OK) return st;
    if (!state || !S_out) return LQ_ERR_INVALID_ARG;
    if (!aligned(state, 256) || !aligned(S_out, 16)) return LQ_ERR_MISALIGNED;
    const lq_config &c = *cfg;
    const Layout L = make_layout(c);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *st8 = const_cast<uint8_t *>(static_cast<const uint8_t *>(state));
    if (c.per_step) {
        Fp32Args a{};
        a.state = st8;
        a.S_out = S_out;
        a.L = L;
        a.F = make_flags(c);
        a.num_heads = c.num_slots * c.num_heads;
        return dispatch_perstep<2>(c, a, s);
    }
    if (c.bits == 32) {
        Fp32Args a{};
        a.state = st8;
        a.S_out = S_out;
        a.L = L;
        return launch_fp32_copy<2>(c, a, s);
    }
    FlushArgs a{st8, nullptr, S_out, L, make_flags(c), c.num_slots * c.num_heads};
    return dispatch_boundary<2>(c, a, s);
}

lq_status lq_check_status(const lq_config *cfg, const void *state, lq_stream_t stream) {
    lq_status st = check_config(cfg);
    if (st != LQ_OK) return st;
    if (!state) return LQ_ERR_INVALID_ARG;
    if (!aligned(state, 256)) return LQ_ERR_MISALIGNED;
    const lq_config &c = *cfg;
    const Layout L = make_layout(c);
    const size_t n = (size_t)c.num_slots * c.num_heads;
    std::vector<uint32_t> words(n);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpy2DAsync(words.data(), sizeof(uint32_t),
                                      static_cast<const uint8_t *>(state) + kHdrStatus, L.blob,
                                      sizeof(uint32_t), n, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return LQ_ERR_CUDA;
    uint32_t any = 0;
    for (uint32_t w : words) any |= w;
    if (any & LQ_DEV_WINDOW_FULL) return LQ_ERR_WINDOW_FULL;
    if (any & LQ_DEV_RANGE) return LQ_ERR_RANGE;
    if (any & LQ_DEV_TIMEOUT) return LQ_ERR_TIMEOUT;
    if (any & LQ_DEV_CORRUPT) return LQ_ERR_CORRUPT;
    return LQ_OK;
}

lq_status lq_state_init_slots(const lq_config *cfg, void *state, const int32_t *slots, int n_active,
                              const float *S0, lq_stream_t stream) {
    lq_status st = check_slots(cfg, state, slots, n_active);
    if (st != LQ_OK) return st;
    if (n_active > 0 && !S0) return LQ_ERR_INVALID_ARG;
    if (!aligned(S0, 16)) return LQ_ERR_MISALIGNED;
    if (n_active == 0) return LQ_OK;
    const lq_config &c = *cfg;
    FlushArgs a{static_cast<uint8_t *>(state), S0, nullptr, make_layout(c), make_flags(c),
                n_active * c.num_heads, SlotMap{slots, c.num_heads, c.num_slots}};
    return dispatch_boundary<1>(c, a, reinterpret_cast<cudaStream_t>(stream));
}

lq_status lq_decode_step_slots(const lq_config *cfg, void *state, const int32_t *slots, int n_active,
                               const void *q, const void *k, const void *v, const float *beta,
                               const float *decay, float *out, lq_stream_t stream) {
    lq_status st = check_slots(cfg, state, slots, n_active);
    if (st != LQ_OK) return st;
    if (n_active > 0 && (!q || !k || !v || !beta || !decay || !out)) return LQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(beta, 4) ||
        !aligned(decay, cfg->decay_kind ? 16 : 4) || !aligned(out, 4))
        return LQ_ERR_MISALIGNED;
    if (n_active == 0) return LQ_OK;
    const lq_config &c = *cfg;
    DecodeArgs a{static_cast<uint8_t *>(state), make_layout(c), make_flags(c), q, k, v, beta, decay, out,
                 n_active * c.num_heads, SlotMap{slots, c.num_heads, c.num_slots}, 1};
    return dispatch_decode(c, a, reinterpret_cast<cudaStream_t>(stream));
}

// T tokens per (slot, head) in one launch: the plain or slot-list kernel for
// T = 1, the multi-token instance above.
static lq_status decode_tokens(const lq_config *cfg, void *state, const int32_t *slots, int rows, int tokens,
                               const void *q, const void *k, const void *v, const float *beta,
                               const float *decay, float *out, lq_stream_t stream) {
    const lq_config &c = *cfg;
    if (tokens < 1 || tokens > c.window) return LQ_ERR_INVALID_ARG;
    if (tokens > kMaxTokens) return LQ_ERR_UNSUPPORTED;
    if (c.bits == 32 || c.per_step) return LQ_ERR_UNSUPPORTED;
    if ((int64_t)rows * tokens * c.num_heads > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED;
    if (rows > 0 && (!q || !k || !v || !beta || !decay || !out)) return LQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(beta, 4) ||
        !aligned(decay, c.decay_kind ? 16 : 4) || !aligned(out, 4))
        return LQ_ERR_MISALIGNED;
    if (rows == 0) return LQ_OK;
    DecodeArgs a{static_cast<uint8_t *>(state), make_layout(c), make_flags(c), q, k, v, beta, decay, out,
                 rows * c.num_heads, SlotMap{slots, c.num_heads, c.num_slots}, tokens};
    return dispatch_decode(c, a, reinterpret_cast<cudaStream_t>(stream));
}

lq_status lq_decode_steps(const lq_config *cfg, void *state, int tokens, const void *q, const void *k,
                          const void *v, const float *beta, const float *decay, float *out, lq_stream_t stream) {
    lq_status st = check_config(cfg);
    if (st != LQ_OK) return st;
    if (!state) return LQ_ERR_INVALID_ARG;
    if (!aligned(state, 256)) return LQ_ERR_MISALIGNED;
    return decode_tokens(cfg, state, nullptr, cfg->num_slots, tokens, q, k, v, beta, decay, out, stream);
}

lq_status lq_decode_steps_slots(const lq_config *cfg, void *state, const int32_t *slots, int n_active, int tokens,
                                const void *q, const void *k, const void *v, const float *beta,
                                const float *decay, float *out, lq_stream_t stream) {
    lq_status st = check_slots(cfg, state, slots, n_active);
    if (st != LQ_OK) return st;
    return decode_tokens(cfg, state, slots, n_active, tokens, q, k, v, beta, decay, out, stream);
}

lq_status lq_window_flush_slots(const lq_config *cfg, void *state, const int32_t *slots, int n_active,
                                lq_stream_t stream) {
    lq_status st = check_slots(cfg, state, slots, n_active);
    if (st != LQ_OK) return st;
    if (n_active == 0) return LQ_OK;
    const lq_config &c = *cfg;
    FlushArgs a{static_cast<uint8_t *>(state), nullptr, nullptr, make_layout(c), make_flags(c),
                n_active * c.num_heads, SlotMap{slots, c.num_heads, c.num_slots}};
    return dispatch_boundary<0>(c, a, reinterpret_cast<cudaStream_t>(stream));
}

lq_status lq_copy_slots(const lq_config *cfg, void *dst, int dst_num_slots, const int32_t *dst_slots,
                        const void *src, int src_num_slots, const int32_t *src_slots, int n,
                        lq_stream_t stream) {
    lq_status st = check_config(cfg);
    if (st != LQ_OK) return st;
    if (!dst || !src || n < 0 || dst_num_slots <= 0 || src_num_slots <= 0 ||
        (n > 0 && (!dst_slots || !src_slots)))
        return LQ_ERR_INVALID_ARG;
    if ((int64_t)n * cfg->num_heads > 0x7FFFFFFF) return LQ_ERR_UNSUPPORTED;
    if (!aligned(dst, 256) || !aligned(src, 256) || !aligned(dst_slots, 4) || !aligned(src_slots, 4))
        return LQ_ERR_MISALIGNED;
    if (n == 0) return LQ_OK;
    const uint32_t blob = make_layout(*cfg).blob;
    copy_slots_kernel<<<(unsigned)(n * cfg->num_heads), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<uint8_t *>(dst), dst_num_slots, dst_slots, static_cast<const uint8_t *>(src), src_num_slots,
        src_slots, cfg->num_heads, blob);
    return launched(cudaSuccess);
}

lq_status lq_prefill(const lq_config *cfg, void *state, int tokens, const int32_t *lengths, const float *S0,
                     const void *q, const void *k, const void *v, const float *beta, const float *decay,
                     float *out, float *S_final, lq_stream_t stream) {
    lq_status st = check_config(cfg);
    if (st != LQ_OK) return st;
    if (!state) return LQ_ERR_INVALID_ARG;
    if (!aligned(state, 256)) return LQ_ERR_MISALIGNED;
    return prefill_rows(cfg, state, nullptr, cfg->num_slots, tokens, lengths, S0, q, k, v, beta, decay, out,
                        S_final, stream);
}

lq_status lq_prefill_slots(const lq_config *cfg, void *state, const int32_t *slots, int n_active, int tokens,
                           const int32_t *lengths, const float *S0, const void *q, const void *k, const void *v,
                           const float *beta, const float *decay, float *out, float *S_final,
                           lq_stream_t stream) {
    lq_status st = check_slots(cfg, state, slots, n_active);
    if (st != LQ_OK) return st;
    return prefill_rows(cfg, state, slots, n_active, tokens, lengths, S0, q, k, v, beta, decay, out, S_final,
                        stream);
}

lq_status lq_selftest_wait(uint32_t *status, lq_stream_t stream) {
    if (!status) return LQ_ERR_INVALID_ARG;
    if (!aligned(status, 4)) return LQ_ERR_MISALIGNED;
    selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status);
    return launched(cudaSuccess);
}

const char *lq_status_string(lq_status s) {
    switch (s) {
        case LQ_OK: return "ok";
        case LQ_ERR_INVALID_ARG: return "invalid argument";
        case LQ_ERR_UNSUPPORTED: return "configuration not supported by this library";
        case LQ_ERR_CUDA: return "CUDA error";
        case LQ_ERR_WINDOW_FULL: return "decode step into a full window (flush every W steps)";
        case LQ_ERR_RANGE: return "a gate (decay) was negative or NaN";
        case LQ_ERR_MISALIGNED: return "pointer misaligned (see the alignment rule in leapquant.h)";
        case LQ_ERR_TIMEOUT: return "on-chip copy wait timed out";
        case LQ_ERR_CORRUPT: return "state blob header failed its checks";
    }
    return "unknown status";
}

}  // extern "C"
