/*
 * leapquant.h -- C ABI of the B200 (sm_100a) LeapQuant decode library.
 *
 * LeapQuant keeps the recurrent state of Gated DeltaNet (GDN) and Kimi Delta
 * Attention (KDA) heads in 8, 6 or 4 bits.  The state is requantized once per
 * window of W tokens instead of after every token; inside a window the low-bit
 * state is fixed, each token's delta-rule update is kept in FP32 as a rank-one
 * pair, and outputs are computed from the fixed state plus those pairs.  The
 * largest outlier lines of the state are kept aside in FP32 as rank-one
 * compensator pairs, and the remaining residual is balanced per key row
 * before it is quantized.
 * Sources: news post "Linear attention has to move state every token it
 * generates; LeapQuant compresses it to 8-bit without losing accuracy"
 * (paragraphs on per-window quantization, Compensator Tokens and residual
 * smoothing) and "LeapQuant: Efficient Linear Attention with Accurate
 * Recurrent State Quantization" (original abstract).  The pages print no
 * equations; the step used is the delta rule
 *     S' = D_t S,  u_t = beta_t (v_t - S'^T k_t),  S_t = S' + k_t u_t^T,
 *     o_t = S_t^T q_t,
 * with D_t = alpha_t I (GDN) or diag(a_t) (KDA), S dk x dv, row i = key
 * channel, column j = value channel.
 *
 * Conventions for every entry point:
 *  - The caller allocates every buffer (device memory unless stated).  The
 *    library allocates nothing and keeps no state between calls.
 *  - Work is enqueued on `stream` and the call returns without waiting,
 *    except lq_check_status, which synchronizes the stream.
 *  - Argument errors are reported before anything is launched (LQ_ERR_*).
 *    A failed launch returns LQ_ERR_CUDA.  Conditions that depend on data on
 *    the device (a full window, a negative or NaN gate, a timed-out
 *    wait) set a sticky bit in that (slot, head)'s status word; the kernels
 *    then skip that (slot, head) and never trap.  lq_check_status reads them.
 *  - Tensors are dense, row-major, contiguous.  N = num_slots (sequences),
 *    H = num_heads.  The state buffer holds N*H consecutive blobs of
 *    lq_state_bytes(cfg) bytes each, blob (n, h) at index n*H + h.
 *    Alignment (LQ_ERR_MISALIGNED otherwise): the state buffer 256 bytes;
 *    q, k, v, S0, S_out and a KDA decay 16 bytes; beta, a GDN decay and out
 *    4 bytes.
 *  - Calls on one state must be ordered (same stream or explicit events);
 *    calls on disjoint states may run concurrently.
 *
 * Per-(slot, head) blob layout (bits 8/6/4), offsets in bytes, every region
 * 128-byte aligned, total rounded up to 256:
 *    0    header: u32 count (tokens buffered in this window), u32 status
 *         (device error bits), u32 ncomp (compensators in use), u32 magic,
 *         f32 g (GDN: decay product since the window start), pad to 64,
 *         u32 comp_meta[16] at 64 (bit 31: 1 = value column, 0 = key row;
 *         bits 0..30: its index; 0xFFFFFFFF = unused)
 *    128  KDA only: f32 g[dk], decay product per key channel since the
 *         window start
 *    then qs[dv]  quantization scale per value column (f32 or f16)
 *    then sm[dk]  smoothing scale per key row, a power of two (f32 or f16)
 *    then comp_vec[r][max(dk,dv)] f32: the compensator lines (a key row's
 *         values over dv, or a value column's values over dk)
 *    then codes[dv][dk*bits/8]: one row per value column, key index
 *         ascending, groups of 16 codes:
 *           8-bit: 16 bytes, byte b = code b, two's complement;
 *           4-bit: 8 bytes, byte b = code 2b (low nibble) | code 2b+1 (high);
 *           6-bit: 12 bytes = little-endian words w0,w1,w2: codes 4q..4q+3
 *                  in bits 0..5 of the bytes of w_q; code 12+b split over
 *                  bits 6..7 of byte b of w0 (its bits 0-1), w1 (2-3),
 *                  w2 (4-5); 6-bit two's complement.
 *    then pairs[W][dk+dv] f32: buffered pair m = khat_m (dk) then u_m (dv),
 *         khat_m = k_m / g_m (the key in the window-start frame).
 * The dense state the blob stands for is
 *    S = diag(g) ( [sm_i qs_j C_ji] + sum_c p_c w_c^T + sum_{m<count} khat_m u_m^T ).
 * The blob holds no pointers: copying it snapshots or restores a state (a
 * prefix-cache entry after lq_window_flush is the prefix up to `pairs`).
 * bits = 32 (the FP32-state reference): header, then f32 S[dk][dv] at 128.
 *
 * Naive per-step baselines (per_step = 1), the comparison points of the
 * accuracy table of the news post: the dense state is stored in a narrow
 * format after every token, with no window, compensators or smoothing.
 *    bits 16 (BF16): header, then bf16 S[dk][dv] at 128; each entry is the
 *         bfloat16 rounding (ties to even) of its FP32 value.
 *    bits 8 (FP8 E4M3): header, then f32 scale[dv] at 128, then at
 *         128 + align128(4 dv) uint8 codes[dk][dv], row = key channel; for
 *         value column j, scale_j = fl32(max_i |S_ij| / 448) and code_ij =
 *         E4M3(fl32(S_ij / scale_j)), ties to even, saturating at 448 (an
 *         all-zero column has scale 0 and codes 0); the value is
 *         fl32(E4M3 value * scale_j).
 * Per-step INT8 without compensators or smoothing is the LeapQuant layout
 * with window = 1, num_comp = 0, smoothing = 0.
 */
#ifndef LEAPQUANT_H
#define LEAPQUANT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LQ_API __attribute__((visibility("default")))
#else
#define LQ_API
#endif

/* Same object as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st *lq_stream_t;

typedef enum lq_status {
    LQ_OK = 0,
    LQ_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad enum     */
    LQ_ERR_UNSUPPORTED = 2,  /* valid but not built: see lq_validate_config   */
    LQ_ERR_CUDA = 3,         /* a CUDA call or launch failed                  */
    LQ_ERR_WINDOW_FULL = 4,  /* device: decode step into a window of W pairs  */
    LQ_ERR_RANGE = 5,        /* device: a gate (decay) was negative or NaN    */
    LQ_ERR_MISALIGNED = 6,   /* a pointer breaks the alignment rule above     */
    LQ_ERR_TIMEOUT = 7,      /* device: an on-chip copy wait gave up          */
    LQ_ERR_CORRUPT = 8       /* device: a blob header failed its checks       */
} lq_status;

/* Device status bits, ORed into a blob's status word. */
#define LQ_DEV_WINDOW_FULL 0x1u
#define LQ_DEV_RANGE 0x2u
#define LQ_DEV_TIMEOUT 0x4u
#define LQ_DEV_CORRUPT 0x8u

typedef struct lq_config {
    int32_t num_slots;   /* N > 0: independent sequences                      */
    int32_t num_heads;   /* H > 0: heads per sequence (all of one kind)       */
    int32_t dk, dv;      /* per-head state shape; built: dk == dv in {64,128} */
    int32_t window;      /* W in [1, 64]: tokens per quantization window      */
    int32_t num_comp;    /* r in [0, 16]: compensator lines                   */
    int32_t bits;        /* 8, 6, 4 (LeapQuant state) or 32 (FP32 state)      */
    int32_t decay_kind;  /* 0: GDN, one alpha per head; 1: KDA, a per key ch. */
    int32_t scale_dtype; /* 0: qs/sm stored as f32; 1: as f16                 */
    int32_t smoothing;   /* 1: per-key-row residual smoothing; 0: sm = 1      */
    int32_t in_dtype;    /* q, k, v element type: 0 f32, 1 bf16               */
    int32_t per_step;    /* 0: LeapQuant (bits 8/6/4) or FP32 (bits 32);
                            1: naive per-step state, bits 16 = BF16 or
                            bits 8 = FP8 E4M3 (window, num_comp, smoothing and
                            scale_dtype are then not used)                    */
} lq_config;

/* LQ_OK if the configuration is valid and built, else why not.  Host only.
 * Library infrastructure: no passage of the pages defines it. */
LQ_API lq_status lq_validate_config(const lq_config *cfg);

/* Bytes of one (slot, head) blob, a multiple of 256; 0 for an invalid or
 * unsupported configuration.  Host only.  The blob holds what the news post's
 * per-window, Compensator Tokens and residual smoothing paragraphs keep per
 * head (low-bit codes, scales, FP32 compensator lines, the window's FP32
 * pairs); its size is this library's layout, which no passage fixes. */
LQ_API size_t lq_state_bytes(const lq_config *cfg);

/* Enter a sequence: compress N*H dense FP32 states into the blobs.
 *   state [N*H blobs]            out, overwritten entirely (header reset)
 *   S0    [N, H, dk, dv] f32     in, row = key channel
 * Runs the window-boundary compression (compensator extraction, smoothing,
 * quantization) on S0; bits = 32 copies S0; per_step rounds S0 to its
 * format.  Source: the prefill state enters
 * the quantized cache; per-window paragraph of the news post. */
LQ_API lq_status lq_state_init(const lq_config *cfg, void *state, const float *S0, lq_stream_t stream);

/* One decode token for every (slot, head).
 *   state  [N*H blobs]           in/out: appends pair (khat_t, u_t), count++
 *   q, k   [N, H, dk]  in_dtype  in
 *   v      [N, H, dv]  in_dtype  in
 *   beta   [N, H] f32            in, write strength
 *   decay  [N, H] f32 (GDN: alpha) or [N, H, dk] f32 (KDA: a), in [0, 1]
 *   out    [N, H, dv] f32        out, o_t = S_t^T q_t
 * Outputs come from the fixed low-bit state, the compensators and the
 * buffered pairs (abstract; per-window paragraph).  A (slot, head) whose
 * window already holds W pairs, or whose status is nonzero, is skipped: its
 * output row is written as zeros and its state is left unchanged.  Call
 * lq_window_flush after every W steps.
 * Gates may be as small as 0.  The buffered keys are stored divided by the
 * decay product since the window start; when a key channel's product falls
 * below 2^-96 the step first moves the window frame to the current token:
 * that channel's factor is multiplied into its smoothing scale (rounded to
 * the scale's storage type), its compensator entries and the buffered keys,
 * and its product restarts at 1 (the state stands for the same matrix, up to
 * one rounding per stored value).  A negative or NaN gate sets LQ_DEV_RANGE
 * and skips the (slot, head). */
LQ_API lq_status lq_decode_step(const lq_config *cfg, void *state, const void *q, const void *k,
                         const void *v, const float *beta, const float *decay, float *out,
                         lq_stream_t stream);

/* Window boundary for every (slot, head): rebuild the FP32 state from the
 * blob, extract r compensator lines, refresh the smoothing scales,
 * requantize, and reset count = 0, g = 1 (news post: per-window, Compensator
 * Tokens and residual smoothing paragraphs).  A (slot, head) with an empty
 * window (count = 0) is left as is.  May be called on a partial window
 * (sequence end, prefix-cache snapshot).  bits = 32 and per_step: no-op. */
LQ_API lq_status lq_window_flush(const lq_config *cfg, void *state, lq_stream_t stream);

/* Write the dense FP32 state each blob stands for, pending pairs included:
 *   S_out [N, H, dk, dv] f32, out.
 * Evaluated exactly as the flush rebuilds it before requantizing, so the
 * flush of a blob compresses bit-for-bit this matrix.  Source: the state is
 * the fixed low-bit part plus the cached high-precision updates (news post,
 * per-window paragraph) plus the compensator pairs (Compensator Tokens
 * paragraph); the FP32 evaluation order is this library's reading:
 *   S_ij = g_i * ( ((qs_j C_ji) sm_i) + compensators in round order
 *                  + fused multiply-add over the pairs in buffer order ). */
LQ_API lq_status lq_dequant_state(const lq_config *cfg, const void *state, float *S_out,
                           lq_stream_t stream);

/* Synchronize `stream`, OR the status words of all N*H blobs and map them to
 * the first set error (WINDOW_FULL, RANGE, TIMEOUT, CORRUPT).  `state` is a
 * device pointer; the read uses one strided device-to-host copy.  Library
 * infrastructure (failure detection): no passage of the pages defines it. */
LQ_API lq_status lq_check_status(const lq_config *cfg, const void *state, lq_stream_t stream);

/* lq_decode_step with call flags:
 *   LQ_STEP_EARLY_STATE  no kernel that may still be running when this step
 *      starts writes `state`.  The library launches with programmatic
 *      dependent launch, so the step can start while the kernel enqueued just
 *      before it drains; it then stages its first blob's compact state and
 *      codes at once, and reads q, k, v, beta and decay only after that
 *      kernel has completed.  The promise holds when (a) the kernel just
 *      before this call does not write `state`, and (b) that kernel is not a
 *      programmatic-dependent launch, or triggers its dependents only after
 *      its own dependency wait (every kernel of this library does), so that
 *      no kernel further back can still be running.  True in a model when
 *      the previous kernel is, say, the projection that produces q, k, v;
 *      false when two steps on the same state follow each other directly.  A
 *      wrong promise reads stale state.
 * Other bits: LQ_ERR_INVALID_ARG.  The flag applies to every format: for
 * bits = 32 and the per_step states the dense state of the first heads is
 * staged early in the same way. */
#define LQ_STEP_EARLY_STATE 0x1u
LQ_API lq_status lq_decode_step_ex(const lq_config *cfg, void *state, const void *q, const void *k,
                                   const void *v, const float *beta, const float *decay, float *out,
                                   uint32_t flags, lq_stream_t stream);

/* T consecutive tokens for every (slot, head) in one launch (speculative
 * verification, multi-token prediction): the compact state is read once for
 * all T tokens.  Token t's output and pair equal those of the t-th of T
 * lq_decode_step calls on the same inputs, bit for bit.
 *   tokens  T, 1 <= T <= W (LQ_ERR_INVALID_ARG otherwise) and T <= 8
 *           (LQ_ERR_UNSUPPORTED above)
 *   q, k    [N, T, H, dk]  in_dtype   v [N, T, H, dv]  in_dtype
 *   beta    [N, T, H] f32;  decay [N, T, H] f32 (GDN) or [N, T, H, dk] (KDA)
 *   out     [N, T, H, dv] f32
 * A (slot, head) whose window lacks room for T more pairs is skipped as a
 * whole (LQ_DEV_WINDOW_FULL, zero outputs).  If token t fails its range
 * check, tokens t.. of that (slot, head) are skipped (zero outputs) and the
 * state keeps the pairs of tokens < t.  bits 8/6/4 only (others:
 * LQ_ERR_UNSUPPORTED); LQ_ERR_UNSUPPORTED too when the launch's shared
 * memory (two stages of W pair slots and T tokens' inputs, plus per-token
 * scratch) exceeds what a block of the device may use, which no
 * configuration within the limits of lq_validate_config reaches on a B200.
 * T = 1 is lq_decode_step.  Every token is committed;
 * to keep only an accepted prefix (speculative decoding), snapshot the rows
 * first with lq_copy_slots, restore the rows that rejected tokens and decode
 * their accepted prefix again. */
LQ_API lq_status lq_decode_steps(const lq_config *cfg, void *state, int tokens, const void *q,
                                 const void *k, const void *v, const float *beta, const float *decay,
                                 float *out, lq_stream_t stream);

/* Enter a prompt: for every (slot, head), run the delta rule in FP32 over its
 * prompt from S0 (or from a zero state), then compress the final state into
 * a fresh blob (count 0, g 1, status cleared) as lq_state_init does with S0.
 * The FP32 state stays on chip between the last token and the compression.
 * Source: the state a prefill leaves enters the quantized cache (news post,
 * per-window paragraph); the step is the delta rule of lq_decode_step.
 *   tokens   T >= 0 (T = 0: lq_state_init from S0, or from zeros)
 *   lengths  [N] int32, device, or NULL: row n's prompt is its first
 *            clamp(lengths[n], 0, T) tokens; later tokens are ignored
 *   S0       [N, H, dk, dv] f32 or NULL (zero state)
 *   q, k     [N, T, H, dk] in_dtype     v [N, T, H, dv] in_dtype
 *   beta     [N, T, H] f32;  decay [N, T, H] (GDN) or [N, T, H, dk] (KDA)
 *   out      [N, T, H, dv] f32 or NULL: o_t = S_t^T q_t, zero past a row's
 *            length
 *   S_final  [N, H, dk, dv] f32 or NULL: the FP32 state that was compressed
 * bits 8/6/4 only (others: LQ_ERR_UNSUPPORTED).  Alignment: S0, S_final 16
 * bytes, lengths 4, the rest as lq_decode_step. */
LQ_API lq_status lq_prefill(const lq_config *cfg, void *state, int tokens, const int32_t *lengths,
                            const float *S0, const void *q, const void *k, const void *v,
                            const float *beta, const float *decay, float *out, float *S_final,
                            lq_stream_t stream);

/* ---- Serving: a subset of the sequences through a slot list ----------
 * A continuous-batching server keeps N sequence slots in one state buffer
 * and decodes, at each step, only the sequences that are running.  The
 * entry points below take those as a device list of slot indices:
 *   slots  [n_active] int32, device, in: row n of the row-indexed tensors
 *          belongs to the sequence in slot slots[n] (blobs slots[n]*H + h).
 *          Entries must be distinct (two rows on one slot race: the result
 *          is undefined, every access still stays inside the buffers).
 * Every kernel bounds-checks each entry against [0, N): a row whose slot is
 * out of range touches no blob; its output row (decode) is written as
 * zeros.  n_active = 0 launches nothing and returns LQ_OK.  The init,
 * decode, prefill and flush calls below take the LeapQuant formats only
 * (bits 8/6/4, per_step = 0), else LQ_ERR_UNSUPPORTED; lq_copy_slots takes
 * any format.  The list is read on the device when the kernel runs, so it
 * may be written by earlier work on the same stream. */

/* lq_state_init for the slots in `slots`:
 *   S0 [n_active, H, dk, dv] f32, in (row n enters slot slots[n]).
 * Status words of those slots are reset; other slots are not touched. */
LQ_API lq_status lq_state_init_slots(const lq_config *cfg, void *state, const int32_t *slots,
                                     int n_active, const float *S0, lq_stream_t stream);

/* lq_decode_step for the slots in `slots`: q, k, v, beta, decay and out are
 * laid out as for lq_decode_step with n_active rows in place of N.  The
 * results of a row equal those lq_decode_step gives for that slot. */
LQ_API lq_status lq_decode_step_slots(const lq_config *cfg, void *state, const int32_t *slots,
                                      int n_active, const void *q, const void *k, const void *v,
                                      const float *beta, const float *decay, float *out,
                                      lq_stream_t stream);

/* lq_decode_steps for the slots in `slots` (row n of the [n_active, T, ...]
 * tensors belongs to slot slots[n]). */
LQ_API lq_status lq_decode_steps_slots(const lq_config *cfg, void *state, const int32_t *slots,
                                       int n_active, int tokens, const void *q, const void *k,
                                       const void *v, const float *beta, const float *decay,
                                       float *out, lq_stream_t stream);

/* lq_prefill into the slots in `slots` (row n of S0, q, k, v, beta, decay,
 * lengths, out and S_final belongs to slot slots[n]): new requests enter
 * free slots while the others keep decoding. */
LQ_API lq_status lq_prefill_slots(const lq_config *cfg, void *state, const int32_t *slots,
                                  int n_active, int tokens, const int32_t *lengths, const float *S0,
                                  const void *q, const void *k, const void *v, const float *beta,
                                  const float *decay, float *out, float *S_final, lq_stream_t stream);

/* lq_window_flush for the slots in `slots` (slots reach their window
 * boundary at different steps when sequences join at different times). */
LQ_API lq_status lq_window_flush_slots(const lq_config *cfg, void *state, const int32_t *slots,
                                       int n_active, lq_stream_t stream);

/* Copy whole sequences between two state buffers with the blob layout of
 * `cfg` (its num_slots is not used; any format, per_step and bits = 32
 * included): for i < n, the H blobs of slot src_slots[i] of `src` (which
 * holds src_num_slots slots) go to slot dst_slots[i] of `dst` (dst_num_slots
 * slots).  Both lists are device int32 arrays; a pair with either index out
 * of range is skipped.  A prefix cache snapshots a flushed sequence into a
 * pool with it and restores it into a serving slot; the bytes are copied
 * as they are, so a restored sequence continues bit for bit.  Source and
 * destination blobs must not overlap. */
LQ_API lq_status lq_copy_slots(const lq_config *cfg, void *dst, int dst_num_slots,
                               const int32_t *dst_slots, const void *src, int src_num_slots,
                               const int32_t *src_slots, int n, lq_stream_t stream);

/* Diagnostic of the device-side failure detection: one kernel thread waits,
 * through the bounded wait every kernel of this library uses, on an on-chip
 * barrier that nothing ever arrives on.  The wait gives up after its time
 * limit (one second) and the kernel writes LQ_DEV_TIMEOUT to *status (a
 * device uint32, 4-byte aligned), then exits: the context stays usable.
 * Enqueued on `stream`; the call does not wait. */
LQ_API lq_status lq_selftest_wait(uint32_t *status, lq_stream_t stream);

/* Static text for a status code.  Library infrastructure. */
LQ_API const char *lq_status_string(lq_status s);

#ifdef __cplusplus
}
#endif

#endif /* LEAPQUANT_H */
