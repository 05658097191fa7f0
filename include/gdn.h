/*
 * gdn.h -- C ABI of the B200 (sm_100a) Gated Delta Rule chunked forward.
 *
 * The operator is the chunked Gated Delta Rule forward of the page
 * "Qwen3Next Samples" (chunk_gated_delta_rule: "Function Prototype",
 * "Parameter Description", "Mathematical Formulas"): q/k L2 normalisation,
 * per-chunk gate cumulative sum, decay mask, pre-attention matrix, the
 * unit-lower-triangular inverse, value/key cumulative decay, recurrent state
 * attention and the state update, over a packed batch of variable-length
 * sequences.  It computes exactly (up to rounding) the token recurrence of the
 * page "lite_boost.ops.recurrent_gated_delta_rule" (algorithm flow):
 *
 *     S = exp(g_t) S;  kv = S^T kh_t;  S += kh_t (beta_t (v_t - kv))^T;  o_t = S^T qh_t
 *
 * with kh = k / sqrt(|k|^2 + eps), qh = scale * q / sqrt(|q|^2 + eps), per
 * sequence and v-head, v-head h reading qk-head h / (Nv / Nqk).  The initial
 * state comes from a slot pool as on the decode page (state, ssm_state_indices)
 * with one slot per sequence.
 *
 * Fixed sizes: head dimension Dk = Dv = 128 and chunk length L = 128 (both
 * fixed on the "Qwen3Next Samples" page, "Parameter Description/Constraints").
 *
 * Conventions shared by every entry point
 *   - Pointers named "device" are device memory owned by the caller; the
 *     library keeps no pointer after a call returns.  All tensors are dense,
 *     row-major, contiguous.
 *   - bf16 tensors are passed as uint16_t* holding the raw bfloat16 bits.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work on `stream` and returns; it never synchronises.
 *     Argument errors are returned before anything is enqueued.  A launch
 *     failure returns GDN_ERR_CUDA; a fault inside a kernel surfaces at the
 *     caller's next synchronisation, as with any CUDA launch.
 *   - Values are not validated on the hot path: gates are expected <= 0 and
 *     beta in [0, 1] (the decode page leaves both unchecked on purpose, since
 *     a reduction over the inputs would cost a pass on the inference path);
 *     state_indices must lie in [0, P).  On request they are checked on the
 *     device (gdn_check_values, and gdn_set_value_checks for the chunked
 *     path), into status bits GDN_DEV_VAL_*.
 *   - Return value: a gdn_status_t code (0 = success).  It covers what the host
 *     can see when it enqueues.  What only the device can see (a malformed
 *     cu_seqlens, a bounded wait that gave up, a value outside the fp16 range)
 *     goes to the status words of the chunked path's workspace, which
 *     gdn_read_status copies out (see "Device status" below).
 *
 * Device status (the chunked path: gdn_chunk_fwd, gdn_chunk_fwd_rule, the
 * stage calls of gdn_stages.h and gdn_chunk_fwd_noalloc).  The decode page's
 * operator raises ValueError for bad arguments and RuntimeError when
 * execution fails; here the host checks come back as the return code and the
 * device-side findings as four int32 words at the start of the workspace:
 *   [0] input errors.  cu_seqlens: GDN_DEV_CU_FIRST (cu[0] != 0),
 *       GDN_DEV_CU_DECREASING, GDN_DEV_CU_TOTAL (cu[B] != T); the chunk table
 *       clamps every token range to [0, T), so nothing is read or written out
 *       of bounds, but the results are those of the clamped lengths.  With
 *       value checks switched on (gdn_set_value_checks): GDN_DEV_VAL_GATE,
 *       GDN_DEV_VAL_BETA, GDN_DEV_VAL_INDEX (see gdn_check_values).
 *   [1] the number of chunks.
 *   [2] bounded waits that gave up: GDN_DEV_WAIT_STATE, GDN_DEV_WAIT_OUTPUT,
 *       GDN_DEV_WAIT_INTRA (GDN_DEV_WAIT_SELFTEST: the test hook of
 *       gdn_testing.h).  Every wait of a kernel on the tensor core or on a TMA
 *       copy gives up after about 0.3 s instead of hanging; the CTA then stops,
 *       lets its copies drain and frees its tensor memory.
 *   [3] values outside the fp16 range (|x| > 65504) in an fp16 intermediate:
 *       GDN_DEV_RANGE_INTRA (U, or beta v, which shows up in U),
 *       GDN_DEV_RANGE_STATE (the state's fp16 operand copy),
 *       GDN_DEV_RANGE_OUTPUT (the output kernel's fp16 operand),
 *       GDN_DEV_RANGE_INPUT (an fp32 q, k or v element of gdn_chunk_fwd_typed,
 *       which the chunked path rounds to fp16).  A NaN in one of them also
 *       sets the bit.  See "fp16 intermediates" below.
 * Words 0, 2 and 3 are cleared at the start of every chunked call (by the
 * chunk-table kernel, on `stream`, before any kernel that sets a bit), so the
 * words describe the last chunked call on that workspace.  A nonzero word 2 or
 * 3 means that call's out and final_state are not valid.  The fused
 * short-sequence path (1 <= max_seqlen <= GDN_SHORT_MAX) computes in fp32,
 * has no waits and no workspace, and writes no status.
 *
 * fp16 intermediates.  The chunked path's tensor-core operands other than the
 * raw q and k rows are fp16 with fp32 accumulation (11 significant bits
 * against bf16's 8).  Values derived from v and from the initial state (U, the
 * state, the output before its bf16 rounding) must therefore stay within
 * +-65504; beyond that the result is not valid and word 3 says so.  Far below
 * 2^-14 (about 6e-5) fp16 loses significant bits and the result loses
 * accuracy without a flag.  The operator is linear in (v, initial state)
 * jointly, so a caller whose v and states are far outside 1e-3 .. 1e3 in
 * magnitude can scale both by a power of two and scale out and final_state
 * back.  The fused short-sequence path and gdn_recurrent_fwd compute in fp32
 * and have neither limit.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_HEAD_DIM 128 /* Dk = Dv */
#define GDN_CHUNK 128    /* L */
#define GDN_SHORT_MAX 16 /* max_seqlen at or below which the fused short-sequence kernel runs */
#define GDN_NOALLOC_SCRATCH_BYTES (64u << 20) /* static workspace of gdn_chunk_fwd_noalloc, per GPU */
#define GDN_MAX_STATE_WINDOW 8 /* largest state_window of gdn_recurrent_window_fwd */

/* element types of the activations and states of gdn_chunk_fwd_typed, gdn_recurrent_fwd and
   gdn_recurrent_window_fwd */
#define GDN_DTYPE_FP32 0
#define GDN_DTYPE_BF16 1
#define GDN_DTYPE_FP16 2

/* update rules of gdn_chunk_fwd_rule and gdn_recurrent_fwd */
#define GDN_RULE_GATED_DELTA 0
#define GDN_RULE_DELTA 1
#define GDN_RULE_GATED 2
#define GDN_RULE_LINEAR 3

/* bits of the device status words (see "Device status" above) */
#define GDN_DEV_CU_FIRST 1      /* word 0: cu[0] != 0                  */
#define GDN_DEV_CU_DECREASING 2 /* word 0: cu[b+1] < cu[b] for some b   */
#define GDN_DEV_CU_TOTAL 4      /* word 0: cu[B] != T                   */
#define GDN_DEV_VAL_GATE 8      /* word 0: a gate that is not <= 0 (or a NaN)   */
#define GDN_DEV_VAL_BETA 16     /* word 0: a beta outside [0, 1] (or a NaN)     */
#define GDN_DEV_VAL_INDEX 32    /* word 0: a state index outside [0, P)         */
#define GDN_DEV_WAIT_STATE 1    /* word 2: a wait of the state pass gave up     */
#define GDN_DEV_WAIT_OUTPUT 2   /* word 2: a wait of the output kernel gave up  */
#define GDN_DEV_WAIT_INTRA 4    /* word 2: a wait of the intra-chunk kernel gave up */
#define GDN_DEV_WAIT_SELFTEST 8 /* word 2: the wait of gdn_selftest_wait gave up */
#define GDN_DEV_RANGE_INTRA 1   /* word 3: U (or beta v) beyond +-65504         */
#define GDN_DEV_RANGE_STATE 2   /* word 3: the state beyond +-65504             */
#define GDN_DEV_RANGE_OUTPUT 4  /* word 3: the output kernel's fp16 operand beyond +-65504 */
#define GDN_DEV_RANGE_INPUT 8   /* word 3: an fp32 activation beyond +-65504 (gdn_chunk_fwd_typed) */

typedef enum {
    GDN_OK = 0,
    GDN_ERR_NULL_ARG = 1,    /* a required pointer is NULL                              */
    GDN_ERR_BAD_SHAPE = 2,   /* negative size, Nv not a multiple of Nqk, P < B without indices */
    GDN_ERR_UNSUPPORTED = 3, /* size beyond what the kernels handle (see each entry)     */
    GDN_ERR_ALIGNMENT = 4,   /* a pointer breaks the 16-byte alignment rule              */
    GDN_ERR_WORKSPACE = 5,   /* caller workspace smaller than gdn_chunk_fwd_workspace_bytes */
    GDN_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed                     */
    GDN_ERR_OVERLAP = 7,     /* an output buffer overlaps an input buffer                */
    GDN_ERR_SCRATCH_LIMIT = 8 /* gdn_chunk_fwd_noalloc: the sizes need more workspace than
                                 GDN_NOALLOC_SCRATCH_BYTES                                 */
} gdn_status_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *gdn_status_string(int status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int gdn_version(void);

/*
 * gdn_read_status -- copy the four device status words (see "Device status")
 * of a chunked-path workspace into status_out, in order on `stream`.
 *
 *   workspace    the device workspace the chunked call ran on (16-byte aligned)
 *   status_out   int32[4], device memory or host memory (pinned host memory
 *                keeps the copy asynchronous; pageable memory makes the call
 *                wait for `stream`); valid once the copy has completed on
 *                `stream`
 * Errors: GDN_ERR_NULL_ARG, GDN_ERR_ALIGNMENT, GDN_ERR_CUDA.  A call of
 * gdn_chunk_fwd with workspace == NULL frees its internal workspace before it
 * returns, so there is nothing to read afterwards: pass a workspace to read
 * the status.
 */
int gdn_read_status(const void *workspace, int32_t *status_out, void *stream);

/*
 * Value checks on the device (the decode page's "Raises" cases that concern
 * values rather than shapes).  One pass over g and beta ([T, Nv], fp32 and
 * bf16, each optional: NULL skips it) and state_indices ([B], int32, NULL
 * skips it), ORing into the device int32 *status_word:
 *   GDN_DEV_VAL_GATE  for a gate that is not <= 0 (a positive value or a NaN),
 *   GDN_DEV_VAL_BETA  for a beta outside [0, 1] (or a NaN),
 *   GDN_DEV_VAL_INDEX for an index outside [0, P).
 * The word is not cleared first; the call enqueues one kernel on `stream` and
 * returns.  It reads about 6 bytes per (token, v-head), which is why the hot
 * path does not run it unless asked.  Errors: GDN_ERR_NULL_ARG (status_word),
 * GDN_ERR_BAD_SHAPE (negative sizes, Nv <= 0, P < 0), GDN_ERR_ALIGNMENT (g or
 * status_word not 4-byte aligned, beta not 2-byte aligned), GDN_ERR_CUDA.
 */
int gdn_check_values(const float *g, const uint16_t *beta, const int32_t *state_indices, int64_t T, int32_t B,
                     int32_t Nv, int32_t P, int32_t *status_word, void *stream);

/*
 * Process-wide switch of the value checks for the chunked entry points
 * (gdn_chunk_fwd, gdn_chunk_fwd_rule, gdn_chunk_fwd_typed, gdn_chunk_fwd_host,
 * gdn_chunk_fwd_noalloc): when on (nonzero), each call runs gdn_check_values
 * on its g, beta and state_indices (the pool's P) right after the chunk table,
 * into status word 0 of its workspace, so gdn_read_status reports them.  The
 * fused short-sequence path has no workspace and is not covered (call
 * gdn_check_values directly).  Off by default.  Returns the previous setting.
 */
int gdn_set_value_checks(int on);

/*
 * Bytes of device workspace that the chunked path of gdn_chunk_fwd needs for
 * these sizes (the fused short-sequence path needs none).  The workspace holds
 * the per-chunk intermediates of the chunked form: the chunk table, inverse
 * norms, cumulative gates, U, W, U' and the chunk-entry states; its layout is
 * given by gdn_workspace_layout (gdn_stages.h).
 */
size_t gdn_chunk_fwd_workspace_bytes(int64_t T, int32_t B, int32_t Nqk, int32_t Nv);

/*
 * gdn_chunk_fwd -- the whole forward pass.
 *
 *   q, k          device bf16 [T, Nqk, 128]   queries / keys (normalised in the op)
 *   v             device bf16 [T, Nv, 128]
 *   g             device fp32 [T, Nv]         log-space gate per token and v-head
 *   beta          device bf16 [T, Nv]
 *   cu_seqlens    device int32 [B+1]          cu[0] = 0, non-decreasing, cu[B] = T;
 *                                             sequence b holds tokens cu[b] .. cu[b+1]-1
 *   state_pool    device fp32 [P, Nv, 128 (Dk), 128 (Dv)], or NULL for zero initial states
 *   state_indices device int32 [B]            slot of each sequence in state_pool, or
 *                                             NULL for slot b (then P >= B is required)
 *   scale         query scale; <= 0 selects 1/sqrt(128)
 *   eps           L2-norm epsilon (inside the square root; 1e-6 on the prefill page)
 *   out           device bf16 [T, Nv, 128]    written for every token
 *   final_state   device fp32 [B, Nv, 128 (Dk), 128 (Dv)], or NULL (not written);
 *                 must not overlap state_pool
 *   T, B, Nqk, Nv, P   sizes (T = cu[B]); Nv % Nqk == 0
 *   max_seqlen    longest sequence if known, else 0.  A value in 1..GDN_SHORT_MAX
 *                 selects the fused short-sequence kernel (token recurrence on
 *                 the state held on chip); any other value selects the chunked
 *                 kernels.  Both paths are correct for any lengths; the hint
 *                 only chooses the faster one.
 *   workspace     device buffer of workspace_bytes >= gdn_chunk_fwd_workspace_bytes,
 *                 or NULL: the call then allocates and frees it stream-ordered
 *                 (cudaMallocAsync / cudaFreeAsync on `stream`).  Its first 16
 *                 bytes receive the device status words (gdn_read_status).
 *
 * Alignment: q, k, v, out, state_pool, final_state and workspace 16-byte aligned.
 * Limits: T < 2^31, Nqk <= 64, Nv <= 256 (else GDN_ERR_UNSUPPORTED).
 * B == 0 is a no-op.  A sequence of length 0 writes no output and copies its
 * initial state to final_state.
 */
int gdn_chunk_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                  const uint16_t *beta, const int32_t *cu_seqlens, const float *state_pool,
                  const int32_t *state_indices, float scale, float eps, uint16_t *out,
                  float *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P,
                  int32_t max_seqlen, void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_chunk_fwd_rule -- gdn_chunk_fwd with the update rule of the page
 * "com.microsoft.LinearAttention" (attribute update_rule) as an argument;
 * gdn_chunk_fwd is this call with GDN_RULE_GATED_DELTA.
 *
 *   update_rule   GDN_RULE_GATED_DELTA   S = e^g S + k (beta (v - S^T k))^T
 *                 GDN_RULE_DELTA         S = S + k (beta (v - S^T k))^T; g not read (may be NULL)
 *                 GDN_RULE_GATED         S = e^g S + k v^T; beta not read (may be NULL)
 *                 GDN_RULE_LINEAR        S = S + k v^T; g and beta not read
 *                 q and k are L2-normalised in every rule; o = S^T q after the update.
 *
 * The chunked form of the rules without the retrieval (gated, linear) has no
 * triangular inverse: U = V, W = 0, so S_new = e^{g_last} S + k_gexp^T V and
 * o = (e^gamma Q) S + P V; the kernels skip the products with W and Mk.  Every
 * other argument, limit and error as for gdn_chunk_fwd; an update_rule outside
 * 0..3 is GDN_ERR_BAD_SHAPE.
 */
int gdn_chunk_fwd_rule(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                       const uint16_t *beta, const int32_t *cu_seqlens, const float *state_pool,
                       const int32_t *state_indices, float scale, float eps, uint16_t *out,
                       float *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P,
                       int32_t update_rule, int32_t max_seqlen, void *workspace, size_t workspace_bytes,
                       void *stream);

/*
 * gdn_chunk_fwd_typed -- gdn_chunk_fwd_rule with the element types of the page
 * "com.microsoft.LinearAttention" ("Activations and state may independently
 * use float16 or float32"), beside the decode page's bf16 activations and bf16
 * state, and with other head dimensions (the decode page's example has
 * Dk = 64, Dv = 512); gdn_chunk_fwd_rule is this call with bf16 activations,
 * an fp32 state and Dk = Dv = 128.
 *
 *   act_dtype     GDN_DTYPE_BF16, GDN_DTYPE_FP16 or GDN_DTYPE_FP32: the type of
 *                 q, k, v and out
 *   state_dtype   GDN_DTYPE_FP32, GDN_DTYPE_FP16 or GDN_DTYPE_BF16: the type of
 *                 state_pool and final_state (the state itself is carried in
 *                 fp32 on the chip; a 16-bit pool is widened exactly, a 16-bit
 *                 final state rounded to nearest even)
 *   Dk, Dv        head dimensions: Dk 64 or 128, Dv 128, 256, 384 or 512, with
 *                 Nv * Dv / 128 <= 256 (else GDN_ERR_UNSUPPORTED).  Layouts:
 *                 q, k [T, Nqk, Dk]; v, out [T, Nv, Dv]; state_pool [P, Nv, Dk, Dv];
 *                 final_state [B, Nv, Dk, Dv].  The kernels compute on 128 x 128
 *                 states: Dk = 64 runs as 128 with the extra key columns zero
 *                 (exact, at the cost of Dk = 128), and a head of Dv = 128 m runs
 *                 as m heads of 128 value columns that share its q, k, gate and
 *                 beta (the columns of the state evolve independently), so the
 *                 work of T, W and Mk is repeated m times.  scale <= 0 selects
 *                 1/sqrt(Dk).
 *   g, beta       fp32 and bf16 as for gdn_chunk_fwd, in every combination
 *   workspace     >= gdn_chunk_fwd_typed_workspace_bytes(T, B, Nqk, Nv, act_dtype,
 *                 Dk, Dv), or NULL (allocated and freed stream-ordered)
 * bf16 and fp16 rows enter the tensor core as they are (both exact operands);
 * fp32 q, k and v are first rounded to fp16 in the workspace (11 significant
 * bits; an element beyond +-65504 sets GDN_DEV_RANGE_INPUT, see "Device
 * status").  The fused short-sequence kernel serves bf16 activations with an
 * fp32 state and Dk = Dv = 128; everything else runs the chunked kernels for
 * any max_seqlen.  Every other argument, limit and error as for
 * gdn_chunk_fwd_rule; an unknown type code is GDN_ERR_BAD_SHAPE.
 */
size_t gdn_chunk_fwd_typed_workspace_bytes(int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t act_dtype,
                                           int32_t Dk, int32_t Dv);
int gdn_chunk_fwd_typed(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                        const int32_t *cu_seqlens, const void *state_pool, const int32_t *state_indices, float scale,
                        float eps, void *out, void *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv,
                        int32_t P, int32_t update_rule, int32_t act_dtype, int32_t state_dtype, int32_t Dk, int32_t Dv,
                        int32_t max_seqlen, void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_chunk_fwd_noalloc -- gdn_chunk_fwd for callers that cannot allocate
 * device memory.  The pages have no counterpart of this call.
 *
 * Some callers cannot call cudaMalloc or cudaMallocAsync and cannot hand over
 * a workspace either: code running inside a host framework that owns every
 * byte of device memory and forbids allocation while it executes (an inference
 * engine's plugin or custom-op enqueue, a serving runtime that reserved the
 * whole GPU for its state pools up front), or an interface with no place for a
 * workspace argument.  This call takes the same arguments as gdn_chunk_fwd
 * without the workspace and allocates nothing: the chunked path runs on a
 * static device buffer of GDN_NOALLOC_SCRATCH_BYTES (64 MiB) inside this
 * library.  Every GPU on which the library's code is loaded holds one such
 * buffer until the process exits.
 *
 * Limit: sizes whose chunked-path workspace (gdn_chunk_fwd_workspace_bytes)
 * exceeds 64 MiB are rejected with GDN_ERR_SCRATCH_LIMIT before anything is
 * enqueued (at B = 1, Nqk = 16, Nv = 32 the longest sequence that fits is
 * 1920 tokens, 15 chunks; for other sizes compare
 * gdn_chunk_fwd_workspace_bytes with GDN_NOALLOC_SCRATCH_BYTES).  Arguments
 * that gdn_chunk_fwd would refuse (a bad shape, unsupported sizes) get that
 * code first.  The fused short-sequence path (1 <= max_seqlen <=
 * GDN_SHORT_MAX) uses no workspace and has no such limit.
 *
 * The buffer used is the one of the calling thread's current device; `stream`
 * must belong to that device.  The first call on a device looks up the
 * buffer's device address (cudaGetSymbolAddress) and keeps it for the life of
 * the process; make that first call before any stream capture.  The kept
 * address belongs to the device's primary context, which the CUDA runtime
 * uses: a caller that switches the thread to another driver context, or calls
 * cudaDeviceReset after the first call, must not use this entry afterwards.
 * All calls on one device share the buffer,
 * which keeps whatever the previous call left in it (every call clears the
 * status words and writes every other region before reading it, so no call
 * depends on what an earlier one left): calls that can overlap on the GPU
 * (unordered streams, several host threads) race on it and corrupt each
 * other's results, so order them on one stream.  gdn_noalloc_read_status
 * copies the scratch's device status words (see "Device status") of the last
 * chunked call out, without allocating.
 */
int gdn_chunk_fwd_noalloc(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                          const uint16_t *beta, const int32_t *cu_seqlens, const float *state_pool,
                          const int32_t *state_indices, float scale, float eps, uint16_t *out,
                          float *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P,
                          int32_t max_seqlen, void *stream);

/*
 * gdn_noalloc_read_status -- gdn_read_status for the static scratch of
 * gdn_chunk_fwd_noalloc on the current device: copies its four status words
 * into status_out (int32[4], device or host memory) in order on `stream`.
 * Allocates nothing.  GDN_ERR_NULL_ARG, GDN_ERR_CUDA.
 */
int gdn_noalloc_read_status(int32_t *status_out, void *stream);

/*
 * gdn_chunk_fwd_host -- gdn_chunk_fwd from host buffers, with the host <-> device
 * copies overlapped with the compute.
 *
 * The prefill page's operator reuses the state across sequence chunks for
 * streaming inference; this call uses that to stream a batch through the GPU.
 * It cuts the tokens into `segments` pieces at 128-token chunk starts of the
 * sequences (a cut never splits a chunk) and, for each piece, uploads its
 * tokens on a copy stream of the library, runs gdn_chunk_fwd on `stream` once
 * they have landed, and downloads its output rows (and the final states of the
 * sequences that end in it) on a second copy stream, so that piece s+1 uploads
 * while s computes and s-1 downloads.  A sequence cut between two pieces
 * resumes from its fp32 state, exactly as a state crosses a chunk range inside
 * one call: out and final_state equal those of one gdn_chunk_fwd call bit for
 * bit.
 *
 *   q, k, v, g, beta   host, layouts as for gdn_chunk_fwd.  Pinned (page-locked)
 *                 memory lets the copies run asynchronously; pageable memory
 *                 works but each copy then waits for the host.
 *   cu_seqlens    host int32 [B+1]: cu[0] = 0, non-decreasing, cu[B] = T
 *                 (checked on the host: GDN_ERR_BAD_SHAPE otherwise)
 *   state_pool    host fp32 [P, Nv, 128, 128] or NULL; only the B slots named by
 *                 state_indices (host int32 [B], each in [0, P), checked; NULL
 *                 for slot b) are uploaded
 *   out           host bf16 [T, Nv, 128]; final_state host fp32 [B, Nv, 128, 128]
 *                 or NULL.  Both are complete once `stream` has reached the
 *                 point after this call.
 *   segments      number of pieces (> 0), or 0 for 8 from 32768 tokens on, 4
 *                 from 4096 on, else 1
 *   device_buffer device memory of device_bytes >= gdn_chunk_fwd_host_bytes(...)
 *                 with the same cu_seqlens and segments, 256-byte aligned: it
 *                 holds the device copies, the per-piece workspace and the
 *                 carried states (GDN_ERR_WORKSPACE when too small).  Its first
 *                 16 bytes hold the call's four device status words ("Device
 *                 status"), folded over its pieces (words 0, 2 and 3 ORed, word 1
 *                 the total number of chunks): gdn_read_status(device_buffer, ...)
 *                 reads them once the call's work is done
 * Same limits as gdn_chunk_fwd.  Asynchronous on `stream` (and on the library's
 * two copy streams, which fork from and join back into `stream` within the call).
 */
size_t gdn_chunk_fwd_host_bytes(const int32_t *cu_seqlens, int64_t T, int32_t B, int32_t Nqk, int32_t Nv,
                                int32_t with_pool, int32_t segments);
int gdn_chunk_fwd_host(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                       const uint16_t *beta, const int32_t *cu_seqlens, const float *state_pool,
                       const int32_t *state_indices, float scale, float eps, uint16_t *out,
                       float *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P,
                       int32_t segments, void *device_buffer, size_t device_bytes, void *stream);

/*
 * gdn_recurrent_fwd -- token recurrence on a state pool updated in place, with
 * one slot index per token (decode and speculative decoding).
 *
 * Page "lite_boost.ops.recurrent_gated_delta_rule": per token, in this order,
 * S = S * exp(g) * exp(gk); kv_mem = S^T k; S = S + k ((v - kv_mem) * beta)^T;
 * o = S^T q, where exp(gk) decays row i of S (key dimension i) by its own factor,
 * with q and k L2-normalised here (eps inside the square root) and q scaled
 * after the normalisation; every token selects a slot of the state pool through
 * its own index (ssm_state_indices), num_accepted_tokens marks how many tokens
 * of a speculative step were accepted, and the updated pool is the result
 * (state_out).  Where the page leaves the slot use open, this call takes:
 *   - sequence b (tokens t0 = cu[b] .. t1 - 1, n = t1 - t0 >= 1) starts from
 *     state_pool[token_slots[t0 + a - 1]], a = num_accepted[b] clamped to
 *     1 .. n (a = n when num_accepted is NULL): the state after its last
 *     accepted token;
 *   - after token t the state is written to state_pool[token_slots[t]]; a run
 *     of consecutive tokens on one slot writes only its last state, so every
 *     slot ends holding the state after its sequence's last token on it;
 *   - a sequence with no tokens reads and writes nothing.
 * Ordinary decoding puts all tokens of sequence b on one slot (its state is
 * then read from and written back to that slot).
 *
 *   q, k          device [T, Nqk, Dk] of act_dtype
 *   v             device [T, Nv, Dv] of act_dtype
 *   g, beta, cu_seqlens   as for gdn_chunk_fwd
 *   gk            device fp32 [T, Nv, Dk], the key-dimension gate
 *                 (expected <= 0, not checked), or NULL for none
 *   update_rule   GDN_RULE_GATED_DELTA (the rule above), GDN_RULE_DELTA (no decay:
 *                 g and gk are not read and may be NULL), GDN_RULE_GATED
 *                 (S = S * exp(g) * exp(gk) + k v^T: no retrieval, beta not read,
 *                 may be NULL) or GDN_RULE_LINEAR (S = S + k v^T: g, gk and beta
 *                 not read) -- the update rules of the page "com.microsoft.
 *                 LinearAttention" (update_rule); q and k are normalised in
 *                 every rule
 *   state_pool    device [P, Nv, Dk, Dv] of state_dtype, read and written in
 *                 place (required); a 16-bit pool is widened to fp32 on load and
 *                 the fp32 result rounded to nearest even when written
 *   act_dtype, state_dtype   GDN_DTYPE_FP32 / _BF16 / _FP16.  bf16 activations
 *                 (the decode page) take an fp32 or bf16 pool; fp16 or fp32
 *                 activations (the LinearAttention page: activations and state
 *                 each fp16 or fp32) take an fp16 or fp32 pool and need Dk = 128;
 *                 other pairs are GDN_ERR_UNSUPPORTED.  g stays fp32 and beta bf16
 *                 in every combination
 *   token_slots   device int32 [T], each in [0, P) (not checked on the device);
 *                 the slots used by different sequences, including each
 *                 sequence's starting slot, must be disjoint
 *   num_accepted  device int32 [B], or NULL
 *   scale         query scale; <= 0 selects 1/sqrt(Dk)
 *   eps           as for gdn_chunk_fwd
 *   out           device [T, Nv, Dv] of act_dtype, written for every token; must not
 *                 overlap any input or state_pool
 *   T, B, Nqk, Nv, P   sizes (T = cu[B]); Nv % Nqk == 0; P >= 1
 *   Dk, Dv        key and value head dimensions: Dk 64 or 128, Dv a multiple
 *                 of 32 (of 64 with a 16-bit pool) up to 1024 (other values:
 *                 GDN_ERR_UNSUPPORTED); the decode page's example has Dk = 64,
 *                 Dv = 512
 *   max_seqlen    longest sequence if known, else 0.  At most 8 selects the
 *                 kernel variant that stages 8 tokens per sequence (eight CTAs
 *                 per SM); any other value the one that stages 16.  Every
 *                 length is exact; tokens past the staged ones are read from
 *                 global memory one at a time (slower).
 *
 * Alignment: q, k, v, out, state_pool, gk 16-byte aligned; g, cu_seqlens,
 * token_slots, num_accepted 4-byte aligned; beta 2-byte aligned.  Errors:
 * GDN_ERR_NULL_ARG, GDN_ERR_BAD_SHAPE, GDN_ERR_UNSUPPORTED, GDN_ERR_ALIGNMENT,
 * GDN_ERR_OVERLAP before anything is enqueued (an unknown dtype code or
 * update_rule is GDN_ERR_BAD_SHAPE); GDN_ERR_CUDA when the launch fails.  B == 0 or T == 0 is a no-op.  Asynchronous on `stream`; the library
 * keeps no pointer after the call returns.
 */
int gdn_recurrent_fwd(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                      const float *gk, const int32_t *cu_seqlens, void *state_pool, int32_t act_dtype,
                      int32_t state_dtype, int32_t update_rule, const int32_t *token_slots,
                      const int32_t *num_accepted, float scale, float eps, void *out, int64_t T, int32_t B,
                      int32_t Nqk, int32_t Nv, int32_t Dk, int32_t Dv, int32_t P, int32_t max_seqlen,
                      void *stream);

/*
 * gdn_recurrent_window_fwd -- the token recurrence of gdn_recurrent_fwd keeping
 * a window of the most recent states, updated in place.
 *
 * Page "com.microsoft.LinearAttention": attribute state_window (0 to 8) is the
 * number of recent recurrent states kept in present_state, and with a window
 * past_state and present_state carry a leading window axis, shape (W, B, H_kv,
 * d_k, d_v), so that a caller can roll back (for example to undo rejected
 * speculative tokens).  The page gives neither the order of the window nor
 * where a step starts; this call takes a first-in-first-out window in time
 * order:
 *   - entry W - 1 is the newest state, and sequence b continues from
 *     state_window[W - 1, b];
 *   - after each token the new state is appended and the oldest entry leaves,
 *     so after n tokens the window holds the last W of [past entries 0 ..
 *     W - 1, S_1, .., S_n]: with n >= W the states after tokens n - W + 1 ..
 *     n, with n < W the W - n newest past entries moved n places towards
 *     entry 0 followed by S_1 .. S_n; a sequence with no tokens keeps its
 *     window;
 *   - rolling back r tokens of the step is reading entry W - 1 - r.
 * An absent past_state is a window of zero states (the page's default): the
 * caller zero-fills the buffer before the first step.  window = 0 (the page's
 * value for no window axis) keeps only the current state: the buffer is then
 * [B, Nv, Dk, Dv], the same as a window of 1.
 *
 *   state_window  device [max(window, 1), B, Nv, Dk, Dv] of state_dtype, read as
 *                 past_state and overwritten as present_state (required)
 *   window        0 .. GDN_MAX_STATE_WINDOW
 *   every other argument as for gdn_recurrent_fwd (no token slots, no accepted
 *   counts: the window decides where each state goes)
 * Cost: besides the recurrence, a sequence of 1 <= n < W tokens moves W - n of
 * its states inside the buffer before the tokens are applied (a kernel ahead
 * of the recurrence on `stream`); the page's layout puts the newest entry
 * last, which makes that move part of every short step.  Errors as for
 * gdn_recurrent_fwd; a window outside 0 .. 8 is GDN_ERR_BAD_SHAPE.
 */
int gdn_recurrent_window_fwd(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                             const float *gk, const int32_t *cu_seqlens, void *state_window, int32_t window,
                             int32_t act_dtype, int32_t state_dtype, int32_t update_rule, float scale, float eps,
                             void *out, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t Dk, int32_t Dv,
                             int32_t max_seqlen, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
