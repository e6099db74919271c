/*
 * sdm.h -- C ABI of the B200 (sm_100a) Sparse Delta Memory memory pass.
 *
 * The pass follows the four-step method of "Sparse Delta Memory: Scaling the State of
 * Linear RNNs through Sparsity" (paper.rainbus.top summary, method paragraph), for one
 * SDM layer whose inputs are already projected:
 *   step 1  product-key top-k slot selection (write keys and read queries),
 *   step 2  gated delta write on the selected write slots only,
 *   step 3  sparse read of the selected read slots, after the token's write,
 *   step 4  RMS normalisation and elementwise output gating (the head-mixing
 *           projection W_o is not part of this library).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer is a DEVICE pointer owned by the caller, 16-byte aligned, to a
 *    contiguous row-major array.  The library allocates no memory; scratch space comes
 *    from the caller through `ws` (size from sdm_workspace_size).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *    Calls are asynchronous on that stream; calls on different streams may run
 *    concurrently as long as they touch disjoint outputs.
 *  - Arguments are validated on the host before anything is launched.  A rejected call
 *    returns SDM_ERR_INVALID_ARG (or SDM_ERR_UNSUPPORTED) and has no effect.  A failed
 *    launch returns SDM_ERR_CUDA.  Conditions detected on the device are recorded in a
 *    per-device status word that sdm_get_device_status() reads and clears.
 *  - Shapes: N = S1*S2 memory slots per head; the flat slot index of the pair
 *    (i1 in the first half, i2 in the second) is i1*S2 + i2.
 *  - Selection order, at every stage: score descending, then slot index ascending;
 *    -0 and +0 are the same score.  Scores are sums of two fp32 half scores (bf16
 *    halves are widened exactly), added once in fp32 round-to-nearest.  NaN scores
 *    are outside the supported domain.
 *  - Slot weights: softmax (temperature 1) of the selected scores over the selected set
 *    ("sparse key value" k^(i) of the write, q^(i) of the read).
 *  - Limits: 1 <= S1, S2 <= 4096; 1 <= W, R <= min(S1, S2, 128); d_v a multiple of 4
 *    (fp32 inputs) or of 8 (bf16 inputs), 8 <= d_v <= 1024 for bf16, 4 <= d_v <= 1024 for
 *    fp32.  N <= 2^31 - 1.
 */
#ifndef SDM_H
#define SDM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SDM_OK = 0,
    SDM_ERR_INVALID_ARG = 1,  /* a pointer, size, alignment or enum is not accepted     */
    SDM_ERR_UNSUPPORTED = 2,  /* valid request that the library does not implement    */
    SDM_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed            */
    SDM_ERR_DEVICE_CHECK = 4, /* a kernel found an out-of-range index in its inputs     */
    SDM_ERR_TIMEOUT = 5       /* a bounded wait inside a kernel ran out                 */
} sdm_status;

typedef enum { SDM_F32 = 0, SDM_BF16 = 1 } sdm_dtype;
typedef enum {
    SDM_ENGINE_AUTO = 0,
    SDM_ENGINE_SEQ = 1,
    SDM_ENGINE_SLOT = 2,
    SDM_ENGINE_CHUNK = 3
} sdm_engine;
typedef enum { SDM_INIT_FROM_M0 = 0, SDM_CONTINUE = 1 } sdm_init;
typedef enum { SDM_GATE_SILU = 0, SDM_GATE_SIGMOID = 1, SDM_GATE_IDENTITY = 2 } sdm_gate_act;

/* Problem shape.  B sequences, T tokens, H heads, S1 + S2 half scores per (token, head),
 * W write slots and R read slots per token, d_v value width.  in_dtype (an sdm_dtype)
 * is the element type of the score halves, v and the gate; alpha, beta, M0, M, y and o
 * are always fp32. */
typedef struct {
    int32_t B, T, H, S1, S2, W, R, d_v;
    int32_t in_dtype;
} sdm_shape;

/*
 * Step 1 alone: product-key top-K selection [paper.rainbus.top summary, method step 1;
 * ai-paper-analysis.pages.dev SDM write-up, 步骤 1].  For each of the B*T*H rows of
 * `halves` ([B,T,H,S1+S2], first half then second half, in_dtype) the K slots with the
 * largest outer-sum scores, in selection order, and their softmax weights.
 *   idx [B,T,H,K] int32 flat slot indices; wt [B,T,H,K] fp32 weights.
 * Uses shape.B, T, H, S1, S2, in_dtype; K replaces W/R (1 <= K <= min(S1, S2, 128)).
 */
sdm_status sdm_select(const void *halves, sdm_shape shape, int32_t K, int32_t *idx, float *wt,
                      void *stream);

/* Bytes of scratch that sdm_scan_forward needs for this shape and engine: the selections
 * of every token (B*T*H*(W+R) indices and weights), plus for the slot engine the events of
 * one time chunk (double-buffered for the radix sort), its histogram and its long-segment
 * list.  SDM_ENGINE_AUTO reserves room for either engine.  Returns 0 for an invalid shape. */
size_t sdm_workspace_size(sdm_shape shape, int32_t engine);

/*
 * Learnable initial memory [ai-paper-analysis.pages.dev SDM write-up, section on the
 * learned initial state M0; m.163.com article, section 三]: M0 [H,N,d_v] is shared by
 * every sequence, so M[b,h,:,:] = M0[h,:,:] for every b.  M [B,H,N,d_v]; M must not
 * overlap M0.
 */
sdm_status sdm_state_init(const float *M0, float *M, sdm_shape shape, void *stream);

/*
 * Prefill: steps 1-4 over T tokens for every (b, h) [paper.rainbus.top summary, method
 * steps 1-4].  Token t of sequence b, head h:
 *   I_w, k = top-W selection of kp[b,t,h,:];  I_r, q = top-R selection of qp[b,t,h,:]
 *   for i in I_w:  M~ = alpha[b,t,h] * M[b,h,i,:]
 *                  M[b,h,i,:] = M~ + beta[b,t,h] * k_i * (v[b,t,h,:] - M~)
 *   y[b,t,h,:] = sum_{i in I_r} q_i * M[b,h,i,:]        (after token t's write)
 *   o[b,t,h,:] = y * rsqrt(mean(y^2) + eps) * gamma * act(gate[b,t,h,:])
 * Arguments:
 *   kp, qp   [B,T,H,S1+S2] in_dtype     v, gate [B,T,H,d_v] in_dtype (gate nullable:
 *                                        no gating factor)
 *   alpha, beta [B,T,H] fp32             M0 [H,N,d_v] fp32 (read only with
 *                                        init == SDM_INIT_FROM_M0, may then be NULL
 *                                        otherwise)
 *   M        [B,H,N,d_v] fp32, in/out: the recurrent state.  init == SDM_INIT_FROM_M0
 *            first sets it to M0; SDM_CONTINUE resumes from its current contents.
 *   y        [B,T,H,d_v] fp32 out.       o [B,T,H,d_v] fp32 out, nullable (no step 4)
 *   gamma    [d_v] fp32, nullable (unit weight).   eps >= 0.   act: sdm_gate_act.
 *   sel_out  nullable int32 out: the selected write slots [B,T,H,W] followed by the
 *            read slots [B,T,H,R], in selection order (for parity checks).
 *   engine   sdm_engine; ws / ws_bytes caller scratch of at least
 *            sdm_workspace_size(shape, engine) bytes, 256-byte aligned.
 *            SDM_ENGINE_SEQ walks the tokens of each (b, h) in order; SDM_ENGINE_SLOT
 *            sorts the writes and reads by slot and runs every slot's recurrence;
 *            SDM_ENGINE_CHUNK is the chunk-wise form [m.163.com article, section 八, the
 *            training-implementation paragraph]: chunks of up to 32 tokens, inside a chunk
 *            the reads as y_t = sum_i q_t(i) e^{L(t,i)} M0[i] + sum_{s<=t} A[t,s] v_s, with
 *            L(t,i) the summed ln(alpha (1 - beta k)) of slot i's writes in the chunk up to
 *            t and A[t,s] the sparse inner product of token t's read list and token s's
 *            write list (a two-pointer merge of the lists in slot order); the state is
 *            carried from chunk to chunk.  It expects alpha (1 - beta k) >= 0 (alpha >= 0,
 *            beta k <= 1, as with alpha = exp(-softplus), beta a sigmoid) and agrees with the
 *            other engines to fp32 rounding of the exponentials.  AUTO picks SEQ or SLOT.
 * T == 0 is valid: only the initialisation (if requested) happens.
 */
sdm_status sdm_scan_forward(const void *kp, const void *qp, const void *v, const float *alpha,
                            const float *beta, const float *M0, float *M, int32_t init,
                            float *y, const void *gate, const float *gamma, float eps,
                            int32_t act, float *o, int32_t *sel_out, int32_t engine, void *ws,
                            size_t ws_bytes, sdm_shape shape, void *stream);

/*
 * Prefill with the coupled delta rule.  The write of [paper.rainbus.top summary, method step
 * 2] predicts each written slot from its own row, M~[i]; the SDM write-up on
 * ai-paper-analysis.pages.dev and the m.163.com article (section 二) also state that SDM
 * reduces exactly to the gated delta rule when every slot is selected, which holds only when
 * the token's written rows share one prediction:
 *   p_t = sum_{j in I_w} k_j * alpha_t * M[j]
 *   M[i] = alpha_t * M[i] + beta_t * k_i * (v_t - p_t)      for i in I_w
 * (with I_w all N slots: M_t = alpha_t (I - beta_t k k^T) M_{t-1} + beta_t k v_t^T).  The
 * read and step 4 are those of sdm_scan_forward, and so are the arguments.  The sequential
 * engine computes it (SDM_ENGINE_AUTO takes it); the slot and chunk-wise engines, which treat
 * every slot as its own recurrence, cannot: SDM_ENGINE_SLOT and SDM_ENGINE_CHUNK return
 * SDM_ERR_UNSUPPORTED.
 */
sdm_status sdm_scan_forward_coupled(const void *kp, const void *qp, const void *v,
                                    const float *alpha, const float *beta, const float *M0,
                                    float *M, int32_t init, float *y, const void *gate,
                                    const float *gamma, float eps, int32_t act, float *o,
                                    int32_t *sel_out, int32_t engine, void *ws, size_t ws_bytes,
                                    sdm_shape shape, void *stream);

/* Size of the fixed scratch of sdm_scan_forward_noalloc (16 MiB per device). */
#define SDM_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * Prefill that allocates nothing (no paper counterpart: a deployment variant of
 * sdm_scan_forward).  It is for callers that cannot allocate device memory while the pass
 * runs: a host engine that owns all device memory in its own pool, a plugin interface
 * without a workspace argument, or a loop that must not call the CUDA allocator once
 * running.  The arguments and results are those of sdm_scan_forward with the sequential
 * engine; the scratch is a fixed device array of SDM_NOALLOC_SCRATCH_BYTES that the library
 * holds on every device that loads it, until the process exits.
 *  - The shape's scratch, sdm_workspace_size(shape, SDM_ENGINE_SEQ), must not exceed
 *    SDM_NOALLOC_SCRATCH_BYTES; a larger shape returns SDM_ERR_INVALID_ARG and launches
 *    nothing (for W = R = 64 that is up to 16384 (sequence, token, head) rows per call).
 *  - The first call on a device looks up the array's device address (once per device);
 *    make that first call before capturing any stream into a CUDA graph.
 *  - Every call on a device shares the one array, which keeps the last call's contents.
 *    Nothing in it needs to start at zero (each call rewrites what it reads), but calls
 *    that overlap on the GPU (different streams, or host threads, at the same time) race
 *    on it: serialise them.
 *  - Calls no cudaMalloc, cudaFree or other allocating routine.
 */
sdm_status sdm_scan_forward_noalloc(const void *kp, const void *qp, const void *v,
                                    const float *alpha, const float *beta, const float *M0,
                                    float *M, int32_t init, float *y, const void *gate,
                                    const float *gamma, float eps, int32_t act, float *o,
                                    int32_t *sel_out, sdm_shape shape, void *stream);

/*
 * Decode: steps 1-4 for ONE token of each of B sequences and H heads, in one fused
 * launch [paper.rainbus.top summary, method steps 1-4; m.163.com article, section 八,
 * on decode].  Same arithmetic as sdm_scan_forward with T = 1 and SDM_CONTINUE:
 *   kp, qp [B,H,S1+S2] in_dtype; v, gate [B,H,d_v] in_dtype (gate nullable);
 *   alpha, beta [B,H] fp32; M [B,H,N,d_v] fp32 in/out; y [B,H,d_v] fp32 out;
 *   o [B,H,d_v] fp32 out, nullable; gamma [d_v] nullable;
 *   sel_out nullable: write slots [B,H,W] followed by read slots [B,H,R].
 * shape.T is ignored.  No scratch memory is used.  The kernel is launched in plain stream
 * order: it starts once the work ahead of it on the stream has finished.
 */
sdm_status sdm_decode_step(const void *kp, const void *qp, const void *v, const float *alpha,
                           const float *beta, float *M, float *y, const void *gate,
                           const float *gamma, float eps, int32_t act, float *o,
                           int32_t *sel_out, sdm_shape shape, void *stream);

/*
 * sdm_decode_step for a chain of decode steps whose inputs are all in device memory before
 * the chain starts (same arguments, same results).  The launch allows programmatic stream
 * serialisation: the step's selection, which reads only kp, qp, v, gate, alpha, beta and
 * gamma, may run while the kernel ahead of it on the stream is finishing (typically the
 * previous step), and the step waits for that kernel before it touches M, y, o or sel_out.
 * Precondition, which the library cannot check: the kernel launched right before this one
 * writes none of this step's inputs.  A kernel that produces them (a projection, for
 * instance) may let its dependents start before its own stores are visible; after such a
 * kernel call sdm_decode_step instead.  sdm_set_option(SDM_OPT_NO_PDL, 1) makes this call
 * launch in plain stream order.
 */
sdm_status sdm_decode_step_chained(const void *kp, const void *qp, const void *v,
                                   const float *alpha, const float *beta, float *M, float *y,
                                   const void *gate, const float *gamma, float eps,
                                   int32_t act, float *o, int32_t *sel_out, sdm_shape shape,
                                   void *stream);

/*
 * One decode step with the coupled delta rule of sdm_scan_forward_coupled (arguments and
 * launch as sdm_decode_step / sdm_decode_step_chained).  The write rows are summed in shared
 * memory: shapes with W * d_v * 4 > 65536 bytes return SDM_ERR_UNSUPPORTED.
 */
sdm_status sdm_decode_step_coupled(const void *kp, const void *qp, const void *v,
                                   const float *alpha, const float *beta, float *M, float *y,
                                   const void *gate, const float *gamma, float eps, int32_t act,
                                   float *o, int32_t *sel_out, sdm_shape shape, void *stream);
sdm_status sdm_decode_step_coupled_chained(const void *kp, const void *qp, const void *v,
                                           const float *alpha, const float *beta, float *M,
                                           float *y, const void *gate, const float *gamma,
                                           float eps, int32_t act, float *o, int32_t *sel_out,
                                           sdm_shape shape, void *stream);

/*
 * Step 4 alone [paper.rainbus.top summary, method step 4]: for each of the B*T*H rows
 * of y [B,T,H,d_v] (fp32), o = y * rsqrt(mean(y^2) + eps) * gamma * act(gate).
 * gate [B,T,H,d_v] in_dtype, nullable; gamma [d_v] fp32, nullable.  o may equal y.
 */
sdm_status sdm_norm_gate(const float *y, const void *gate, const float *gamma, float eps,
                         int32_t act, sdm_shape shape, float *o, void *stream);

/*
 * Prefill that also keeps the undo log of its in-place writes [m.163.com article on SDM,
 * section 八, the memory-efficiency paragraph: the state is updated in place and the
 * updates are undone during backpropagation, so that one state and the overwritten rows,
 * O(N d + T W d), are kept instead of a state per chunk].  Arguments, engines and results
 * as sdm_scan_forward (the per-slot rule); in addition, for write j of token row
 * r = (b * T + t) * H + h, wlog[(r * W + j) * d_v + c] receives the written row as that
 * write found it, before the write.  wlog: fp32 [B,T,H,W,d_v], device, 16-byte aligned, not
 * overlapping M or y; NULL is SDM_ERR_INVALID_ARG (T > 0).  Keep sel_out as well: the undo
 * needs the write slots.  The sequential and slot engines keep the log; SDM_ENGINE_CHUNK
 * returns SDM_ERR_UNSUPPORTED.  The log holds the engine's own row values: the slot engine's hot
 * slots are stepped by composed affine maps, so an entry after a slot's first write in a
 * chunk can differ from a token-by-token state by rounding; each slot's first logged entry
 * in the pass is the starting row exactly.  To keep a smaller log, pack it afterwards
 * (sdm_state_pack, B*T*H*W rows of d_v).
 */
sdm_status sdm_scan_forward_logged(const void *kp, const void *qp, const void *v,
                                   const float *alpha, const float *beta, const float *M0,
                                   float *M, int32_t init, float *y, const void *gate,
                                   const float *gamma, float eps, int32_t act, float *o,
                                   int32_t *sel_out, int32_t engine, void *ws, size_t ws_bytes,
                                   sdm_shape shape, float *wlog, void *stream);

/* Workspace bytes of sdm_state_undo for `shape` (B*H*N 32-bit entries); 0 for an invalid
 * shape. */
size_t sdm_undo_workspace_size(sdm_shape shape);

/*
 * Undoes a logged pass in place: M [B,H,N,d_v] (the state right after the pass) gets back,
 * for every slot the pass wrote, the row that the slot's first write in the pass found, i.e.
 * the state the pass started from; other rows are not touched.  sel_w: the pass's write
 * slots [B,T,H,W] int32 (the first B*T*H*W entries of its sel_out); wlog: its undo log.
 * ws: at least sdm_undo_workspace_size bytes, 256-byte aligned.  Device pointers, none
 * overlapping another; invalid arguments return SDM_ERR_INVALID_ARG before any launch; an
 * out-of-range slot sets SDM_ERR_DEVICE_CHECK (sdm_get_device_status) and is skipped.  A
 * memset and two launches, asynchronous on `stream`.  With an fp32 log of the same pass, M
 * is restored bit for bit.
 */
sdm_status sdm_state_undo(float *M, const int32_t *sel_w, const float *wlog, sdm_shape shape,
                          void *ws, size_t ws_bytes, void *stream);

/*
 * Low-precision state rows (state checkpoints) [m.163.com article on SDM, section 八, the
 * memory-efficiency paragraph: the state checkpoints of 128k fine-tuning stored as fp8 or
 * int4, with no loss in training loss or final quality].  A checkpoint row holds one row of
 * d_v fp32 state values as
 *   SDM_ROWS_BF16: d_v 16-bit codes, each value rounded to nearest-even bf16; no scale;
 *   SDM_ROWS_E4M3: d_v 8-bit OCP FP8 E4M3 codes of x / s and one fp32 scale s = amax / 448
 *                  (amax: the row's largest |x|), rounded to nearest-even and saturating at
 *                  +-448; a zero result is the code 0x00;
 *   SDM_ROWS_INT4: d_v / 2 bytes of 4-bit two's-complement codes, element 2i in the low
 *                  nibble of byte i, of x / s rounded to nearest-even and clamped to [-7, 7],
 *                  and one fp32 scale s = amax / 7.
 * s, x / s and the unpacked code * s are single fp32 operations rounded to nearest; s = 0
 * gives all-zero codes.  The live state of the pass stays fp32: these calls make and read
 * checkpoints of it (any `rows` rows of d_v values, e.g. M [B,H,N,d_v] as B*H*N rows).
 */
typedef enum { SDM_ROWS_BF16 = 1, SDM_ROWS_E4M3 = 2, SDM_ROWS_INT4 = 3 } sdm_row_format;

/* Bytes of the codes of `rows` rows of d_v values in `format`; 0 for invalid arguments
 * (rows < 0, d_v outside [4, 512] or not a multiple of 4, unknown format). */
size_t sdm_state_rows_bytes(int64_t rows, int32_t d_v, int32_t format);

/* Packs M [rows, d_v] (fp32, device) into codes (device, sdm_state_rows_bytes bytes) and, for
 * E4M3 and INT4, scales [rows] (fp32, device; ignored for BF16).  M and codes 16-byte
 * aligned, scales 4-byte aligned; none may overlap.  Invalid arguments return
 * SDM_ERR_INVALID_ARG before anything is launched; rows = 0 launches nothing.  One launch,
 * asynchronous on `stream`. */
sdm_status sdm_state_pack(const float *M, int64_t rows, int32_t d_v, int32_t format,
                          void *codes, float *scales, void *stream);

/* Unpacks codes (+ scales) made by sdm_state_pack into M [rows, d_v] (fp32): each value is
 * its code's value times the row's scale (BF16: the code widened).  Same rules as
 * sdm_state_pack. */
sdm_status sdm_state_unpack(const void *codes, const float *scales, int64_t rows, int32_t d_v,
                            int32_t format, float *M, void *stream);

/* Kinds of kernel launch reported by the timing calls below. */
typedef enum {
    SDM_KERNEL_STATE_INIT = 0, /* M0 broadcast into M                         */
    SDM_KERNEL_SELECT = 1,     /* step 1 pre-pass                             */
    SDM_KERNEL_SCAN_SEQ = 2,   /* steps 2-3, token-sequential engine          */
    SDM_KERNEL_SCAN_SLOT = 3,  /* steps 2-3, slot-parallel engine             */
    SDM_KERNEL_NORM_GATE = 4,  /* step 4                                      */
    SDM_KERNEL_DECODE = 5,     /* fused decode step                           */
    SDM_KERNEL_SLOT_SORT = 6,  /* slot engine: event build and radix sort      */
    SDM_KERNEL_STATE_ROWS = 7, /* state checkpoint pack / unpack              */
    SDM_KERNEL_UNDO = 8,       /* undo of a logged pass                       */
    SDM_KERNEL_SCAN_CHUNK = 9, /* steps 2-3, chunk-wise engine                */
    SDM_KERNEL_KINDS = 16
} sdm_kernel_kind;

/* Kernel timing.  While enabled (on != 0), every kernel launch the library makes is
 * bracketed by two CUDA events recorded on the launch's stream (a few microseconds of
 * host time per launch, nothing on the device).  Enabling or disabling drops what was
 * recorded.  Do not enable it while a stream is being captured into a CUDA graph. */
sdm_status sdm_profile_enable(int32_t on);

/* Waits for the launches recorded since the last enable/read and returns, per
 * sdm_kernel_kind, the summed device time in milliseconds (ms[SDM_KERNEL_KINDS]) and the
 * number of launches (launches[SDM_KERNEL_KINDS]); then forgets them. */
sdm_status sdm_profile_read(double *ms, int64_t *launches);

/* Process-wide launch options, for testing and tuning; every option defaults to 0, which
 * is what normal use wants.  The library reads no environment variable: these calls are
 * the only switches.  A value applies to the calls made after it is set, on every device
 * and stream of the process; set options before any stream capture and not while another
 * host thread is calling the library. */
typedef enum {
    SDM_OPT_NO_PDL = 1,             /* 1: every kernel in plain stream order, including
                                       sdm_decode_step_chained                          */
    SDM_OPT_SELECT_GENERAL = 2,     /* 1: bf16 rows also take the general selection path
                                       (same results; compares the two paths)           */
    SDM_OPT_SELECT_CTAS_PER_SM = 3, /* n > 0: at most n selection CTAs per SM           */
    SDM_OPT_SLOT_CTAS_PER_SM = 4,   /* n > 0: at most n slot-engine scan CTAs per SM     */
    SDM_OPT_SEQ_COLUMNS = 5,        /* 4, 8, 16 or 32: the sequential engine's column
                                       slice (0: chosen by shape)                       */
    SDM_OPT_SEQ_DEPTH = 6,          /* 4 or 8: the sequential engine's gather-ahead
                                       depth in tokens (0: chosen by slice)             */
    SDM_OPT_SLOT_CTA_STATS = 7,     /* 1: the slot engine records per-CTA work
                                       (sdm_slot_cta_stats)                             */
    SDM_OPT_SELECT_SCHEDULE = 8     /* the slot engine's selection, when T spans more
                                       than one time chunk: 1 the whole selection first,
                                       2 pipelined (chunk c + 1's selection on an
                                       internal low-priority stream beside chunk c's
                                       work on an internal high-priority one, joined
                                       back to the caller's stream), 0 the library's
                                       default; every schedule gives the same
                                       selections and state.  The internal streams are
                                       per device and shared by the process: pipelined
                                       calls from several host threads are enqueued one
                                       at a time and run one after another.             */
} sdm_option;

/* Sets an option.  SDM_ERR_INVALID_ARG (and no change) for an unknown option or a value
 * outside the ranges above. */
sdm_status sdm_set_option(int32_t option, int32_t value);

/* The option's current value, or -1 for an unknown option. */
int32_t sdm_get_option(int32_t option);

/* Load balance of the slot engine.  While SDM_OPT_SLOT_CTA_STATS is 1, every launch of the
 * engine's chunk kernel adds, for each of its CTAs (by block index, the first
 * SDM_SLOT_STATS_CTAS of them), four counters to a table the library holds on each device:
 * [0] events applied from short segments, [1] events of the long (hot-slot) segments it
 * took, [2] spans of sorted events it took from the work queue, [3] the summed busy
 * nanoseconds of its warps.  sdm_slot_cta_stats waits for the calling device to finish its
 * work, copies the first max_ctas rows of that device's table to out[max_ctas][4] (host
 * memory) and, when reset != 0, clears the table.  The counters use the device's global
 * timer; nothing else changes with the option. */
#define SDM_SLOT_STATS_CTAS 1024
sdm_status sdm_slot_cta_stats(uint64_t *out, int32_t max_ctas, int32_t reset);

/* Number of kernels this library has launched in this process, on every device. */
uint64_t sdm_launch_count(void);

/* Synchronises `stream`, then reads and clears the calling device's status word:
 * SDM_OK, SDM_ERR_DEVICE_CHECK (an index outside [0, N) reached a kernel) or
 * SDM_ERR_TIMEOUT (a bounded wait expired).  SDM_ERR_CUDA if the synchronisation fails. */
sdm_status sdm_get_device_status(void *stream);

/* Static, human-readable name of a status code. */
const char *sdm_status_string(sdm_status status);

#ifdef __cplusplus
}
#endif

#endif /* SDM_H */
