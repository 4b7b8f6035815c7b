/*
 * gdn.h -- C ABI of the Gated DeltaNet core for NVIDIA B200 (sm_100a).
 *
 * The library computes the gated delta rule in two modes, chunked prefill and
 * a one-token recurrent decode step, plus the gate computation that feeds both.
 *
 *   Gates ("Gated DeltaNet ... Qwen3-next" page, section 2.1, gate code):
 *       beta = sigmoid(b),  g = -exp(A_log) * softplus(a + dt_bias),  alpha = exp(g)
 *   Rule ("Gated DeltaNet and reasoning scaffolds" research log, third update rule):
 *       S_t = S_{t-1} (alpha_t (I - beta_t k_t k_t^T)) + beta_t v_t k_t^T,  o_t = scale * S_t q_t
 *
 * State orientation.  S_t is Dv x Dk (S k ~ v).  The library stores its
 * transpose H = S^T, shape [.., Dk, Dv] row-major (the "k delta^T" form of the
 * "QWEN3.5" Q&A page, question 2), always in fp32: one 128 x 128 head is 64 KB.
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE memory, allocated, owned and freed by the
 *     caller.  The library never allocates, frees or synchronises, except in
 *     gdn_chunk_prefill_status(), which synchronises the given stream.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Arguments are validated on the host before anything is
 *     launched; a non-GDN_OK return means nothing was launched.
 *   - Tensors are contiguous, token-major:  q, k [.., HK, Dk];  v, o [.., HV, Dv];
 *     g, beta [.., HV].  Value head h reads q/k head h / (HV / HK).
 *   - Pointers must be 16-byte aligned.  Outputs must not overlap any input or
 *     each other (checked by address range).
 *   - Supported sizes: Dk, Dv in {64, 128}; HV % HK == 0.
 *   - io dtype GDN_BF16: q, k, v, o are bf16 and all arithmetic on them is fp32
 *     accumulation with bf16 tensor-core operands; GDN_F32: everything fp32 on
 *     CUDA cores (no TF32).
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_ABI_VERSION 1

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_NULL = 1,        /* a required pointer is NULL                                  */
    GDN_ERR_SHAPE = 2,       /* a size is negative, zero where it must not be, or inconsistent */
    GDN_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                            */
    GDN_ERR_UNSUPPORTED = 4, /* valid but not implemented (head dim, chunk size, dtype)     */
    GDN_ERR_ALIAS = 5,       /* an output overlaps an input or another output               */
    GDN_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than the size query returned      */
    GDN_ERR_CUDA = 7,        /* a CUDA call or launch failed                                */
    GDN_ERR_DEVICE = 8       /* a device-side check failed (reported by a status query)     */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Device-side error codes written into the prefill workspace's status word. */
#define GDN_DEVERR_NONE 0
#define GDN_DEVERR_CU_SEQLENS 1   /* cu_seqlens[0] != 0, decreasing, or last != T */
#define GDN_DEVERR_TIMEOUT 2      /* a bounded wait inside a kernel expired; outputs invalid */

/* Human-readable name of a gdn_status value (static storage, never NULL). */
GDN_API const char* gdn_status_string(int status);

/* GDN_ABI_VERSION of the loaded library. */
GDN_API int gdn_abi_version(void);

/* Number of kernels this library has launched in this process (all devices,
 * all threads), counted at each successful launch.  For accounting only. */
GDN_API uint64_t gdn_kernel_launches(void);

/* Last CUDA error code (cudaError_t as int) seen by a call that returned
 * GDN_ERR_CUDA on this host thread; 0 if none. */
GDN_API int gdn_last_cuda_error(void);

/*
 * gdn_gates -- the gate formula ("Gated DeltaNet ... Qwen3-next" page, section 2.1).
 *   a, b      [n_tokens, HV]  fp32 or bf16 (ab_dtype)       (read)
 *   A_log     [HV] fp32,  dt_bias [HV] fp32                  (read)
 *   g, beta   [n_tokens, HV] fp32                            (written)
 *   g = -exp(A_log[h]) * softplus(a[t,h] + dt_bias[h]);  beta = 1 / (1 + exp(-b[t,h])).
 * n_tokens may be 0 (nothing launched).  Errors: NULL, SHAPE (HV <= 0 or
 * n_tokens < 0), ALIGN, ALIAS (g/beta overlapping inputs or each other), CUDA.
 */
GDN_API gdn_status gdn_gates(const void* a, const void* b, gdn_dtype ab_dtype,
                     const float* A_log, const float* dt_bias,
                     int64_t n_tokens, int32_t HV,
                     float* g, float* beta, void* stream);

/*
 * Workspace size in bytes that gdn_chunk_prefill needs for these sizes (always
 * >= 256: the first 256 bytes hold the device status word).  Returns 0 for
 * sizes that gdn_chunk_prefill would reject, including totals past the 32-bit
 * coordinates of the tile copies (over 2^31 - 1 tokens, or chunks x heads x 64 rows).
 */
GDN_API size_t gdn_chunk_prefill_workspace_bytes(int64_t n_tokens, int32_t n_seqs,
                                         int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                                         int32_t BT, gdn_dtype io_dtype);

/*
 * gdn_chunk_prefill -- the rule over whole sequences, computed chunk by chunk
 * ("QWEN3.5" Q&A page, question 1: chunks of BT tokens, parallel inside a chunk,
 * state carried serially across chunks; the call shape is the
 * chunk_gated_delta_rule(query, key, value, g, beta, initial_state) ->
 * (out, last_state) call of the "Gated DeltaNet ... Qwen3-next" page, section 3.1).
 *
 *   Dense layout (cu_seqlens == NULL): B sequences of T tokens each; n_seqs must
 *   equal B.  Packed layout (cu_seqlens != NULL): B must be 1, T is the total
 *   token count, and sequence n is tokens cu_seqlens[n] .. cu_seqlens[n+1]-1.
 *
 *   q, k          [B, T, HK, Dk]   io_dtype                  (read)
 *   v             [B, T, HV, Dv]   io_dtype                  (read)
 *   g, beta       [B, T, HV]       fp32 log-decay and write strength (read)
 *   initial_state [n_seqs, HV, Dk, Dv] fp32, or NULL for zero states (read)
 *   cu_seqlens    [n_seqs + 1] int32 device, or NULL          (read)
 *   o             [B, T, HV, Dv]   io_dtype                  (written)
 *   final_state   [n_seqs, HV, Dk, Dv] fp32, or NULL          (written; may
 *                 equal initial_state exactly for an in-place update, no other
 *                 overlap allowed)
 *   workspace     device scratch of >= gdn_chunk_prefill_workspace_bytes(...) bytes,
 *                 owned by the caller, contents need not be initialised; it must
 *                 not be shared by calls that may run concurrently.
 *   BT            chunk length: 16, 32 or 64.  BT only changes rounding, never the
 *                 result's definition.
 *                 GDN_BF16 with Dk = Dv = 128, HV / HK in {1, 2, 4} and BT = 64 runs on
 *                 the tensor cores (tcgen05); every other configuration runs on CUDA cores.
 *   scale         multiplies o (1.0 = the plain rule).
 *   qk_l2norm     nonzero: q and k rows are replaced by x / sqrt(sum x^2 + 1e-6)
 *                 before use (per token and q/k head).
 *
 * cu_seqlens is checked on the device (first entry 0, non-decreasing, last
 * entry T).  A bad table makes every kernel of the call exit without writing o
 * or final_state and leaves GDN_DEVERR_CU_SEQLENS in the workspace status word;
 * read it with gdn_chunk_prefill_status().  Zero-length sequences are allowed
 * (their final state equals the initial state).
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED, ALIAS, WORKSPACE, CUDA.
 */
GDN_API gdn_status gdn_chunk_prefill(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                             const float* g, const float* beta,
                             const float* initial_state, const int32_t* cu_seqlens,
                             int32_t B, int64_t T, int32_t n_seqs,
                             int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                             int32_t BT, float scale, int32_t qk_l2norm,
                             void* o, float* final_state,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * gdn_chunk_prefill_gated -- gdn_chunk_prefill with the gate prologue fused in: instead of
 * g and beta it takes the gate inputs and forms
 *     g = -exp(A_log[h]) * softplus(a + dt_bias[h]),   beta = sigmoid(b)
 * (the gate code of the "Gated DeltaNet ... Qwen3-next" page, section 2.1) per (token,
 * value head) inside the chunk-local kernel, with the same arithmetic as gdn_gates, so the
 * results are bit-identical to gdn_gates followed by gdn_chunk_prefill; g and beta are never
 * written to memory.
 *   a, b          [B, T, HV] (packed: [T, HV]), ab_dtype fp32 or bf16     (read)
 *   A_log, dt_bias [HV] fp32                                             (read)
 *   everything else as gdn_chunk_prefill, same workspace size.
 * The tensor-core shapes only (bf16, Dk = Dv = 128, BT = 64, HV / HK in {1, 2, 4});
 * others return UNSUPPORTED (use gdn_gates and gdn_chunk_prefill).
 * Errors: those of gdn_chunk_prefill; ALIAS also for outputs over a, b, A_log, dt_bias.
 */
GDN_API gdn_status gdn_chunk_prefill_gated(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                             const void* a, const void* b, gdn_dtype ab_dtype,
                             const float* A_log, const float* dt_bias,
                             const float* initial_state, const int32_t* cu_seqlens,
                             int32_t B, int64_t T, int32_t n_seqs,
                             int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                             int32_t BT, float scale, int32_t qk_l2norm,
                             void* o, float* final_state,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * gdn_chunk_prefill_outgate -- gdn_chunk_prefill with the output epilogue fused into the
 * output store: each output row of a value head (Dv values) becomes
 *     o * rsqrt(mean(o^2) + eps) * (1 + norm_w) * sigmoid(z)
 * the zero-centred RMSNorm of the Qwen3-next page (section 3.2: weight initialised to
 * zero) and the sigmoid output gate of the GDN resource-allocation page (applied after the
 * attention output, before the residual add).
 *   z       [B, T, HV, Dv] (or [T_total, HV, Dv] packed) io_dtype, the gate inputs  (read)
 *   norm_w  [Dv] fp32, shared by the value heads                                    (read)
 *   eps     >= 0 (the workloads' reading: 1e-6)
 * Other arguments as gdn_chunk_prefill, whose workspace size applies.  Only the
 * tensor-core configuration (bf16, Dk = Dv = 128, BT = 64, HV / HK in {1, 2, 4}); others
 * return UNSUPPORTED.  Errors: those of gdn_chunk_prefill, NULL (z or norm_w), SHAPE
 * (eps < 0 or NaN), ALIAS (o, final_state or workspace over z or norm_w).
 */
GDN_API gdn_status gdn_chunk_prefill_outgate(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                             const float* g, const float* beta,
                             const float* initial_state, const int32_t* cu_seqlens,
                             int32_t B, int64_t T, int32_t n_seqs,
                             int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                             int32_t BT, float scale, int32_t qk_l2norm,
                             const void* z, const float* norm_w, float eps,
                             void* o, float* final_state,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * gdn_conv_prefill -- the prefill prologue: the causal depthwise convolution of kernel 4
 * that the "Gated DeltaNet ... Qwen3-next" page (section 3.1) places before the gated
 * update (kernel size from the tutorial page, section 6, linear_conv_kernel_dim = 4),
 * over whole sequences, from the raw q | k | v projections to the q, k, v inputs of
 * gdn_chunk_prefill, with the rolling state of each sequence carried in and out:
 *   y_t = w0 x_{t-3} + w1 x_{t-2} + w2 x_{t-1} + w3 x_t per channel, then identity or SiLU.
 * Sequences as gdn_chunk_prefill: dense (cu_seqlens == NULL, B sequences of T tokens,
 * n_seqs == B) or packed (B == 1, T total tokens, n_seqs sequences in cu_seqlens).
 *   x      [B, T, C] io_dtype, C = 2 HK Dk + HV Dv: q channels (head-major), then k, then v
 *                                                                              (read)
 *   conv_w [C, 4] fp32, taps oldest first                                      (read)
 *   conv_state_in  [n_seqs, 3, C] fp32, the three inputs before each sequence, oldest
 *          first, or NULL for zeros                                            (read)
 *   conv_act  0: y;  1: SiLU, y / (1 + exp(-y))   (the pages name no activation)
 *   q, k   [B, T, HK, Dk] io_dtype;  v [B, T, HV, Dv] io_dtype: y rounded to io_dtype
 *                                                                              (written)
 *   conv_state_out [n_seqs, 3, C] fp32, each sequence's three newest inputs (with the
 *          carried state for sequences shorter than 3; a zero-length sequence passes its
 *          state through), or NULL (written).  It is the conv_state_in of the next
 *          prefill piece or of gdn_decode_step_fused.
 * No output may overlap an input or another output (conv_state_out may not be
 * conv_state_in).  cu_seqlens is not checked here (gdn_chunk_prefill checks the same
 * table on the device); with a bad table the outputs are undefined, but every access
 * stays inside the buffers the sizes describe.
 * For bf16 the convolution runs as a persistent kernel fed by tile copies, whose waits are
 * bounded; if one expires (no such case is known) the launch stops early and records
 * GDN_DEVERR_TIMEOUT, which gdn_conv_status reports.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED (Dk, Dv not 64 or 128), ALIAS, CUDA.
 */
GDN_API gdn_status gdn_conv_prefill(const void* x, gdn_dtype io_dtype, const float* conv_w,
                                    const float* conv_state_in, const int32_t* cu_seqlens,
                                    int32_t B, int64_t T, int32_t n_seqs,
                                    int32_t HK, int32_t HV, int32_t Dk, int32_t Dv, int32_t conv_act,
                                    void* q, void* k, void* v, float* conv_state_out, void* stream);

/*
 * Synchronises the device, then reads and clears the device word of the convolution kernel
 * (GDN_DEVERR_NONE or GDN_DEVERR_TIMEOUT, shared by every gdn_conv_prefill launch on that
 * device) into *device_error.  Returns GDN_ERR_DEVICE if it is nonzero.
 * Errors: NULL, CUDA.
 */
GDN_API gdn_status gdn_conv_status(int32_t* device_error);

/*
 * gdn_cp_segment -- one rank's work on its segment in a context-parallel prefill (see
 * gdn_cp_combine): the segment's gdn_chunk_prefill (o, final_state, from initial_state or
 * zero) and, on the same chunk-local stage, its transition run (v = 0 from the identity):
 *   c          [B, T, HV, Dv] io_dtype: c_t = scale A_{<=t}^T q_t                   (written)
 *   transition [n_seqs, HV, Dk, Dk] fp32: A, the product of the segment's transitions
 *                                                                                   (written)
 * The other arguments and the errors are those of gdn_chunk_prefill; only the tensor-core
 * configuration (bf16, Dk = Dv = 128, BT = 64, HV / HK in {1, 2, 4}) is supported (others:
 * UNSUPPORTED; two gdn_chunk_prefill calls give the same results).  c and transition may
 * not overlap any other buffer.
 */
GDN_API gdn_status gdn_cp_segment(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                                  const float* g, const float* beta, const float* initial_state,
                                  const int32_t* cu_seqlens, int32_t B, int64_t T, int32_t n_seqs,
                                  int32_t HK, int32_t HV, int32_t Dk, int32_t Dv, int32_t BT, float scale,
                                  int32_t qk_l2norm, void* o, float* final_state, void* c,
                                  float* transition, void* workspace, size_t workspace_bytes, void* stream);

/*
 * gdn_cp_combine -- the exchange step of a context-parallel prefill, in which each of R
 * ranks holds one consecutive segment of the same sequences (rank r the r-th segment of
 * T_seg tokens).  Over a segment the rule is affine in the state it starts from (the
 * product form of the update, "Gated DeltaNet" research log; H = S^T):
 *     H_end = A H_start + B,   o_t = o0_t + H_start^T c_t,
 * B and o0 being the segment's gdn_chunk_prefill from a zero state, A and c its
 * gdn_chunk_prefill with v = 0 from H_start = I (A = the product of the segment's
 * transitions, c_t = scale A_{<=t}^T q_t).  With every rank's (A, B) gathered, this call
 * forms H_start(rank) by the scan H_start(0) = initial_state, H_start(r + 1) = A_r
 * H_start(r) + B_r, the sequences' final states, and corrects o in place.
 *   A_all, B_all  [R, n_seqs, HV, 128, 128] fp32, rank-major                     (read)
 *   initial_state [n_seqs, HV, 128, 128] fp32, the state before segment 0, or NULL (read)
 *   o             [n_seqs, T_seg, HV, 128] io_dtype: o0 in, the rank's outputs out
 *   c             [n_seqs, T_seg, HV, 128] io_dtype                              (read)
 *   start_state   [n_seqs, HV, 128, 128] fp32, H_start of this rank's segment   (written)
 *   final_state   [n_seqs, HV, 128, 128] fp32, the state after segment R - 1, or NULL
 * Dk = Dv = 128 only; up to 65535 x 128 tokens per segment (fp32) or 2^31 - 129 tokens over
 * all sequences (bf16).  No output may overlap an input or another output.  For bf16 the
 * correction runs on the tensor cores (H_start rounded to bf16 for the product) with
 * bounded waits; a wait that expires (no such case is known) records GDN_DEVERR_TIMEOUT,
 * which gdn_cp_status reports.
 * Errors: NULL, SHAPE (R, rank, sizes), ALIGN, UNSUPPORTED, ALIAS, CUDA.
 */
GDN_API gdn_status gdn_cp_combine(const float* A_all, const float* B_all, const float* initial_state,
                                  int32_t R, int32_t rank, int32_t n_seqs, int64_t T_seg, int32_t HV,
                                  int32_t Dk, int32_t Dv, gdn_dtype io_dtype, void* o, const void* c,
                                  float* start_state, float* final_state, void* stream);

/*
 * Synchronises the device, then reads and clears the device word of gdn_cp_combine's
 * tensor-core correction (GDN_DEVERR_NONE or GDN_DEVERR_TIMEOUT) into *device_error.
 * Returns GDN_ERR_DEVICE if it is nonzero.  Errors: NULL, CUDA.
 */
GDN_API gdn_status gdn_cp_status(int32_t* device_error);

/*
 * Synchronises `stream`, then reads the device status word of a prefill
 * workspace into *device_error (GDN_DEVERR_*).  Returns GDN_ERR_DEVICE if it
 * is nonzero, GDN_ERR_CUDA if the synchronisation failed, else GDN_OK.
 */
GDN_API gdn_status gdn_chunk_prefill_status(const void* workspace, void* stream, int32_t* device_error);

/*
 * gdn_chunk_prefill_static_ws -- gdn_chunk_prefill without a caller-provided workspace.
 * The pages describe no such call: it exists for callers whose host code may not
 * allocate device memory (a serving loop under a no-allocation rule, where an
 * allocation can synchronise the device; code called back from a framework that owns
 * the device memory and offers no allocator).  Arguments, layouts and results are those
 * of gdn_chunk_prefill minus workspace / workspace_bytes; nothing is allocated or freed.
 *
 * The scratch is one file-scope device array of GDN_STATIC_SCRATCH_BYTES inside the
 * library, present on every GPU that loads the library until the process exits.
 *   - Sizes whose gdn_chunk_prefill_workspace_bytes(...) exceeds GDN_STATIC_SCRATCH_BYTES
 *     are rejected with GDN_ERR_WORKSPACE before anything is launched (for bf16, 128-dim
 *     heads that is about 2K tokens at 32 value heads).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it.  Under CUDA's lazy module loading (the
 *     default since CUDA 12.2) that lookup is also what loads the library's device code
 *     and with it the GDN_STATIC_SCRATCH_BYTES array: a device allocation that can
 *     synchronise the device.  Make the first call on each device during set-up, before
 *     the code that must not allocate runs and before any stream capture on that device.
 *   - Every call on a device shares the one array, and it keeps the previous call's
 *     contents; each call rewrites all of it that it reads, so nothing needs clearing.
 *     Calls whose executions overlap on the GPU (other streams, other host threads)
 *     race on the array and give wrong results: serialise them.
 *   - The device status word lives in the array, so a bad cu_seqlens table (outputs left
 *     unwritten) cannot be read back through this call; validate the table beforehand.
 * Errors: those of gdn_chunk_prefill, GDN_ERR_WORKSPACE for sizes over the cap, and
 * GDN_ERR_CUDA if the array's address cannot be obtained.
 */
#define GDN_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)
GDN_API gdn_status gdn_chunk_prefill_static_ws(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                             const float* g, const float* beta,
                             const float* initial_state, const int32_t* cu_seqlens,
                             int32_t B, int64_t T, int32_t n_seqs,
                             int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                             int32_t BT, float scale, int32_t qk_l2norm,
                             void* o, float* final_state, void* stream);

/*
 * gdn_chunk_prefill_host -- gdn_gates followed by gdn_chunk_prefill for inputs and outputs
 * that live in HOST memory (on the tensor-core shapes, gdn_chunk_prefill_gated: the gates
 * formed inside the prefill, bit for bit the same).  The sequences are streamed through the GPU in pieces of
 * `piece_tokens` tokens (a multiple of BT): the host -> device copies of one piece, the
 * kernels of the previous piece and the device -> host copies of the one before overlap
 * on three library-owned streams with two buffer slots each way, and the state is carried
 * between pieces in place on the device.  The pages have no counterpart of this call; it
 * is the runtime around the chunked form of the "QWEN3.5" Q&A page, question 1 (chunks in
 * order, the state carried serially), for callers whose data arrives from the host.
 *   q, k   [B, T, HK, Dk] io_dtype;  v [B, T, HV, Dv] io_dtype      (host, read)
 *   a, b   [B, T, HV] ab_dtype;  A_log, dt_bias [HV] fp32            (host, read)
 *   initial_state [B, HV, Dk, Dv] fp32 or NULL (zeros)              (host, read)
 *   o      [B, T, HV, Dv] io_dtype                                  (host, written)
 *   final_state [B, HV, Dk, Dv] fp32 or NULL                        (host, written)
 *   workspace   device, 256-byte aligned, gdn_chunk_prefill_host_workspace_bytes() bytes
 * Dense sequences only (no cu_seqlens).  Results equal gdn_chunk_prefill's up to the
 * rounding of the fp16 intermediates, whose power-of-two scale is chosen per piece.
 * Asynchronous: returns once the work is enqueued; `stream` waits for all of it, so the
 * host buffers must stay valid until `stream` reaches that point, and page-locked host
 * memory is needed for the copies to overlap.  The internal streams and events are
 * created on the first call on a device and kept for the life of the process; calls on
 * one device are serialised.  Not for use inside a CUDA graph capture.
 * Errors: NULL, SHAPE (piece_tokens <= 0 or not a multiple of BT), UNSUPPORTED, ALIGN
 * (workspace), WORKSPACE, CUDA, or any error of the two calls it makes.
 */
GDN_API size_t gdn_chunk_prefill_host_workspace_bytes(int32_t B, int64_t T, int32_t HK, int32_t HV,
                             int32_t Dk, int32_t Dv, int32_t BT, gdn_dtype io_dtype, gdn_dtype ab_dtype,
                             int64_t piece_tokens);
GDN_API gdn_status gdn_chunk_prefill_host(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                             const void* a, const void* b, gdn_dtype ab_dtype,
                             const float* A_log, const float* dt_bias, const float* initial_state,
                             int32_t B, int64_t T, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                             int32_t BT, float scale, int32_t qk_l2norm, int64_t piece_tokens,
                             void* o, float* final_state, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * gdn_decode_step -- one token per sequence, state updated in place (the
 * incremental update of the "QWEN3.5" Q&A page, question 2a: decay the whole
 * state by alpha, then clear and write along the current key with strength beta).
 *   q, k   [B, HK, Dk] io_dtype;  v [B, HV, Dv] io_dtype;  g, beta [B, HV] fp32  (read)
 *   state  [B, HV, Dk, Dv] fp32                            (read and written in place)
 *   o      [B, HV, Dv] io_dtype                            (written; o = scale * S_t q_t
 *                                                           with the updated state)
 * B may be 0 (nothing launched).
 * For Dk = Dv = 128 the step runs as a persistent kernel whose waits are bounded; if one
 * expires (no such case is known) the launch stops early and records
 * GDN_DEVERR_TIMEOUT, which gdn_decode_status reports.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED, ALIAS, CUDA.
 */
GDN_API gdn_status gdn_decode_step(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                           const float* g, const float* beta, float* state,
                           int32_t B, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                           float scale, int32_t qk_l2norm, void* o, void* stream);

/*
 * gdn_decode_step_gated -- the same step with the gate prologue fused in: g and beta are
 * formed inside the kernel from the raw gate inputs with the formula of gdn_gates
 * ("Gated DeltaNet ... Qwen3-next" page, section 2.1), bit for bit as gdn_gates would
 * write them, instead of being read from memory.  Saves the separate gates launch and its
 * round trip through HBM on every decode step.
 *   a, b     [B, HV] ab_dtype (fp32 or bf16)                 (read)
 *   A_log, dt_bias [HV] fp32                                  (read)
 *   other arguments as gdn_decode_step.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED, ALIAS (state or o over any input), CUDA.
 */
GDN_API gdn_status gdn_decode_step_gated(const void* q, const void* k, const void* v, gdn_dtype io_dtype,
                           const void* a, const void* b, gdn_dtype ab_dtype,
                           const float* A_log, const float* dt_bias, float* state,
                           int32_t B, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                           float scale, int32_t qk_l2norm, void* o, void* stream);

/*
 * gdn_decode_step_fused -- the whole decode step from raw projections in one kernel:
 * the causal depthwise convolution of kernel 4 that the Qwen3-next page (section 3.1)
 * places before the gated update (kernel size from the tutorial page, section 6,
 * linear_conv_kernel_dim = 4), the q/k L2 norm, the gates and the state update.
 *   x      [B, C] io_dtype, C = 2 HK Dk + HV Dv: per sequence the raw q | k | v
 *          projections of the current token, q/k head-major then v head-major  (read)
 *   conv_w [C, 4] fp32, taps oldest first: y = w0 x_{t-3} + w1 x_{t-2} + w2 x_{t-1} + w3 x_t
 *   conv_state_in  [B, 3, C] fp32, the three previous inputs, oldest first      (read)
 *   conv_state_out [B, 3, C] fp32, the three newest inputs after this token     (written;
 *          must not overlap conv_state_in: value heads that share a q/k head read the
 *          old q/k channels while another writes the new ones)
 *   conv_act  0: q, k, v = y;  1: SiLU, y * sigmoid(y)  (the pages name no activation)
 *   a, b, A_log, dt_bias, state, o and the rest as gdn_decode_step_gated.
 * Dk = Dv = 128 only (others: UNSUPPORTED).  q, k, v are kept in fp32 after the
 * convolution (no rounding to io_dtype).
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED, ALIAS (any output over any input or another
 * output), CUDA.
 */
GDN_API gdn_status gdn_decode_step_fused(const void* x, gdn_dtype io_dtype,
                           const float* conv_w, const float* conv_state_in, float* conv_state_out,
                           int32_t conv_act, const void* a, const void* b, gdn_dtype ab_dtype,
                           const float* A_log, const float* dt_bias, float* state,
                           int32_t B, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                           float scale, int32_t qk_l2norm, void* o, void* stream);

/*
 * gdn_decode_step_fused_outgate -- gdn_decode_step_fused with the output epilogue applied to
 * each output row before the store:
 *     out = o * rsqrt(mean(o^2) + eps) * (1 + norm_w) * sigmoid(z)
 * per (sequence, value head) over its Dv values: the zero-centred RMSNorm of the
 * "Gated DeltaNet ... Qwen3-next" page (section 3.2: a norm weight initialised to zero, so
 * stored as w with the scale 1 + w) and the sigmoid output gate of the GDN resource-
 * allocation page; the same epilogue as gdn_chunk_prefill_outgate, so a sequence prefilled
 * with that call continues here.  sigmoid is formed from the hardware tanh (absolute error
 * below 2^-12).
 *   z        [B, HV, Dv] io_dtype                                   (read)
 *   norm_w   [Dv] fp32, eps >= 0                                    (read)
 *   everything else as gdn_decode_step_fused (Dk = Dv = 128).
 * Errors: those of gdn_decode_step_fused; NULL for z or norm_w NULL, SHAPE for eps < 0 or
 * NaN, ALIGN, ALIAS also for the outputs over z or norm_w.
 */
GDN_API gdn_status gdn_decode_step_fused_outgate(const void* x, gdn_dtype io_dtype,
                           const float* conv_w, const float* conv_state_in, float* conv_state_out,
                           int32_t conv_act, const void* a, const void* b, gdn_dtype ab_dtype,
                           const float* A_log, const float* dt_bias, float* state,
                           int32_t B, int32_t HK, int32_t HV, int32_t Dk, int32_t Dv,
                           float scale, int32_t qk_l2norm, const void* z, const float* norm_w,
                           float eps, void* o, void* stream);

/*
 * gdn_decode_status -- synchronises the current device and writes its decode error
 * word (GDN_DEVERR_NONE or GDN_DEVERR_TIMEOUT, shared by every decode launch on that
 * device) into *device_error, then clears it.  This is library bookkeeping with no
 * counterpart in the method.  Returns OK if the word was 0, DEVICE if not, NULL for a
 * NULL argument, CUDA on a CUDA error.
 */
GDN_API gdn_status gdn_decode_status(int32_t* device_error);

/*
 * gdn_testing_stall -- a test hook with no counterpart in the method: it lets a test see
 * a kernel's bounded wait run out without any fault.  With a site other than
 * GDN_STALL_NONE, later launches of that kernel (from any host thread, on any device)
 * withhold the copies of one work item of their first CTA, so that the CTA's wait for
 * them ends at the wait limit (2 s): the kernel records GDN_DEVERR_TIMEOUT, lets what it
 * did issue land, frees its tensor memory and returns; the outputs of that call are
 * invalid.  Sites:
 *   GDN_STALL_DECODE        the staged decode kernel (Dk = Dv = 128: gdn_decode_step,
 *                           _gated, _fused): the first item's state and rows; reported
 *                           by gdn_decode_status
 *   GDN_STALL_PREFILL_PREP  the chunk-local stage of the tensor-core prefill: the first
 *                           chunk's V tile; reported by gdn_chunk_prefill_status (the
 *                           state-carry launch of that call then does nothing)
 * GDN_STALL_NONE restores normal operation.  Not for production use.  Errors: SHAPE for
 * an unknown site.
 */
#define GDN_STALL_NONE 0
#define GDN_STALL_DECODE 1
#define GDN_STALL_PREFILL_PREP 2
GDN_API gdn_status gdn_testing_stall(int32_t site);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
