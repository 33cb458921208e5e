/*
 * gdr.h - C ABI of libgdr: the gated delta rule token mixers (GDN and KDA) on
 * NVIDIA B200 (sm_100a).
 *
 * The operation.  "Super Apriel: One Checkpoint, Many Speeds", §2A (Mixer
 * Vocabulary) names two recurrent mixers: Gated DeltaNet (GDN), the delta rule
 * with a scalar gate, and Kimi Delta Attention (KDA), the delta rule with a
 * channel-wise gate; §1 and §4 (context-length scaling) rest on their state
 * having a fixed size.  For every (sequence, head) the state S is a d_v x d_k
 * fp32 matrix and each token t applies
 *
 *     S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t
 *
 * with alpha_t one scalar per (token, head) for GDN and one value per key
 * channel (a d_k-vector) for KDA.  No scaling is applied to q; callers that want
 * 1/sqrt(d_k) or L2-normalised q/k apply it before the call.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, dense
 *     (row-major, no strides), and 16-byte aligned.  The library never frees or
 *     retains them after the call returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  A GDR_OK return means the arguments
 *     were accepted and the kernels were enqueued; device-side problems surface
 *     at the caller's next synchronisation (or through gdr_workspace_status).
 *   - Nothing throws across the ABI.  On a non-OK status nothing was enqueued,
 *     and gdr_last_error() returns a message for the calling thread.
 *   - alpha is taken as the gate itself, in [0, 1]; the kernels work with
 *     max(log(alpha), -GDR_LOG_GATE_FLOOR), so a gate below e^-30 acts as e^-30
 *     (a factor below 1e-13 on what the state carried).  Values are not checked
 *     on the device.
 *   - Supported head sizes: d_k, d_v in {32, 64, 128}.  The chunk length of the
 *     prefill is 64 tokens; the last chunk of a sequence may be shorter.
 *   - The library is thread-safe for calls on different streams; calls that
 *     share a workspace must not overlap on the device.
 *
 * Environment variables, read at every call (neither is needed in normal use)
 *   GDR_SPIN_LIMIT  polls of every bounded device-side wait before it gives up
 *                   and records GDR_ERR_TIMEOUT (default 2^24; 0 gives up
 *                   without polling, which tests use to reach that path; the
 *                   work in flight still completes and is drained).
 *   GDR_CARRY       state carry of the two-kernel prefill: unset (or any other
 *                   value) = the chained carry; "rows" = one CTA per (sequence,
 *                   head) with the output products off its chain; "sliced" = the
 *                   value rows of each head split over several CTAs.  All three
 *                   give results within the same tolerance; they differ in speed.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdr_status {
  GDR_OK = 0,
  GDR_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad enum    */
  GDR_ERR_UNSUPPORTED = 2,   /* valid request this build has no kernel for     */
  GDR_ERR_CUDA = 3,          /* a CUDA runtime call failed (message says which) */
  GDR_ERR_TIMEOUT = 4        /* a bounded device-side wait gave up             */
} gdr_status;

typedef enum gdr_dtype {
  GDR_F32 = 0,               /* IEEE fp32                                      */
  GDR_BF16 = 1               /* bfloat16                                       */
} gdr_dtype;

#if defined(__GNUC__)
#define GDR_API __attribute__((visibility("default")))
#else
#define GDR_API
#endif

#define GDR_CHUNK 64
#define GDR_LOG_GATE_FLOOR 30.0f

/* Fused prologue flags of the *_ex entry points (0 = the plain entry points):
 *   GDR_PROLOGUE_L2NORM_QK  q and k arrive raw; each (token, head) vector is divided
 *                           by sqrt(sum of its squares + GDR_L2NORM_EPS) in fp32, and
 *                           with bf16 inputs rounded back to bf16, before use
 *   GDR_PROLOGUE_GATE_LOGIT the alpha argument holds the gate's pre-activation x, and
 *                           alpha = exp(-softplus(x)) is formed in the kernel */
#define GDR_PROLOGUE_L2NORM_QK 1u
#define GDR_PROLOGUE_GATE_LOGIT 2u
#define GDR_L2NORM_EPS 1e-6f

/* Version of this ABI (major * 10000 + minor * 100 + patch). */
GDR_API int gdr_version(void);

/* Message describing the last non-OK status returned on the calling thread
 * (empty string if none).  The pointer stays valid until the thread's next call
 * into the library. */
GDR_API const char* gdr_last_error(void);

/* Bytes of device workspace with which gdn_prefill / kda_prefill run their
 * fastest path for these sizes (kda != 0 selects KDA); 0 when the sizes are
 * invalid.  The workspace holds the device status word of the bounded waits
 * (the first 256 bytes) and, for the bf16 two-kernel prefills (d_k = 128, d_v a
 * multiple of 32), the precomputed operands of every chunk of 64 tokens per
 * (sequence, head): 128.5 KB per chunk for either mixer.  Any workspace of at least
 * 256 bytes is accepted: with less than the returned size the single-kernel
 * tensor-core path runs (slower; it needs the status word only).  It must be
 * zero-filled once when allocated; the library leaves it ready for the next call. */
GDR_API size_t gdr_prefill_workspace_bytes(int B, int T, int H, int dk, int dv, int kda);

/* Chunked prefill: runs the recurrence over T tokens for B sequences and H heads
 * and returns every output plus the final state.
 *
 *   q, k     [B, T, H, d_k]   in_dtype
 *   v        [B, T, H, d_v]   in_dtype
 *   alpha    GDN: [B, T, H] fp32, one gate per (token, head)
 *            KDA: [B, T, H, d_k] fp32, one gate per key channel
 *   beta     [B, T, H] fp32
 *   s0       [B, H, d_v, d_k] fp32 initial state, or NULL for zeros
 *   o        [B, T, H, d_v]   out_dtype (written)
 *   s_final  [B, H, d_v, d_k] fp32 (written), or NULL to skip; may be the same
 *            pointer as s0 (in-place carry), must not otherwise overlap inputs
 *   chunk    must be GDR_CHUNK (64)
 *   workspace, ws_bytes: at least 256 bytes (gdr_prefill_workspace_bytes(...)
 *            for the fastest path), zero-filled at allocation, 256-byte aligned
 * B, T or H equal to 0 is a valid empty call (with T == 0, s_final receives s0,
 * or zeros when s0 is NULL).  in_dtype GDR_F32 runs the fp32 CUDA-core kernel;
 * GDR_BF16 runs the tensor-core kernel where one exists for (d_k, d_v). */
GDR_API gdr_status gdn_prefill(const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta, const float* s0,
                       void* o, float* s_final,
                       int B, int T, int H, int dk, int dv,
                       int in_dtype, int out_dtype, int chunk,
                       void* workspace, size_t ws_bytes, void* stream);

/* Same contract as gdn_prefill with the per-channel gate alpha [B, T, H, d_k]. */
GDR_API gdr_status kda_prefill(const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta, const float* s0,
                       void* o, float* s_final,
                       int B, int T, int H, int dk, int dv,
                       int in_dtype, int out_dtype, int chunk,
                       void* workspace, size_t ws_bytes, void* stream);

/* Packed variable-length prefill.  "Super Apriel: One Checkpoint, Many Speeds", §2D
 * (inference and serving) and §4 (context-length scaling): a serving engine prefills
 * prompts of many lengths together and keeps each one's recurrent state for its later
 * decode steps.  nseq sequences are packed along the token axis:
 *
 *   q, k        [total, H, d_k]  bf16; sequence i is rows cu_seqlens[i] .. cu_seqlens[i+1]-1
 *   v           [total, H, d_v]  bf16
 *   alpha       GDN: [total, H] fp32;  KDA: [total, H, d_k] fp32
 *   beta        [total, H] fp32
 *   cu_seqlens  [nseq + 1] int32 DEVICE array, cu_seqlens[0] = 0, non-decreasing,
 *               cu_seqlens[nseq] = total (a sequence may be empty)
 *   state       [nslots, H, d_v, d_k] fp32 pool: sequence i starts from slot slots[i]
 *               and its final state is written back there (in place); slots is an
 *               int32 DEVICE array [nseq], or NULL for slot i; slots must be distinct
 *               and within the pool (a negative slot leaves the pool untouched for
 *               that sequence; the checks build also records it, see gdr_check_status)
 *   o           [total, H, d_v]  out_dtype (written)
 *   workspace   gdr_prefill_varlen_workspace_bytes(...) bytes, 256-byte aligned,
 *               zero-filled at allocation (the status word stays zero between calls)
 *
 * Chunks of 64 tokens never cross a sequence boundary.  Runs on the bf16 two-kernel
 * tensor-core path only: in_dtype GDR_BF16, d_k = 128, d_v in {32, 64, 128}; other
 * parameters return GDR_ERR_UNSUPPORTED.  Offsets that are not a partition of
 * [0, total) are detected on the device: no chunk is processed and
 * gdr_workspace_status returns GDR_ERR_INVALID_ARG. */
GDR_API size_t gdr_prefill_varlen_workspace_bytes(int nseq, int total, int H, int dk, int dv,
                                                  int kda);
GDR_API gdr_status gdn_prefill_varlen(const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta, const int* cu_seqlens,
                       const int* slots, float* state, void* o,
                       int nseq, int total, int H, int dk, int dv,
                       int in_dtype, int out_dtype, int chunk,
                       void* workspace, size_t ws_bytes, void* stream);
/* Same contract as gdn_prefill_varlen with the per-channel gate alpha [total, H, d_k]. */
GDR_API gdr_status kda_prefill_varlen(const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta, const int* cu_seqlens,
                       const int* slots, float* state, void* o,
                       int nseq, int total, int H, int dk, int dv,
                       int in_dtype, int out_dtype, int chunk,
                       void* workspace, size_t ws_bytes, void* stream);

/* One decode step: one new token for each of N sequences, the state updated IN
 * PLACE.
 *
 *   q, k     [N, H, d_k]   in_dtype
 *   v        [N, H, d_v]   in_dtype
 *   alpha    GDN: [N, H] fp32; KDA: [N, H, d_k] fp32
 *   beta     [N, H] fp32
 *   state    [N, H, d_v, d_k] fp32, read and overwritten with S_t
 *   o        [N, H, d_v]   out_dtype (written), o = S_t q_t
 * N or H equal to 0 is a valid empty call.  No workspace is used. */
GDR_API gdr_status gdn_decode(const void* q, const void* k, const void* v,
                      const float* alpha, const float* beta, float* state, void* o,
                      int N, int H, int dk, int dv, int in_dtype, int out_dtype,
                      void* stream);

/* Same contract as gdn_decode with the per-channel gate alpha [N, H, d_k]. */
GDR_API gdr_status kda_decode(const void* q, const void* k, const void* v,
                      const float* alpha, const float* beta, float* state, void* o,
                      int N, int H, int dk, int dv, int in_dtype, int out_dtype,
                      void* stream);

/* gdn_prefill for callers that cannot allocate device memory.  The paper has no
 * counterpart to this entry point; it exists for callers such as serving loops
 * that must never stall the device (cudaMalloc and cudaFree can synchronize it)
 * and embedders whose device memory is owned by another allocator under a fixed
 * budget.  Arguments, results and errors are those of gdn_prefill without the
 * workspace: the library uses a static device array of 4096 bytes instead,
 * reserved on every GPU that loads the library until the process exits.  The
 * prefill it runs (the single-kernel tensor-core kernel for bf16 inputs with
 * d_k = 128, else the CUDA-core kernel) needs only the 256-byte status word of
 * that array, for any sizes; sizes beyond what the library indexes (those for which
 * gdr_prefill_workspace_bytes returns 0) are rejected with GDR_ERR_INVALID_ARG.  The
 * first call on a device looks up the array's device address with that device
 * current, so make that first call before any stream capture; a failed lookup is
 * tried again on the next call.  The call allocates nothing.  After the prefill it
 * enqueues a one-warp kernel that moves the array's status word into a sticky
 * per-device word, which gdr_noalloc_status reads; if that launch fails the call
 * returns GDR_ERR_CUDA although the prefill was already enqueued.  All calls share
 * the one array: calls that overlap on the GPU (streams without ordering between
 * them) race. */
GDR_API gdr_status gdn_prefill_noalloc(const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta, const float* s0,
                       void* o, float* s_final,
                       int B, int T, int H, int dk, int dv,
                       int in_dtype, int out_dtype, int chunk, void* stream);

/* Synchronises `stream`, then reads and clears the sticky status of
 * gdn_prefill_noalloc on the current device: GDR_ERR_TIMEOUT if a bounded device
 * wait of any call since the last query gave up (the outputs of those calls are
 * undefined), GDR_OK otherwise.  No counterpart in the paper; allocates nothing. */
GDR_API gdr_status gdr_noalloc_status(void* stream);

/* Largest number of tokens per (sequence, head) that gdn_verify / kda_verify take. */
#define GDR_VERIFY_MAX_TOKENS 16

/* Multi-token step from a carried state, keeping the state after every token.
 * "Super Apriel: One Checkpoint, Many Speeds", §2D (inference and serving) and §4
 * (speculative decoding): the all-GDN placement drafts tokens that the all-FA placement
 * verifies, with no separate draft model, so a recurrent mixer must be able to run K
 * tokens from its state and then continue from whichever of them was the last one
 * accepted.  For each of N sequences and H heads this runs the recurrence over K tokens
 * (1 <= K <= GDR_VERIFY_MAX_TOKENS) starting from `state`:
 *
 *   q, k       [N, K, H, d_k]   in_dtype
 *   v          [N, K, H, d_v]   in_dtype
 *   alpha      GDN: [N, K, H] fp32;  KDA: [N, K, H, d_k] fp32
 *   beta       [N, K, H] fp32
 *   state      [N, H, d_v, d_k] fp32, the state before the first token
 *   snapshots  [K, N, H, d_v, d_k] fp32 (written): snapshots[t] is the whole state
 *              after token t+1, so the caller adopts snapshots[m-1] after accepting m
 *              tokens without a copy; `state` is then only read.  NULL: no snapshots,
 *              and `state` is updated in place to the state after the K tokens (a
 *              K-token decode).  Must not overlap state or the inputs.
 *   o          [N, K, H, d_v]   out_dtype (written), o[n, t] = S_{t+1} q_t
 *
 * N or H equal to 0 is a valid empty call.  No workspace is used.  Same head sizes and
 * dtypes as the decode entry points. */
GDR_API gdr_status gdn_verify(const void* q, const void* k, const void* v,
                      const float* alpha, const float* beta, float* state, float* snapshots,
                      void* o, int N, int K, int H, int dk, int dv,
                      int in_dtype, int out_dtype, void* stream);

/* Same contract as gdn_verify with the per-channel gate alpha [N, K, H, d_k]. */
GDR_API gdr_status kda_verify(const void* q, const void* k, const void* v,
                      const float* alpha, const float* beta, float* state, float* snapshots,
                      void* o, int N, int K, int H, int dk, int dv,
                      int in_dtype, int out_dtype, void* stream);

/* Fused prologue.  The configurations draw q and k L2-normalised per (token, head) and
 * the gates as alpha = exp(-softplus(x)) of a pre-activation x; these variants take the
 * raw tensors and do that inside the kernels (the pages leave the projections around the
 * mixer unspecified, so this is the form the configurations imply).  Each has the
 * arguments of its plain counterpart plus `prologue`, a set of GDR_PROLOGUE_* flags
 * (0 = the plain call; other bits: GDR_ERR_INVALID_ARG):
 *   GDR_PROLOGUE_L2NORM_QK   q, k raw (any scale): used as q / sqrt(|q|^2 + 1e-6), the
 *                            same for k, formed in fp32 and, for bf16 inputs, rounded to
 *                            bf16 before use
 *   GDR_PROLOGUE_GATE_LOGIT  alpha holds x (same shape); the gate is exp(-softplus(x))
 * The bf16 d_k = 128 prefill fuses the prologue into its per-chunk prep kernel when the
 * workspace has gdr_prefill_workspace_bytes(...) bytes, else runs the CUDA-core kernel
 * (which fuses it as well); decode and verify fuse it into their kernels. */
GDR_API gdr_status gdn_prefill_ex(const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta, const float* s0,
                       void* o, float* s_final, int B, int T, int H, int dk, int dv,
                       int in_dtype, int out_dtype, int chunk,
                       void* workspace, size_t ws_bytes, void* stream, unsigned prologue);
GDR_API gdr_status kda_prefill_ex(const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta, const float* s0,
                       void* o, float* s_final, int B, int T, int H, int dk, int dv,
                       int in_dtype, int out_dtype, int chunk,
                       void* workspace, size_t ws_bytes, void* stream, unsigned prologue);
GDR_API gdr_status gdn_decode_ex(const void* q, const void* k, const void* v,
                      const float* alpha, const float* beta, float* state, void* o,
                      int N, int H, int dk, int dv, int in_dtype, int out_dtype,
                      void* stream, unsigned prologue);
GDR_API gdr_status kda_decode_ex(const void* q, const void* k, const void* v,
                      const float* alpha, const float* beta, float* state, void* o,
                      int N, int H, int dk, int dv, int in_dtype, int out_dtype,
                      void* stream, unsigned prologue);
GDR_API gdr_status gdn_verify_ex(const void* q, const void* k, const void* v,
                      const float* alpha, const float* beta, float* state,
                      float* snapshots, void* o, int N, int K, int H, int dk, int dv,
                      int in_dtype, int out_dtype, void* stream, unsigned prologue);
GDR_API gdr_status kda_verify_ex(const void* q, const void* k, const void* v,
                      const float* alpha, const float* beta, float* state,
                      float* snapshots, void* o, int N, int K, int H, int dk, int dv,
                      int in_dtype, int out_dtype, void* stream, unsigned prologue);
GDR_API gdr_status gdn_prefill_varlen_ex(const void* q, const void* k, const void* v,
                              const float* alpha, const float* beta,
                              const int* cu_seqlens, const int* slots, float* state,
                              void* o, int nseq, int total, int H, int dk, int dv,
                              int in_dtype, int out_dtype, int chunk, void* workspace,
                              size_t ws_bytes, void* stream, unsigned prologue);
GDR_API gdr_status kda_prefill_varlen_ex(const void* q, const void* k, const void* v,
                              const float* alpha, const float* beta,
                              const int* cu_seqlens, const int* slots, float* state,
                              void* o, int nseq, int total, int H, int dk, int dv,
                              int in_dtype, int out_dtype, int chunk, void* workspace,
                              size_t ws_bytes, void* stream, unsigned prologue);

/* Gradients of the mixers.  "Super Apriel: One Checkpoint, Many Speeds", §2B (Training
 * Recipe): the mixers are trained (stochastic distillation, then supervised fine-tuning),
 * so the recurrence of §2A is differentiated with respect to its inputs, gates and
 * initial state.  For a dense batch with the forward arguments of gdn_prefill /
 * kda_prefill, and the gradients of a loss L with respect to the outputs and the final
 * state:
 *
 *   dO        [B, T, H, d_v]   do_dtype, dL/do
 *   ds_final  [B, H, d_v, d_k] fp32 dL/dS_T, or NULL for zeros
 *
 * writes (all fp32, none may overlap another argument)
 *
 *   dq, dk    [B, T, H, d_k]
 *   dv        [B, T, H, d_v]
 *   dalpha    GDN: [B, T, H];  KDA: [B, T, H, d_k]   (with respect to alpha itself)
 *   dbeta     [B, T, H]
 *   ds0       [B, H, d_v, d_k] (dL/ds0; written also when s0 is NULL)
 *
 * d_k, d_v in {32, 64, 128}; in_dtype and do_dtype GDR_F32 or GDR_BF16; any T >= 0
 * (T == 0 writes ds0 = ds_final).  The gates enter as given: alpha = 0 is exact here
 * (the forward kernels floor log alpha at -GDR_LOG_GATE_FLOOR).  The workspace must hold
 * gdr_backward_workspace_bytes(B, T, H, d_k, d_v, kda) bytes, 16-byte aligned (no zero
 * fill needed): the state entering every chunk of 64 tokens and two fp32 values per
 * token and value channel.  Pointers are device pointers, 16-byte aligned.  Results are
 * deterministic (no atomics). */
GDR_API size_t gdr_backward_workspace_bytes(int B, int T, int H, int dk, int dv, int kda);
GDR_API gdr_status gdn_backward(const void* q, const void* k, const void* v,
                        const float* alpha, const float* beta, const float* s0,
                        const void* dO, const float* ds_final,
                        float* dq, float* dk_out, float* dv_out, float* dalpha,
                        float* dbeta, float* ds0,
                        int B, int T, int H, int dk, int dv,
                        int in_dtype, int do_dtype,
                        void* workspace, size_t ws_bytes, void* stream);
/* Same contract with the per-channel gate alpha [B, T, H, d_k] and dalpha likewise. */
GDR_API gdr_status kda_backward(const void* q, const void* k, const void* v,
                        const float* alpha, const float* beta, const float* s0,
                        const void* dO, const float* ds_final,
                        float* dq, float* dk_out, float* dv_out, float* dalpha,
                        float* dbeta, float* ds0,
                        int B, int T, int H, int dk, int dv,
                        int in_dtype, int do_dtype,
                        void* workspace, size_t ws_bytes, void* stream);

/* Which prefill kernel a call with these parameters runs: 1 = the bf16
 * tensor-core (tcgen05) kernel, 0 = the fp32 CUDA-core kernel, -1 = the
 * parameters are not supported.  Pure host query, no CUDA call. */
GDR_API int gdr_prefill_path(int dk, int dv, int in_dtype, int kda);

/* Synchronises `stream`, reads the device status word in `workspace` and clears
 * it.  Returns GDR_OK, GDR_ERR_TIMEOUT if a bounded device-side wait of a
 * prefill kernel gave up since the last check (the outputs of that call are
 * then undefined), GDR_ERR_INVALID_ARG if a packed-sequence call found its offsets
 * inconsistent (nothing was processed), or GDR_ERR_CUDA. */
GDR_API gdr_status gdr_workspace_status(void* workspace, size_t ws_bytes, void* stream);

/* Debug aid; the paper has no counterpart.  The library also comes as a debug build,
 * libgdr_checks.so (compiled with -DGDR_CHECKS), whose kernels test the indices they
 * derive from device data and from their launch layout before using them: a chunk's
 * sequence, first token and length against the tensors (bit 1), a batch entry or
 * state-pool slot (bit 2; slots only for sign, the pool size is not passed), a chunk
 * image against the workspace (bit 4), a decode / verify thread's rows (bit 8).  A
 * failed test skips the access and sets its bit in one device word per GPU.  This
 * call synchronises `stream`, reads and clears that word of the current device and
 * returns GDR_OK, or GDR_ERR_INVALID_ARG naming the bits.  The product build,
 * libgdr.so, has no such checks and returns GDR_ERR_UNSUPPORTED without a CUDA call. */
GDR_API gdr_status gdr_check_status(void* stream);

/* Measurement aid; the paper has no counterpart.  gdr_timing_start() clears the
 * record and makes every later prefill call record a CUDA event on its stream when
 * it starts and after each kernel it launches (the two-kernel paths launch a
 * per-chunk prep kernel, then the state carry).  gdr_timing_stop() stops
 * recording, waits for the recorded events and writes to avg_ms[i] the mean
 * duration in milliseconds of the i-th kernel of a call over the recorded calls
 * (at most max_kernels entries; avg_ms may be NULL), and the number of recorded
 * calls to *ncalls (may be NULL).  Returns the number of kernels per call, or -1
 * if reading an event failed.  Process-wide; not for use inside stream capture. */
GDR_API int gdr_timing_start(void);
GDR_API int gdr_timing_stop(float* avg_ms, int max_kernels, int* ncalls);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* GDR_H_ */
