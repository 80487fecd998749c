/*
 * kda.h -- C ABI of libkda, a CUDA (sm_100a / B200) implementation of the
 * Kimi Delta Attention (KDA) recurrence.
 *
 * The operation (web page "NLP--技术报告解读-Kimi-K3", joezjh.github.io,
 * section Model Architecture > Kimi Delta Attention (KDA)):
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *   o_t = scale * S_t^T q_t,          S_t in R^{dk x dv},  alpha_t = exp(g_t),
 *
 * with the lower-bounded log-decay gate of the same section
 *   g_t^h = g_min * Sigmoid(exp(A_h) z_t^h),  g_min = -5,  so alpha > e^-5.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is a DEVICE pointer owned by the caller; libkda
 *    never allocates, frees or keeps device memory.  Scratch space comes from
 *    a caller-provided workspace whose size a *_workspace_size query returns.
 *  - Layouts are dense row-major ("C order"), innermost dimension last, with
 *    no padding: q, k, g [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H];
 *    o [B, T, H, dv]; states [N, H, dk, dv] (row index = key channel).
 *    Varlen batches pack N sequences along T with B == 1.
 *  - q, k, v and o share one element type (kda_dtype); g, beta, z, A_log and
 *    all states are fp32.  Arithmetic is fp32 (fp32 accumulation; bf16 or
 *    tf32 tensor-core operands on the bf16 path).  o is rounded to nearest
 *    even when it is bf16.
 *  - Every pointer must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Calls are asynchronous: they return after enqueueing work.
 *  - Argument errors are detected on the host BEFORE anything is enqueued;
 *    the call then returns the error and touches no buffer.  A failed launch
 *    returns KDA_ERR_CUDA.  Problems found on the device (a bounded wait that
 *    ran out, malformed cu_seqlens) are never trapped: they are written to a
 *    status word in the workspace, read back with kda_get_device_status().
 *  - Debug builds (the same sources compiled with -DKDA_DEBUG_CHECKS, shipped
 *    as libkda_debug.so beside libkda.so) add device-side bounds checks where
 *    a kernel derives an index from data or from a split plan: the unit and
 *    segment a CTA resolves (rows from cu_seqlens or the segment plan, state
 *    slots), the rows of o a chunk stores, the backward's per-chunk workspace
 *    slices and gradient rows.  A failed check records KDA_ERR_BOUNDS (detail:
 *    the check site) in the workspace status word and the access is skipped;
 *    nothing traps.  The decode kernels (no workspace, no status word) are not
 *    instrumented.  Release builds compile the checks away.
 */
#ifndef LIBKDA_KDA_H_
#define LIBKDA_KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kda_status {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad scale */
  KDA_ERR_UNSUPPORTED = 2,  /* dk/dv/chunk/dtype combination not built */
  KDA_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned */
  KDA_ERR_WORKSPACE = 4,    /* workspace missing or too small */
  KDA_ERR_CUDA = 5,         /* a CUDA launch or runtime call failed */
  KDA_ERR_TIMEOUT = 6,      /* device: a bounded wait gave up */
  KDA_ERR_BAD_SEQLENS = 7,  /* device: cu_seqlens not monotone / not ending at T */
  KDA_ERR_BOUNDS = 8        /* device, KDA_DEBUG_CHECKS builds: an index left its buffer */
} kda_status;

typedef enum kda_dtype { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/* Human-readable name of a status code (static storage, never NULL). */
KDA_API const char *kda_status_string(kda_status s);

/*
 * Gate (same page, Model Architecture > KDA > Lower-bounded decay):
 *   g[r, h, i] = g_min * Sigmoid(exp(A_log[h]) * z[r, h, i])
 * z, g : fp32 [rows, H, dk] (rows = B*T);  A_log : fp32 [H].
 * g may not alias z.  g_min must be finite and negative (KDA uses -5).
 */
KDA_API kda_status kda_gate_fwd(const float *z, const float *A_log, float g_min,
                        float *g, int64_t rows, int H, int dk, void *stream);

/*
 * Bytes of workspace kda_chunk_fwd needs for these arguments (always > 0:
 * it holds at least the device status word).  num_seqs is the number of
 * varlen sequences, or 0 for a dense batch.  The tensor-core path adds the
 * segment states of its long-sequence split; the fp32-accuracy path adds
 * three 32 x 32 matrices per (sequence, head) and 32-token chunk (12 KB).
 */
KDA_API size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv,
                                    int num_seqs, int chunk_size,
                                    kda_dtype in_dtype);

/*
 * Gate backward: the chain rule of kda_gate_fwd's formula (the pages give
 * the forward only).  With x = exp(A_log[h]) z and s = Sigmoid(x):
 *   dz[r, h, i]  = dg[r, h, i] g_min s (1 - s) exp(A_log[h])
 *   dA_log[h]    = sum over r, i of dg[r, h, i] g_min s (1 - s) x
 * so a caller of kda_recurrent_bwd with a gated g gets dz and dA_log from
 * its dg.  z, dg, dz : fp32 [rows, H, dk];  A_log, dA_log : fp32 [H].
 * dz may equal dg (in place); no other aliasing.  dA_log is summed in a fixed
 * order (deterministic), through a workspace of
 * kda_gate_bwd_workspace_size(H) bytes.  Supported: dk a power of two in
 * [4, 1024].
 */
KDA_API size_t kda_gate_bwd_workspace_size(int H);

KDA_API kda_status kda_gate_bwd(const float *z, const float *A_log, float g_min,
                                const float *dg, float *dz, float *dA_log, int64_t rows,
                                int H, int dk, void *workspace, size_t workspace_bytes,
                                void *stream);

/*
 * Chunkwise prefill / training forward of the recurrence above.
 *
 * Within chunks of chunk_size tokens the recurrence is evaluated in its
 * WY/UT form as dense contractions; the state is carried across chunks
 * (FlashKDA: same page, Infrastructure > KDA kernels, "training and
 * prefill"), and a long sequence with too few (sequence, head) pairs to
 * fill the GPU is split into segments whose transitions are computed
 * independently and combined exactly (same bullet list, "intra-device CP";
 * Infrastructure > KDA Context Parallelism, S = S~ + M S_prev).
 *
 *  q, k, v      : in_dtype, [B, T, H, dk|dv]
 *  g            : fp32 [B, T, H, dk]  log-decay (typically kda_gate_fwd's output)
 *  beta         : fp32 [B, T, H]
 *  init_state   : fp32 [N, H, dk, dv] or NULL for zeros (N = num_seqs if
 *                 cu_seqlens is given, else B).  May equal final_state.
 *  cu_seqlens   : NULL for a dense batch, or device int32 [num_seqs + 1],
 *                 non-decreasing from 0 to T, with B == 1.  Zero-length
 *                 sequences are allowed (final = init, no output rows).
 *                 Malformed offsets are reported on the device
 *                 (KDA_ERR_BAD_SEQLENS) and no unit runs.
 *  scale        : finite factor on o (1.0 for o = S^T q).
 *  chunk_size   : 0 = library choice, or 16, 32, 64.  The result does not
 *                 depend on it beyond rounding.  bf16 with dk = dv = 128 and
 *                 chunk 0 or 32 runs the tcgen05 tensor-core kernel; other
 *                 inputs with chunk 0 or 32 (fp32, or dk / dv below 128) run
 *                 the chunk form at fp32 accuracy on tensor-core products
 *                 with split tf32 operands (two kernels: the key-side
 *                 matrices of every chunk, then the state scan with the
 *                 outputs -- at dk = dv = 128 a tcgen05 scan whose CTA holds
 *                 all 512 TMEM columns of its SM and whose bounded waits
 *                 record KDA_ERR_TIMEOUT, detail 0xB422, if they run out;
 *                 warp-level MMAs otherwise); chunk 16 or 64 runs an fp32
 *                 CUDA-core kernel.
 *  out          : in_dtype [B, T, H, dv]; must not alias any input.
 *  final_state  : fp32 [N, H, dk, dv] or NULL.
 *  workspace    : device buffer of >= kda_chunk_fwd_workspace_size() bytes;
 *                 its first 256 bytes hold the device status word, cleared
 *                 by this call.
 * Supported: dk, dv in {32, 64, 128}; in_dtype KDA_F32 or KDA_BF16.
 */
KDA_API kda_status kda_chunk_fwd(const void *q, const void *k, const void *v,
                         const float *g, const float *beta, kda_dtype in_dtype,
                         const float *init_state, const int32_t *cu_seqlens,
                         int num_seqs, int B, int T, int H, int dk, int dv,
                         float scale, int chunk_size, void *out,
                         float *final_state, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * Cross-device context parallelism, "NLP--技术报告解读-Kimi-K3"
 * (joezjh.github.io), Infrastructure > KDA kernels (KCP): with a sequence
 * cut into consecutive segments, the state a segment leaves is
 * S_end = S~ + M S_in, where S~ is the state the segment leaves from a zero
 * state and M (dk x dk) the product of its per-token transitions
 * (I - beta_t k_t k_t^T) Diag(exp(g_t)).  Each device computes the pair of
 * its own segment, the pairs are exchanged, and each device folds the pairs
 * of the segments before its own into its incoming state.
 *
 * kda_chunk_segment_transition: the pair of every (b, h) over the T tokens
 * of q, k, v, z, beta (layouts as kda_chunk_fwd_gated, gate fused):
 *  pairs  : fp32 [B, H, 2, 128, 128]; pairs[b][h][0] = S~, pairs[b][h][1] = M
 *           (row-major, M acts on the left of the state).  Must not alias an
 *           input.
 *  workspace : device buffer of >= 256 bytes (device status word, cleared
 *           by this call).
 * Supported: in_dtype KDA_BF16, dk = dv = 128 (KDA_ERR_UNSUPPORTED
 * otherwise).  Errors as kda_chunk_fwd.
 */
KDA_API kda_status kda_chunk_segment_transition(const void *q, const void *k, const void *v,
                                                const float *z, const float *A_log,
                                                float g_min, const float *beta,
                                                kda_dtype in_dtype, int B, int T, int H,
                                                int dk, int dv, float *pairs, void *workspace,
                                                size_t workspace_bytes, void *stream);

/*
 * kda_chunk_state_prefix: the incoming state of segment `index` of `count`
 * consecutive segments: S_in[0] = init_state (or zeros if NULL),
 * S_in[r + 1] = S~_r + M_r S_in[r].
 *  pairs      : fp32 [count, B, H, 2, 128, 128], the segments' pairs in order
 *               (as gathered from the devices); only the first `index` are read.
 *  init_state : fp32 [B, H, 128, 128] or NULL.
 *  state_out  : fp32 [B, H, 128, 128]; must not alias pairs or init_state.
 * 0 <= index < count.  Supported: dk = dv = 128.
 */
KDA_API kda_status kda_chunk_state_prefix(const float *pairs, int count, int index,
                                          const float *init_state, int B, int H, int dk,
                                          int dv, float *state_out, void *stream);

/*
 * kda_chunk_fwd with the gate fused in (the chunk kernels read z instead of
 * g and form g = g_min * Sigmoid(exp(A_log[h]) * z) on the fly, saving the
 * write and re-read of g):
 *  z      : fp32 [B, T, H, dk]   (replaces g)
 *  A_log  : fp32 [H]
 *  g_min  : finite and negative (KDA uses -5)
 * Every other argument, the workspace size and the errors are as for
 * kda_chunk_fwd.
 */
KDA_API kda_status kda_chunk_fwd_gated(const void *q, const void *k, const void *v,
                               const float *z, const float *A_log, float g_min,
                               const float *beta, kda_dtype in_dtype,
                               const float *init_state, const int32_t *cu_seqlens,
                               int num_seqs, int B, int T, int H, int dk, int dv,
                               float scale, int chunk_size, void *out,
                               float *final_state, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * kda_chunk_fwd_gated (the chunkwise prefill of Infrastructure > KDA kernels,
 * same page) for a dense batch held in HOST memory: the same
 * result as copying q, k, v, z, beta (and init_state) to the device, calling
 * kda_chunk_fwd_gated and copying o and the final state back, but the batch
 * goes through the device in time slices of about T/8 tokens (>= 512), so
 * the host-to-device copies of one slice, the kernels of the previous one
 * and the device-to-host copy of the one before overlap.  The state passes
 * from slice to slice on the device.
 *  q, k, v, z, beta, A_log, init_state : HOST pointers, layouts and dtypes as
 *      kda_chunk_fwd_gated (init_state may be NULL: zeros).  Page-locked
 *      memory lets the copies run asynchronously; pageable memory works but
 *      serialises them.
 *  out : HOST [B, T, H, dv] in_dtype;  final_state : HOST fp32 [B, H, dk, dv]
 *      or NULL.  Written when `stream` reaches the end of this call's work;
 *      host buffers must stay valid until then.
 *  workspace : DEVICE, 256-byte aligned, at least
 *      kda_chunk_fwd_gated_host_workspace_size(...) bytes (two slices of
 *      inputs and outputs, two states, the chunk workspace; its first 256
 *      bytes are the device status word of every slice, for
 *      kda_get_device_status).
 *  stream : kernels and device-to-host copies; copy_stream : host-to-device
 *      copies (NULL = `stream`, no overlap).  The copies into the workspace
 *      wait for work already queued on `stream`.
 * Dense batches only (no cu_seqlens).  Supported shapes as
 * kda_chunk_fwd_gated.
 */
KDA_API size_t kda_chunk_fwd_gated_host_workspace_size(int B, int T, int H, int dk, int dv,
                                                       kda_dtype in_dtype);

KDA_API kda_status kda_chunk_fwd_gated_host(const void *q, const void *k, const void *v,
                                    const float *z, const float *A_log, float g_min,
                                    const float *beta, kda_dtype in_dtype,
                                    const float *init_state, int B, int T, int H, int dk,
                                    int dv, float scale, void *out, float *final_state,
                                    void *workspace, size_t workspace_bytes, void *stream,
                                    void *copy_stream);

/*
 * One single-token decode step for N sequences, updating the state in place
 * (KDA decoding: same page, Online serving > high-performance kernels; the
 * state is rewritten in place every token).  Per (n, h):
 *   S' = Diag(exp(g)) S;  e = beta (v - S'^T k);  S = S' + k e^T;
 *   o  = scale * S^T q.
 *  q, k : in_dtype [N, H, dk];  v, out : in_dtype [N, H, dv]
 *  g    : fp32 [N, H, dk];      beta : fp32 [N, H]
 *  state: fp32 [N, H, dk, dv], read and written once.
 * Supported: dk, dv in {32, 64, 128}.  No workspace is needed.
 */
KDA_API kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const float *g, const float *beta,
                           kda_dtype in_dtype, float *state, int N, int H,
                           int dk, int dv, float scale, void *out,
                           void *stream);

/*
 * kda_decode_step with the gate fused in: z (fp32 [N, H, dk]) and A_log
 * (fp32 [H]) replace g, and the kernel forms
 * alpha = exp(g_min * Sigmoid(exp(A_log[h]) * z)).  Other arguments as for
 * kda_decode_step.
 */
KDA_API kda_status kda_decode_step_gated(const void *q, const void *k, const void *v,
                                 const float *z, const float *A_log, float g_min,
                                 const float *beta, kda_dtype in_dtype,
                                 float *state, int N, int H, int dk, int dv,
                                 float scale, void *out, void *stream);

/*
 * Speculative decoding: verify K draft tokens per sequence without touching
 * the state (KDA Decoding: same page, Online serving > high-performance
 * kernels -- keep the draft tokens' projected inputs instead of state
 * snapshots, and rebuild the state by replaying the accepted ones).  For each
 * (n, h) the recurrence runs over tokens t = 0 .. K-1 from the committed state
 * and writes o for every token; `state` is only read.
 *  q, k, g : [N, K, H, dk]   v, out : [N, K, H, dv]   beta : fp32 [N, K, H]
 *  g is the log-decay g, or z when A_log (fp32 [H]) is not NULL, in which
 *  case g = g_min * Sigmoid(exp(A_log[h]) * z) is formed in the kernel.
 *  state : fp32 [N, H, dk, dv]  (read only)
 * Supported: 1 <= K <= 16, dk, dv in {32, 64, 128}.
 */
KDA_API kda_status kda_decode_verify(const void *q, const void *k, const void *v,
                             const float *g, const float *A_log, float g_min,
                             const float *beta, kda_dtype in_dtype,
                             const float *state, int N, int H, int K, int dk,
                             int dv, float scale, void *out, void *stream);

/*
 * Commit the accepted prefix of the draft tokens: for each (n, h) apply the
 * first m_n = accept_len[n] tokens (k, v, g or z, beta laid out as for
 * kda_decode_verify) to the state in place; m_n = 0 leaves it untouched.
 * accept_len is a device int32 [N]; values are clamped to [0, K].
 */
KDA_API kda_status kda_decode_replay(const void *k, const void *v, const float *g,
                             const float *A_log, float g_min, const float *beta,
                             kda_dtype in_dtype, float *state,
                             const int32_t *accept_len, int N, int H, int K,
                             int dk, int dv, void *stream);

/*
 * Training backward: gradients of a loss L through the recurrence, given
 * dL/do (dout) and, optionally, dL/dS_T of the final state (d_final).  The
 * pages define the forward only (Model Architecture > Kimi Delta Attention
 * (KDA); FlashKDA serves training too: Infrastructure > KDA kernels); this
 * is the chain rule of that recurrence, evaluated in the chunk form of the
 * forward (32-token chunks): a forward pass saves every chunk's start state
 * and key-side matrices, a reverse pass carries dL/dS from chunk to chunk,
 * and every chunk's token gradients are then formed in parallel.  fp32
 * arithmetic throughout (exponents of the decay taken as differences <= 0,
 * so g must be <= 0, as the gate makes it).
 *  q, k, g : [B, T, H, dk]   v, dout : [B, T, H, dv]   beta : fp32 [B, T, H]
 *  cu_seqlens, num_seqs : as kda_chunk_fwd (NULL and 0 for a dense batch; a
 *      packed batch has B == 1; malformed offsets are reported on the device,
 *      KDA_ERR_BAD_SEQLENS through kda_get_device_status, and nothing is
 *      written)
 *  init_state, d_final : fp32 [N, H, dk, dv] or NULL (zeros), N = num_seqs or B
 * Outputs (fp32, written whole; d_init may be NULL to skip it):
 *  dq, dk_out, dg : [B, T, H, dk]   dv_out : [B, T, H, dv]   dbeta : [B, T, H]
 *  d_init : [N, H, dk, dv]  (dL/dS_0)
 * dout has the element type of q, k, v.  g is the log-decay (a gated caller
 * chains dg through its gate: kda_gate_bwd).  The workspace (size from
 * kda_recurrent_bwd_workspace_size: the 256-byte device status word, the
 * packed batch's chunk offsets, and per (sequence, head) and 32-token chunk
 * two dk x dv states, three 32 x 32 matrices and four 32 x dv tiles; 0 for
 * unsupported shapes) is scratch; outputs must not alias inputs.  Dense
 * batches longer than 8192 tokens run in windows of 8192 tokens: the
 * workspace then holds one window's chunks, the start state of every later
 * window and two state gradients, so it grows by one dk x dv state per 8192
 * tokens instead of two per 32.  The forward scan runs twice (once to
 * checkpoint the window start states, once per window from its checkpoint);
 * every per-chunk step is the same arithmetic as in a single pass, with the
 * fp32 state and state gradient handed across windows unrounded.
 * Tensor cores: at dk = dv = 128 the two state scans, and at dk = 128 the
 * token-gradient pass, run their products as tcgen05 MMAs (tf32 operands
 * split into high and low parts, fp32 accumulators in TMEM: fp32 accuracy);
 * each scan CTA holds all 512 TMEM columns of its SM, so a kernel of another
 * stream that holds TMEM delays it.  Their waits on the MMAs are bounded: one
 * that runs out records KDA_ERR_TIMEOUT (detail 0xB410 the token-gradient
 * pass, 0xB420 the forward scan, 0xB421 the state-gradient scan).
 * Supported: dk, dv in {32, 64, 128}, B * T * H < 2^31.
 */
KDA_API size_t kda_recurrent_bwd_workspace_size(int B, int T, int H, int dk, int dv,
                                                int num_seqs);

KDA_API kda_status kda_recurrent_bwd(const void *q, const void *k, const void *v,
                             const float *g, const float *beta, kda_dtype in_dtype,
                             const float *init_state, const void *dout,
                             const float *d_final, const int32_t *cu_seqlens,
                             int num_seqs, int B, int T, int H, int dk,
                             int dv, float scale, float *dq, float *dk_out,
                             float *dv_out, float *dg, float *dbeta, float *d_init,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Name and description of the last CUDA error a libkda call on this host
 * thread turned into KDA_ERR_CUDA ("no error" if none).  Static storage.
 */
KDA_API const char *kda_last_cuda_error_string(void);

/*
 * Synchronises `stream`, then returns the device status word that kernels
 * of an earlier kda_chunk_fwd call on this workspace recorded (KDA_OK if
 * none).  If detail is not NULL it receives a code-specific value (the
 * block that recorded the error).  Returns KDA_ERR_CUDA if the
 * synchronisation itself failed.
 */
KDA_API kda_status kda_get_device_status(const void *workspace, void *stream,
                                 int32_t *detail);

/*
 * Diagnostic for the device-side failure path: launches one block that
 * waits on a flag in the workspace that nothing sets, giving up after
 * `spin_limit_ns` nanoseconds (clamped to [1e3, 5e9]), and records
 * KDA_ERR_TIMEOUT in the status word exactly as the chunk kernels do when
 * one of their waits runs out.  Needs 256 bytes of workspace.
 */
/*
 * 1 in a KDA_DEBUG_CHECKS build, 0 otherwise (host only, no CUDA call).
 */
KDA_API int kda_debug_checks_enabled(void);

/*
 * Diagnostic for the debug build's bounds checks: launches one thread that
 * asks the device-side check whether index 1 lies in a buffer of 1 element.
 * The check records KDA_ERR_BOUNDS (detail 0x5E1F) in the status word of
 * `workspace` (256 bytes needed) and no memory is accessed.  Returns
 * KDA_ERR_UNSUPPORTED without launching in a release build.
 */
KDA_API kda_status kda_selftest_bounds_check(void *workspace, void *stream);

KDA_API kda_status kda_selftest_bounded_wait(void *workspace, int64_t spin_limit_ns,
                                     void *stream);

/*
 * Diagnostic for the chunk kernels' own failure path: sets the limit of
 * every bounded wait inside the tensor-core chunk kernel (the hand-offs
 * between its warp roles), process-wide, for launches that follow.  The
 * default is 2e9 ns (far above any real wait); `limit_ns` is clamped to
 * [0, 5e9].  With a limit of 0 a wait that is not satisfied at its first
 * poll runs out: the kernel records KDA_ERR_TIMEOUT in the workspace status
 * word, lets the asynchronous copies and tensor-core operations it issued
 * land, releases its tensor memory and returns, leaving its outputs
 * partly written; the context stays usable.  Waits that drain in-flight work
 * keep the default bound.  Returns KDA_OK.
 */
KDA_API kda_status kda_set_wait_limit_ns(int64_t limit_ns);

/*
 * kda_chunk_fwd without a workspace, for callers that cannot allocate device
 * memory (an engine plugin limited to memory its host planned up front, a
 * service whose allocator is frozen after warm-up, a fixed device-memory
 * budget).  The pages have no counterpart: this is a library convenience.
 *
 * Arguments, results and host-side errors are those of kda_chunk_fwd minus
 * the workspace.  Its scratch is a __device__ array of
 * KDA_NOALLOC_SCRATCH_BYTES compiled into the library, held on every GPU
 * that loads the library until the process exits; a problem whose scratch
 * would not fit (for instance a very long sequence with few heads, which
 * the segment split needs room for) returns KDA_ERR_WORKSPACE with nothing
 * enqueued.  All calls share that array, so calls whose GPU work overlaps
 * race and must be serialised by the caller.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress) with that
 * device current: make it before any stream capture.  If the device is
 * reset (cudaDeviceReset), the next call sees a new context and looks the
 * address up again.  Device-side status (KDA_ERR_BAD_SEQLENS,
 * KDA_ERR_TIMEOUT) is recorded in the built-in array, where
 * kda_noalloc_get_device_status reads it; with malformed cu_seqlens no unit
 * runs and out / final_state are left as they were.  Returns KDA_ERR_CUDA if
 * no device is current.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (8u << 20)

KDA_API kda_status kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                 const float *g, const float *beta,
                                 kda_dtype in_dtype, const float *init_state,
                                 const int32_t *cu_seqlens, int num_seqs, int B,
                                 int T, int H, int dk, int dv, float scale,
                                 int chunk_size, void *out, float *final_state,
                                 void *stream);

/*
 * The device status word of the last kda_chunk_fwd_noalloc call on the
 * current device: synchronises `stream`, then reads the status the kernels
 * recorded in the built-in scratch (KDA_OK if none), exactly as
 * kda_get_device_status does for a workspace; `detail` (nullable) receives
 * the code-specific value.  The pages have no counterpart.  Allocates
 * nothing.  Returns KDA_ERR_CUDA if the synchronisation or the read failed.
 */
KDA_API kda_status kda_noalloc_get_device_status(int32_t *detail, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBKDA_KDA_H_ */
