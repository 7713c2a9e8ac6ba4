/*
 * kda.h -- C ABI of libkda.so: the KDA (Kimi Delta Attention) forward pass and
 * single-token decode step on NVIDIA B200 (sm_100a).
 *
 * The method.  The worldcybernews article "Kimi K3 Open Model Surpasses Closed
 * GPT and Anthropic Systems on Independent Benchmarks", paragraph 2, replaces
 * the KV cache by a fixed-size state matrix S per head, updated by the delta
 * rule with a write strength beta and a forgetting coefficient alpha that is
 * clamped between e^-5 and 1.  Paragraph 3 of the same article processes the
 * tokens of a chunk in parallel and reconstructs the sequential states across
 * chunks with a prefix scan.  The page prints no equation; this library
 * computes, per sequence and head, with alpha per key channel:
 *
 *     a_t = clamp(alpha_t, e^-5, 1)                               [d_k]
 *     S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T   [d_k x d_v]
 *     o_t = S_t^T q_t                                             [d_v]
 *
 * No query scale and no normalisation are applied: q and k are used as given.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never frees or retains them beyond the call.
 *   - Row-major layouts, innermost dimension last, no padding.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream); no
 *     entry point synchronises the device except where stated.
 *   - Arguments are validated before anything is launched; a rejected call has
 *     no side effects.  Nothing is thrown across the ABI.
 *   - Alignment: kda_forward's q, k, v, alpha, S0, out and S_final and
 *     kda_decode_step's S must be 16-byte aligned; every other pointer must be
 *     aligned to its element size.  A misaligned pointer is KDA_ERR_INVALID_ARG.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle type as cudaStream_t / CUstream. */
typedef struct CUstream_st* kda_stream_t;

typedef enum {
    KDA_F32 = 0,   /* IEEE binary32 */
    KDA_BF16 = 1   /* bfloat16 */
} kda_dtype_t;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,     /* a NULL, misaligned or inconsistent argument */
    KDA_ERR_UNSUPPORTED = 2,     /* valid, but a size or dtype the library has no kernel for */
    KDA_ERR_CUDA = 3,            /* a CUDA runtime error (launch or device) */
    KDA_ERR_DEVICE_TIMEOUT = 4   /* a bounded device-side wait gave up */
} kda_status_t;

/*
 * kda_forward -- chunk-parallel KDA forward over whole sequences (prefill).
 * Article paragraph 2 (the update) and paragraph 3 (chunk-parallel processing
 * with sequential states reconstructed across chunks).
 *
 *   q, k, alpha : [B, T, H, d_k]   in_dtype
 *   v           : [B, T, H, d_v]   in_dtype
 *   beta        : [B, T, H]        in_dtype
 *   S0          : NULL (zero initial state) or fp32 [N, H, d_k, d_v]
 *   cu_seqlens  : NULL for a dense batch (N = B sequences of T tokens), or
 *                 int32 [num_seqs + 1] for a packed batch: B must be 1,
 *                 N = num_seqs, sequence n owns tokens [cu_seqlens[n],
 *                 cu_seqlens[n+1]), cu_seqlens[0] = 0, cu_seqlens[num_seqs] = T,
 *                 non-decreasing.  cu_seqlens is device memory and only the
 *                 kernels read it; each kernel clamps the offsets it reads into
 *                 [0, T] (a malformed table gives wrong results, never an
 *                 out-of-bounds access).
 *   out         : [B, T, H, d_v]   out_dtype (written for every token)
 *   S_final     : NULL or fp32 [N, H, d_k, d_v]; the state after each
 *                 sequence's last token.  May alias S0 exactly (in-place update);
 *                 any other overlap is undefined.
 *   chunk       : tokens per chunk: 64 (16 and 32 are accepted by the fp32 path).
 *   in_dtype    : KDA_F32 or KDA_BF16 for q, k, v, alpha, beta.
 *   out_dtype   : KDA_F32 or KDA_BF16.
 *
 * Supported: d_k, d_v in {64, 128}; H >= 1; T >= 0 (T = 0 only writes S_final
 * = S0).  bf16 inputs with d_k = d_v = 128 and chunk 64 run on the
 * tensor-core (tcgen05) kernel; every other supported combination runs on the
 * fp32 CUDA-core kernel.
 * Returns KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED or KDA_ERR_CUDA.
 */
kda_status_t kda_forward(const void* q, const void* k, const void* v,
                         const void* alpha, const void* beta, const float* S0,
                         const int32_t* cu_seqlens, int32_t num_seqs,
                         void* out, float* S_final,
                         int32_t B, int64_t T, int32_t H, int32_t d_k, int32_t d_v,
                         int32_t chunk, kda_dtype_t in_dtype, kda_dtype_t out_dtype,
                         kda_stream_t stream);

/*
 * kda_decode_step -- one token for each of N sequences, the state updated in
 * place (the fixed-size state that replaces the KV cache, article paragraph 2).
 *
 *   q, k, alpha : [N, H, d_k]      in_dtype
 *   v           : [N, H, d_v]      in_dtype
 *   beta        : [N, H]           in_dtype
 *   S           : fp32 [N, H, d_k, d_v], read and overwritten with S_t
 *   out         : [N, H, d_v]      out_dtype, o_t = S_t^T q_t
 *
 * Supported: d_k, d_v in {64, 128}.  Returns as kda_forward.
 */
kda_status_t kda_decode_step(const void* q, const void* k, const void* v,
                             const void* alpha, const void* beta, float* S, void* out,
                             int32_t N, int32_t H, int32_t d_k, int32_t d_v,
                             kda_dtype_t in_dtype, kda_dtype_t out_dtype,
                             kda_stream_t stream);

/*
 * kda_segment_maps -- the affine state map of every sequence's token range:
 * S_end = M S_start + N, with M (d_k x d_k) and N (d_k x d_v), for the
 * sequence-parallel forward.  The article's paragraph 3 reconstructs the
 * sequential states across GPUs with a prefix scan; the pages give no algebra
 * for it.  Here each rank holds one contiguous time segment of the sequences,
 * computes these maps for it, exchanges them (an all-gather) and applies the
 * maps of the earlier segments to S0 with kda_segment_scan to get its own start
 * state, then runs kda_forward from that state.  Per chunk of C tokens the map is
 * M_c = Diag(gamma_C) - (k*eta)^T Tb (k*gamma) and N_c = (k*eta)^T Tb V
 * (notation of kda_forward's chunk form), composed in order.
 *
 *   k, alpha : [B, T, H, d_k]   in_dtype;  v : [B, T, H, d_v];  beta : [B, T, H]
 *   cu_seqlens, num_seqs : as kda_forward (packed batch when non-NULL)
 *   maps     : fp32 [N, H, d_k, d_k + d_v], row c = [M[c, :] | N[c, :]] (written)
 *
 * Supported: bf16 inputs, d_k = d_v = 128, chunk 64 (the tensor-core kernel in
 * its map mode).  A sequence with no tokens gets [I | 0].  16-byte alignment for
 * k, v, alpha and maps.  Returns as kda_forward.
 */
kda_status_t kda_segment_maps(const void* k, const void* v, const void* alpha, const void* beta,
                              const int32_t* cu_seqlens, int32_t num_seqs, float* maps,
                              int32_t B, int64_t T, int32_t H, int32_t d_k, int32_t d_v,
                              int32_t chunk, kda_dtype_t in_dtype, kda_stream_t stream);

/*
 * kda_segment_scan -- applies num_maps segment maps in order to S0:
 * S <- M_g S + N_g for g = 0 .. num_maps-1, in fp32, and writes the result.
 *
 *   S0   : NULL (zero state) or fp32 [N, H, d_k, d_v]
 *   maps : fp32 [num_maps, N, H, d_k, d_k + d_v] (kda_segment_maps outputs, stacked
 *          in segment order)
 *   out  : fp32 [N, H, d_k, d_v]; may alias S0 exactly
 *
 * Supported: d_k = d_v = 128; num_maps >= 0 (0 copies S0, or zeros).  16-byte
 * alignment for every pointer.  Returns as kda_forward.
 */
kda_status_t kda_segment_scan(const float* S0, const float* maps, int32_t num_maps, float* out,
                              int32_t num_seqs, int32_t H, int32_t d_k, int32_t d_v,
                              kda_stream_t stream);

/*
 * Fused input-side transforms (no counterpart on the pages: the forms that the
 * gates and keys take before the update).  Same arguments and layouts as
 * kda_forward / kda_decode_step, but:
 *   alpha_logits x : the gate is alpha = exp(-softplus(x)) = 1 / (1 + e^x), then
 *                    clamped to [e^-5, 1] as usual;
 *   beta_logits  y : beta = sigmoid(y) = 1 / (1 + e^-y);
 *   q, k           : raw; each (token, head) vector is L2-normalised inside
 *                    (q / sqrt(max(||q||^2, 1e-12))), in fp32.
 * The transforms run inside the kernels that consume the inputs, so no extra
 * pass over the inputs is made.  kda_forward_fused supports the tensor-core
 * configuration only (bf16 in and out, d_k = d_v = 128, chunk 64; time
 * segments as kda_forward); kda_decode_step_fused every configuration of
 * kda_decode_step.  Returns as kda_forward.
 */
kda_status_t kda_forward_fused(const void* q, const void* k, const void* v,
                               const void* alpha_logits, const void* beta_logits,
                               const float* S0, const int32_t* cu_seqlens, int32_t num_seqs,
                               void* out, float* S_final, int32_t B, int64_t T, int32_t H,
                               int32_t d_k, int32_t d_v, int32_t chunk, kda_dtype_t in_dtype,
                               kda_dtype_t out_dtype, kda_stream_t stream);
kda_status_t kda_decode_step_fused(const void* q, const void* k, const void* v,
                                   const void* alpha_logits, const void* beta_logits, float* S,
                                   void* out, int32_t N, int32_t H, int32_t d_k, int32_t d_v,
                                   kda_dtype_t in_dtype, kda_dtype_t out_dtype,
                                   kda_stream_t stream);

/*
 * State slots for serving (no counterpart on the pages beyond paragraph 2's
 * fixed-size state that replaces the KV cache): the states of many sequences
 * live in one pool S_pool, fp32 [num_slots, H, d_k, d_v], and each call names
 * the slot of every sequence it advances, int32 slots[N] (device memory).  A
 * slot outside [0, num_slots) marks a padding sequence: it is computed from a
 * zero state and no state is written.  Two sequences of one call must not name
 * the same slot (undefined result).  Every slot not named is left untouched.
 *
 * kda_forward_indexed -- kda_forward over N sequences of any length (e.g. 2-16
 * draft tokens per sequence in a multi-token decode step), starting from and
 * updating S_pool[slots[n]] in place.  Arguments otherwise as kda_forward; it
 * never splits sequences along time.  A dense batch of at most 16 tokens per
 * sequence runs token by token in fp32 with the state held on chip for the
 * whole step (read and written once); longer or packed batches run on the
 * chunk kernels.
 *
 * kda_decode_step_indexed -- kda_decode_step with the state of sequence n at
 * S_pool[slots[n]], updated in place.
 *
 * Returns as kda_forward.
 */
kda_status_t kda_forward_indexed(const void* q, const void* k, const void* v,
                                 const void* alpha, const void* beta, float* S_pool,
                                 int32_t num_slots, const int32_t* slots,
                                 const int32_t* cu_seqlens, int32_t num_seqs, void* out,
                                 int32_t B, int64_t T, int32_t H, int32_t d_k, int32_t d_v,
                                 int32_t chunk, kda_dtype_t in_dtype, kda_dtype_t out_dtype,
                                 kda_stream_t stream);
kda_status_t kda_decode_step_indexed(const void* q, const void* k, const void* v,
                                     const void* alpha, const void* beta, float* S_pool,
                                     int32_t num_slots, const int32_t* slots, void* out,
                                     int32_t N, int32_t H, int32_t d_k, int32_t d_v,
                                     kda_dtype_t in_dtype, kda_dtype_t out_dtype,
                                     kda_stream_t stream);

/* A static, human-readable name for a status code (never NULL). */
const char* kda_status_string(kda_status_t status);

/*
 * Bytes of device workspace kda_forward uses for a dense batch of these sizes:
 * the per-device status word (4 bytes, allocated on the first tensor-core call
 * on a device and kept until exit) plus, when the tensor-core path splits the
 * sequences along time (see kda_forward_segments), every segment's map and
 * start state, B * H * g * d_k * (d_k + 2 d_v) fp32 values for g segments, and
 * the map rows Qg of every token, B * T * H * d_k bf16 values (as large as the
 * output).  That part is allocated stream-ordered on the call's stream from a
 * memory pool of this library, which keeps what it has reserved for later calls
 * (kda_release_workspace hands it back), and freed into that pool behind the
 * call's kernels; if it cannot be allocated the call runs unsplit.  Host-only.
 */
size_t kda_forward_workspace_bytes(int32_t B, int64_t T, int32_t H, int32_t d_k,
                                   int32_t d_v, int32_t chunk);

/*
 * Returns the device memory that the current device's workspace pool (see
 * kda_forward_workspace_bytes) keeps between calls, except what work still
 * queued on a stream uses.  Returns KDA_OK, or KDA_ERR_CUDA.  Later calls
 * allocate again as needed.
 */
kda_status_t kda_release_workspace(void);

/*
 * Time segments per sequence that kda_forward's tensor-core path uses for
 * num_seqs sequences of tokens_per_seq tokens (a packed batch uses its mean
 * length) and H heads on a GPU with num_sms SMs (0: the current device's, 148
 * if none is visible).  1 = each (sequence, head) runs whole on one CTA.  With
 * g > 1, every sequence's chunks are cut into g runs, all run in parallel by one
 * kernel from a zero start: each run's affine state map S_end = M S_start + N,
 * its output O0 from a zero start state and the rows Qg that carry the start
 * state into the output (o = O0 + Qg S_start, the output being affine in the
 * start state too); a scan kernel chains the start states in fp32 (and gives
 * S_final), and a last kernel adds Qg S_start to the output (the article's
 * paragraph 3: states reconstructed across chunks by a prefix scan).  The
 * choice only balances the SMs: every g gives the same result up to rounding.
 * Host-only.
 */
int32_t kda_forward_segments(int32_t num_seqs, int64_t tokens_per_seq, int32_t H, int32_t num_sms);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* kda_last_error(void);

/*
 * Name of the kernel kda_forward would launch for these arguments, or NULL if
 * it would reject them: "chunk_tc_bf16" (tcgen05 tensor-core kernel) or
 * "chunk_simt_f32" (fp32 CUDA-core kernel).  Host-only, launches nothing.
 */
const char* kda_forward_kernel_name(int32_t d_k, int32_t d_v, int32_t chunk,
                                    kda_dtype_t in_dtype, kda_dtype_t out_dtype);

/*
 * Number of kernels this library has launched in this process (all entry
 * points, all threads).  A host-side counter, for accounting in benchmarks.
 */
uint64_t kda_launch_count(void);

/*
 * Device-side error check.  Every wait inside the tensor-core kernel is
 * bounded (2 s); a kernel whose wait gives up stops, frees its tensor memory
 * and sets a per-device status word instead of hanging.  This call
 * synchronises `stream`, reads and clears that word for the current device and
 * returns KDA_ERR_DEVICE_TIMEOUT if it was set, else KDA_OK (or KDA_ERR_CUDA).
 * With the environment variable KDA_DEBUG=1, kda_forward makes this check
 * itself after every tensor-core launch (and therefore synchronises).
 */
kda_status_t kda_device_status(kda_stream_t stream);

/*
 * Self-test of the device-timeout path (no counterpart on the pages).  Launches
 * one warp that waits, bounded by limit_ns nanoseconds (1 ns .. 10 s), on an
 * mbarrier that nothing ever arrives on, using the same bounded wait as the
 * tensor-core kernel; when the wait gives up the kernel sets the device status
 * word and returns.  A following kda_device_status reports
 * KDA_ERR_DEVICE_TIMEOUT (and clears the word).  Nothing faults or hangs.
 */
kda_status_t kda_selftest_timeout(uint64_t limit_ns, kda_stream_t stream);

/*
 * Capacity of kda_forward_noalloc's fixed scratch: (sequence, head) pairs per call.
 */
#define KDA_NOALLOC_MAX_SEQ_HEADS 16384

/*
 * kda_forward_noalloc -- kda_forward's tensor-core path without any device
 * allocation.  The pages have no counterpart: this exists for callers that
 * cannot call cudaMalloc (for example a server or training loop that has
 * reserved the device memory for its own pool, or a latency-critical loop in
 * which an allocation may synchronise the device).  kda_forward allocates one
 * status word per GPU on its first tensor-core call; this entry point instead
 * uses a fixed device array compiled into the library.
 *
 *   Arguments, layouts and results are those of kda_forward.  Only the
 *   tensor-core configuration is accepted: in_dtype = out_dtype = KDA_BF16,
 *   d_k = d_v = 128, chunk = 64 (anything else: KDA_ERR_UNSUPPORTED).
 *   Scratch: one status word per (sequence, head), at most
 *   KDA_NOALLOC_MAX_SEQ_HEADS (64 KiB per GPU, held by every GPU that loads
 *   the library until the process exits).  More (sequence, head) pairs than
 *   that: KDA_ERR_UNSUPPORTED, with the reason in kda_last_error().
 *   Every call on a device shares the array, which keeps the last call's
 *   contents (word n * H + h: 0 = finished, 1 = a bounded device wait of that
 *   (sequence, head) gave up and its out / S_final rows are not valid); each
 *   CTA writes its own word, so nothing needs clearing first.  The call itself
 *   returns KDA_OK once the kernel is launched: read the words back with
 *   kda_noalloc_status to learn of a timeout.  Calls whose kernels overlap on
 *   the GPU race on the array.
 *   With the environment variable KDA_DEBUG set (not "0"), the call waits for
 *   its kernel and returns what kda_noalloc_status reports for its words.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current and keeps it for the
 *   life of the process; make that first call before any stream capture, and
 *   do not use these entry points on a device after cudaDeviceReset.  No
 *   cudaMalloc, cudaFree or other allocating routine is called.
 */
kda_status_t kda_forward_noalloc(const void* q, const void* k, const void* v,
                                 const void* alpha, const void* beta, const float* S0,
                                 const int32_t* cu_seqlens, int32_t num_seqs,
                                 void* out, float* S_final,
                                 int32_t B, int64_t T, int32_t H, int32_t d_k, int32_t d_v,
                                 int32_t chunk, kda_dtype_t in_dtype, kda_dtype_t out_dtype,
                                 kda_stream_t stream);

/*
 * Status words of kda_forward_noalloc (no counterpart on the pages; allocates
 * nothing).  Synchronises `stream`, then copies the first num_words words
 * (0 .. KDA_NOALLOC_MAX_SEQ_HEADS) of the fixed array of the current device
 * into host_words (host memory the caller owns, num_words int32 values; NULL:
 * the words are only inspected) and returns KDA_ERR_DEVICE_TIMEOUT if any of
 * them is non-zero, KDA_OK if all are 0, KDA_ERR_INVALID_ARG for a bad count,
 * KDA_ERR_CUDA on a runtime error.  After a kda_forward_noalloc call of
 * N sequences and H heads, the first N * H words are that call's.
 */
kda_status_t kda_noalloc_status(int32_t num_words, int32_t* host_words, kda_stream_t stream);

/*
 * Self-test of kda_forward_noalloc's timeout report (no counterpart on the
 * pages).  Launches one warp that waits, bounded by limit_ns nanoseconds
 * (1 ns .. 10 s), on an mbarrier nothing arrives on, with the forward kernel's
 * bounded wait, and writes the outcome into word `word` (0 ..
 * KDA_NOALLOC_MAX_SEQ_HEADS - 1) of the fixed array as a forward CTA does
 * (1 = gave up).  Nothing faults or hangs; allocates nothing.
 */
kda_status_t kda_noalloc_selftest_timeout(uint64_t limit_ns, int32_t word, kda_stream_t stream);

/*
 * kda_backward -- gradients of kda_forward's outputs with respect to all of
 * its inputs (the backward pass, for training).  The pages print no backward;
 * this is the reverse mode of the recurrence of the worldcybernews article
 * "Kimi K3 Open Model Surpasses Closed GPT and Anthropic Systems on Independent
 * Benchmarks", paragraph 2, as kda_forward computes it (a_t = clamp(alpha_t,
 * e^-5, 1); S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T;
 * o_t = S_t^T q_t).  For a loss L, given dL/d out (`dout`) and dL/d S_final
 * (`dS_final`, NULL = zero), it writes dL/dq, dL/dk, dL/dv, dL/dalpha,
 * dL/dbeta and dL/dS0.  The clamp passes the gradient to alpha where alpha lies
 * in [e^-5, 1] (bounds included) and blocks it outside.
 *
 *   q, k, alpha, v, beta, S0, cu_seqlens, num_seqs, B, T, H, d_k, d_v: as
 *     kda_forward (device pointers, caller-owned; S0 NULL = zero state).
 *   dout: like out, in in_dtype ([B, T, H, d_v]).
 *   dq, dk, dalpha: fp32 [B, T, H, d_k]; dv: fp32 [B, T, H, d_v]; dbeta: fp32
 *     [B, T, H]; all written for every token.  dS0: fp32 like S0 (NULL = not
 *     wanted).  None of them may alias an input.
 *   workspace: NULL, or device memory of at least kda_backward_workspace_bytes
 *     (16-byte aligned, caller-owned, contents not preserved).  NULL: the call
 *     allocates what its kernels need stream-ordered (cudaMallocAsync) and
 *     frees it after them, on `stream`.
 *   Supported: d_k, d_v in {64, 128}; in_dtype KDA_F32 or KDA_BF16; S0,
 *     dS_final, dS0 and workspace 16-byte aligned.
 *   Two implementations, chosen by the arguments:
 *   - in_dtype KDA_BF16 with d_k = d_v = 128 (and at most 65535 sequences):
 *     the chunk-parallel form on the tensor cores (bf16 MMA operands, fp32
 *     accumulation; errors of a few 1e-3 relative to an exact backward).  Three
 *     kernels: the forward recurrence writes, per chunk of 64 tokens and head, a
 *     record of its start state and operand tiles (about 233 KB); a reverse pass
 *     per (sequence, head) carries dS_final back to dS0 and writes dv and part
 *     of dbeta; a pass over all (chunk, head) pairs in parallel writes dq, dk,
 *     dalpha and the rest of dbeta.  Workspace: the records, about 3.6 KB per
 *     (token, head).  A bounded device wait that gives up sets the device status
 *     word (kda_device_status).
 *   - otherwise: the token-sequential reverse mode in fp32 (one CTA per
 *     (sequence, head), state and gradient in registers, states recomputed from
 *     checkpoints every 8 tokens; the workspace holds ceil(T / 8) + 8 states of
 *     d_k x d_v fp32 per (sequence, head)).
 *   Tokens of a packed batch outside [cu_seqlens[0], cu_seqlens[num_seqs]) are
 *   not written.
 *
 *   Returns KDA_OK; KDA_ERR_INVALID_ARG (missing or misaligned pointer, bad
 *   size, workspace too small); KDA_ERR_UNSUPPORTED (head dims, more than
 *   2^31 - 1 (sequence, head) pairs); KDA_ERR_CUDA (launch or allocation
 *   failure, reason in kda_last_error()).
 */
kda_status_t kda_backward(const void* q, const void* k, const void* v, const void* alpha,
                          const void* beta, const float* S0, const void* dout,
                          const float* dS_final, const int32_t* cu_seqlens, int32_t num_seqs,
                          float* dq, float* dk, float* dv, float* dalpha, float* dbeta,
                          float* dS0, int32_t B, int64_t T, int32_t H, int32_t d_k, int32_t d_v,
                          kda_dtype_t in_dtype, void* workspace, size_t workspace_bytes,
                          kda_stream_t stream);
/* Workspace bytes kda_backward needs for these sizes (cu_seqlens given: packed
 * = 1, num_seqs sequences in T packed tokens; else B sequences of T tokens).  The
 * dtype is not an argument: for d_k = d_v = 128 the value covers both
 * implementations (the larger of the two). */
size_t kda_backward_workspace_bytes(int32_t B, int64_t T, int32_t H, int32_t d_k, int32_t d_v,
                                    int32_t packed, int32_t num_seqs);

#ifdef __cplusplus
}
#endif
#endif /* KDA_H_ */
