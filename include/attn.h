/*
 * attn.h -- C ABI of the B200 (sm_100a) exact-attention library (libattn.so).
 *
 * The library computes exact scaled-dot-product attention in bf16 with fp32
 * accumulation:
 *
 *   forward   O = softmax(scale * Q K^T + mask) V   and the per-row
 *             log-sum-exp LSE_i = log sum_j exp(scale * q_i . k_j) over the
 *             allowed keys j (natural log of the scaled scores),
 *   backward  dQ, dK, dV of a loss L given dO = dL/dO, with P recomputed
 *             from the LSE.
 *
 * This is the operation the attention pages benchmark: the cosmos-framework
 * issue #118 ("FA2 vs NATTEN on A100", benchmark script) calls it through a
 * varlen frontend with cu_seqlens and max_seqlen, 32 query / 8 key-value heads
 * and head_dim 128; the flash-attention issue #2729 ("FA4/B200 return_lse=True
 * makes D64 forward about 19% faster", repro script) calls the forward with
 * caller-provided out and lse buffers and a return_lse switch and checks it
 * against torch's scaled_dot_product_attention; the "FA4 head_dim=256 B200
 * Regression Check" (Environment, Results) times forward and backward at
 * head_dim^-0.5 scale, MHA and GQA with one key-value head, causal and not; the
 * FA4 repository guide (Key Patterns, Backward Kernels) describes a forward that
 * streams K/V blocks past a resident Q tile with an online softmax and writes O
 * and the LSE, and a backward split into preprocess, main and postprocess kernels.
 *
 * Layouts (row-major, last index fastest, every pointer DEVICE memory):
 *   q, out, dout, dq : bf16  [total_q][nheads_q][head_dim]
 *   k, v, dk, dv     : bf16  [total_k][nheads_kv][head_dim]
 *   lse              : fp32  [nheads_q][total_q]
 *   cu_seqlens_q/_k  : int32 [batch + 1], cu[0] = 0, non-decreasing,
 *                      cu_q[batch] = total_q, cu_k[batch] = total_k.
 * Segment b holds query rows [cu_q[b], cu_q[b+1]) and key rows
 * [cu_k[b], cu_k[b+1]); a dense (batch, seqlen) tensor is the packed case with
 * cu = {0, S, 2S, ...} and needs no copy.  A segment may be empty.
 *
 * Heads: query head h reads key/value head h / (nheads_q / nheads_kv)
 * (contiguous groups; nheads_q must be a multiple of nheads_kv).  MHA is
 * nheads_kv = nheads_q, MQA is nheads_kv = 1.
 *
 * Causal masking is bottom-right aligned: query row i of a segment may see key
 * j iff j <= i + (s_k - s_q).  A query row that sees no key gets O = 0,
 * LSE = -inf and contributes nothing to any gradient.
 *
 * head_dim is 64, 128 or 256.  scale must be finite and > 0 (the pages use
 * head_dim^-0.5).  Every base pointer must be 16-byte aligned.
 *
 * Ownership: the caller allocates every buffer, including the workspace the
 * backward needs.  The library allocates no device memory, keeps no state
 * between calls except one device error word per device, and never
 * synchronises the stream except in attn_last_device_error.  All work is
 * enqueued on `stream` (0 = legacy default stream).
 *
 * Errors: arguments are checked on the host before anything is launched;
 * a bad argument returns ATTN_ERR_INVALID_ARG (or ATTN_ERR_UNSUPPORTED for a
 * head_dim or device the library has no kernel for) and launches nothing.
 * A failed launch returns ATTN_ERR_CUDA.  Every wait inside a kernel is
 * bounded; if one runs out, the kernel records it in the device error word and
 * exits without trapping, and attn_last_device_error reports ATTN_ERR_TIMEOUT.
 * The contents of cu_seqlens are not checked on the device: they must satisfy
 * the conditions above and max_seqlen_q/k must bound every segment length.
 */
#ifndef EXACT_ATTENTION_B200_ATTN_H
#define EXACT_ATTENTION_B200_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* attn_stream_t; /* same type as cudaStream_t */

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,
  ATTN_ERR_UNSUPPORTED = 2,
  ATTN_ERR_CUDA = 3,
  ATTN_ERR_TIMEOUT = 4,
  ATTN_ERR_SCRATCH_TOO_SMALL = 5 /* attn_bwd_static_scratch: problem too large */
} attn_status_t;

/*
 * Forward pass (FA4 repository guide, Key Patterns: a resident Q tile, a
 * pipelined loop over K/V blocks with an online softmax, then O and the LSE are
 * stored; issue #2729's repro calls the forward with out, lse and return_lse).
 *
 *   q, k, v        inputs, layouts above (read only).
 *   cu_seqlens_q/k device int32 [batch+1].
 *   batch          number of segments, >= 1.
 *   total_q        rows of q/out (= cu_q[batch]); sizes the LSE rows.
 *   total_k        rows of k/v  (= cu_k[batch]).
 *   max_seqlen_q/k upper bounds of the segment lengths (>= 0).
 *   nheads_q, nheads_kv, head_dim, scale, causal  as described above.
 *   return_lse     0: lse is not written (may be NULL); 1: lse must be valid.
 *   out            bf16 [total_q][nheads_q][head_dim], written.
 *   lse            fp32 [nheads_q][total_q], written iff return_lse.
 *   stream         CUDA stream.
 * Returns ATTN_OK once the kernel is enqueued.
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v,
                       const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                       int32_t batch, int32_t total_q, int32_t total_k,
                       int32_t max_seqlen_q, int32_t max_seqlen_k,
                       int32_t nheads_q, int32_t nheads_kv, int32_t head_dim,
                       float scale, int32_t causal, int32_t return_lse,
                       void* out, float* lse, attn_stream_t stream);

/*
 * Forward pass with a local (sliding-window) mask and a softcap (FA4
 * repository guide, Public API: window_size_left/right and softcap are
 * parameters of the varlen entry point; the page gives no formula, and this
 * library takes the plainest reading):
 *
 *   window_left, window_right  with delta = s_k - s_q of the segment, key j is
 *                  allowed for query row i iff j >= i + delta - window_left
 *                  (when window_left >= 0) and j <= i + delta + window_right
 *                  (when window_right >= 0); a negative bound means none.
 *                  causal = 1 adds j <= i + delta as before.  Rows left with
 *                  no allowed key get O = 0 and LSE = -inf.
 *   softcap        0: none; > 0: every scaled score s = scale * q_i . k_j
 *                  becomes softcap * tanh(s / softcap) before the softmax (the
 *                  LSE is over the capped scores).  Negative or non-finite
 *                  values return ATTN_ERR_INVALID_ARG.
 *
 * Every other argument is as for attn_fwd; attn_fwd is attn_fwd_ex with
 * window_left = window_right = -1 and softcap = 0.
 */
attn_status_t attn_fwd_ex(const void* q, const void* k, const void* v,
                          const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                          int32_t batch, int32_t total_q, int32_t total_k,
                          int32_t max_seqlen_q, int32_t max_seqlen_k,
                          int32_t nheads_q, int32_t nheads_kv, int32_t head_dim,
                          float scale, int32_t causal, int32_t window_left,
                          int32_t window_right, float softcap, int32_t return_lse,
                          void* out, float* lse, attn_stream_t stream);

/*
 * SplitKV forward (FA4 repository guide, Forward Kernels: the Blackwell forward
 * supports SplitKV, and a combine kernel merges the SplitKV partial results).
 * For short query segments against long key segments (decode-like shapes) the
 * plain grid has too few CTAs; here every CTA's range of key blocks is cut into
 * num_splits contiguous parts, each run by its own CTA, which writes its part's
 * O (normalised over its own keys) and LSE to the workspace; a second kernel
 * merges them: LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s.
 *
 *   num_splits     1..128; batch * num_splits <= 65535.  1 computes exactly
 *                  what attn_fwd_ex computes (and needs no workspace).
 *   workspace      device memory of at least attn_fwd_split_workspace_size(...)
 *                  bytes, 256-byte aligned (may be NULL when num_splits == 1);
 *                  clobbered.  Calls sharing a workspace must not overlap on
 *                  the GPU.
 * Every other argument is as for attn_fwd_ex.  The result equals the
 * unsplit one up to fp32 rounding of the merge (O is still rounded to bf16
 * once, at the end).
 */
attn_status_t attn_fwd_split(const void* q, const void* k, const void* v,
                             const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                             int32_t batch, int32_t total_q, int32_t total_k,
                             int32_t max_seqlen_q, int32_t max_seqlen_k,
                             int32_t nheads_q, int32_t nheads_kv, int32_t head_dim,
                             float scale, int32_t causal, int32_t window_left,
                             int32_t window_right, float softcap, int32_t num_splits,
                             int32_t return_lse, void* out, float* lse, void* workspace,
                             size_t workspace_bytes, attn_stream_t stream);

/*
 * Bytes of device workspace attn_fwd_split needs (fp32 partial O and LSE of
 * every split; 0 for invalid sizes).
 */
size_t attn_fwd_split_workspace_size(int32_t total_q, int32_t nheads_q, int32_t head_dim,
                                     int32_t num_splits);

/*
 * Bytes of device workspace attn_bwd needs for these sizes (a pure function of
 * its arguments; 0 for invalid sizes).  The workspace holds the fp32 dQ
 * accumulator and the fp32 row-dot D_i = dO_i . O_i.
 */
size_t attn_bwd_workspace_size(int32_t batch, int32_t total_q, int32_t nheads_q,
                               int32_t head_dim);

/*
 * Backward pass (FA4 repository guide, Backward Kernels: a preprocess kernel,
 * the main kernel that recomputes P from the LSE, and a postprocess kernel).
 *
 *   q, k, v, out   as given to / produced by attn_fwd.
 *   lse            fp32 [nheads_q][total_q] from attn_fwd(return_lse = 1).
 *   dout           bf16 like out: the incoming gradient dL/dO.
 *   dq             bf16 like q, written.
 *   dk, dv         bf16 like k and v, written; for GQA each key/value head
 *                  receives the sum over its group of query heads.
 *   workspace      device memory of at least attn_bwd_workspace_size(...)
 *                  bytes, 256-byte aligned; its contents on entry do not
 *                  matter and are clobbered.
 * Other arguments as for attn_fwd.  Calls that share a workspace must not
 * overlap on the GPU.  When max_seqlen_k <= 128 every key segment fits one key
 * block, dQ is stored directly (no accumulator, two kernel launches instead of
 * three) and the accumulator part of the workspace is left untouched; the
 * results are the same bit for bit.
 */
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* out,
                       const float* lse, const void* dout,
                       const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                       int32_t batch, int32_t total_q, int32_t total_k,
                       int32_t max_seqlen_q, int32_t max_seqlen_k,
                       int32_t nheads_q, int32_t nheads_kv, int32_t head_dim,
                       float scale, int32_t causal,
                       void* dq, void* dk, void* dv,
                       void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * Backward pass with a local mask and a softcap: the gradient of attn_fwd_ex
 * with the same window_left, window_right and softcap (which must match the
 * forward call that produced out and lse).  With a softcap, dS carries the
 * derivative of the cap, 1 - (s' / softcap)^2 at the capped score s'.  Every
 * other argument is as for attn_bwd; attn_bwd is attn_bwd_ex with
 * window_left = window_right = -1 and softcap = 0.
 */
attn_status_t attn_bwd_ex(const void* q, const void* k, const void* v, const void* out,
                          const float* lse, const void* dout,
                          const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                          int32_t batch, int32_t total_q, int32_t total_k,
                          int32_t max_seqlen_q, int32_t max_seqlen_k,
                          int32_t nheads_q, int32_t nheads_kv, int32_t head_dim,
                          float scale, int32_t causal, int32_t window_left,
                          int32_t window_right, float softcap,
                          void* dq, void* dk, void* dv,
                          void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * Backward pass that allocates nothing and takes no workspace.
 *
 * The pages have no counterpart to this entry point; it exists for callers that
 * cannot call cudaMalloc and have no spare device buffer to lend as workspace:
 * plug-ins whose host process owns all device memory and exposes no allocator,
 * services that have reserved the whole device for their own pool (where a
 * foreign allocation fails or fragments it), and latency-critical loops that ban
 * allocator calls because cudaMalloc/cudaFree can synchronise the device.
 *
 * It computes exactly what attn_bwd computes, with the same arguments minus the
 * workspace: the scratch attn_bwd would take from `workspace` (the fp32 dQ
 * accumulator and the fp32 row-dot D_i) lives instead in one file-scope device
 * array of ATTN_STATIC_SCRATCH_BYTES inside the library, which every GPU that
 * loads the library holds until the process exits.
 *
 * Limits and rules:
 *   - the problem must fit: attn_bwd_workspace_size(batch, total_q, nheads_q,
 *     head_dim) <= ATTN_STATIC_SCRATCH_BYTES, else ATTN_ERR_SCRATCH_TOO_SMALL is
 *     returned and nothing is launched;
 *   - the first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture;
 *   - every call on a device shares the one array and finds the previous call's
 *     contents in it; the call clears what must start at zero itself, but calls
 *     that overlap on the GPU (other streams, other host threads) race on it and
 *     must be serialised by the caller;
 *   - no cudaMalloc, cudaFree or other allocating routine is called.
 */
#define ATTN_STATIC_SCRATCH_BYTES (64u << 20)
attn_status_t attn_bwd_static_scratch(const void* q, const void* k, const void* v,
                                      const void* out, const float* lse, const void* dout,
                                      const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                      int32_t batch, int32_t total_q, int32_t total_k,
                                      int32_t max_seqlen_q, int32_t max_seqlen_k,
                                      int32_t nheads_q, int32_t nheads_kv, int32_t head_dim,
                                      float scale, int32_t causal,
                                      void* dq, void* dk, void* dv, attn_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word.  Returns ATTN_OK, ATTN_ERR_TIMEOUT (a bounded wait in a kernel ran out;
 * `msg` names the kernel and the wait) or ATTN_ERR_CUDA (the stream reported
 * an error).  `msg` (may be NULL) receives a NUL-terminated description of at
 * most msg_len bytes.
 */
attn_status_t attn_last_device_error(attn_stream_t stream, char* msg, size_t msg_len);

/*
 * Profiling aid (not part of the computation).  After this call, in the calling
 * host thread, every attn_fwd (kernel = ATTN_KERNEL_FWD) or attn_bwd
 * (kernel = ATTN_KERNEL_BWD_MAIN: its main kernel, between the preprocess and
 * the dQ conversion) records `start` just before and `stop` just after that
 * kernel on the call's stream, so cudaEventElapsedTime gives the kernel's own
 * duration.  start/stop are cudaEvent_t handles owned by the caller; passing
 * NULL for both turns recording off.  Returns ATTN_ERR_INVALID_ARG for an
 * unknown kernel id or for exactly one NULL event.
 */
enum { ATTN_KERNEL_FWD = 0, ATTN_KERNEL_BWD_MAIN = 1 };
attn_status_t attn_set_timing_events(int32_t kernel, void* start, void* stop);

/*
 * Watchdog self-test (diagnostic, not part of the computation): launches one
 * CTA whose thread waits, through the same bounded wait every kernel uses, on a
 * shared-memory barrier that nothing ever arrives on.  The wait gives up after
 * timeout_us microseconds (1..1000000), records the give-up in the device error
 * word and the kernel exits normally: nothing traps or hangs.  A following
 * attn_last_device_error(stream, ...) then reports ATTN_ERR_TIMEOUT naming the
 * self-test.  Returns ATTN_ERR_INVALID_ARG for an out-of-range timeout.
 */
attn_status_t attn_watchdog_selftest(int32_t timeout_us, attn_stream_t stream);

/* Library version string, e.g. "exact_attention_b200 0.1 sm_100a". */
const char* attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_B200_ATTN_H */
