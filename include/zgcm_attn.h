/*
 * zgcm_attn.h — C ABI of the ZGCM-1 gated window-attention layer on B200 (sm_100a).
 *
 * One attention layer of the ZGCM-1 hybrid decoder, forward and backward:
 *
 *   per-head QK-RMSNorm -> partial RoPE on the first `rope_dims` head dims ->
 *   GQA (query head h reads KV head h / (Hq/Hkv)) -> causal attention restricted to
 *   the `window` most recent keys (key j visible to query i iff i - window < j <= i) ->
 *   output multiplied elementwise by sigmoid(g).
 *
 * Where each piece is defined:
 *   - window of 128 nearest tokens, 5:1 local:global interleave, global layers at
 *     6/12/18/24/30: ZGCM-1 summary (paper.rainbus.top), section "前置知识 / 滑动窗口注意力
 *     (SWA)与混合注意力"; the same facts in the shibing624 review, section "架构：5:1 的门控滑窗注意力".
 *   - QK-RMSNorm, RoPE ratio 0.33, GQA 32 query / 8 KV heads: shibing624 review, section
 *     "架构"; ZGCM-1 summary, section "核心方法".
 *   - the sigmoid output gate: shibing624 review, section "架构" (the sentence says the
 *     local attention output is multiplied by a sigmoid gate; the formula itself was lost
 *     from the page).  Read here as out = sigmoid(g) * attn with g supplied by the caller,
 *     one logit per output element.
 *   - gated sliding-window and full attention interleaved: yunkai-blog summary, section
 *     "关键技术点 1 (Architecture & System Co-design)".
 *   window >= S gives the full-causal global layer of the same model.
 *
 * Conventions shared by every entry point
 *   - Tensors are DEVICE pointers, contiguous, BSHD order, bf16 (raw 16-bit storage)
 *     unless stated: q, g, out, dout, dq, dg are [B, S, Hq, D]; k, v, dk, dv are
 *     [B, S, Hkv, D]; lse is fp32 [B, Hq, S]; gamma_q, gamma_k, dgamma_q, dgamma_k are
 *     fp32 [D].  Every pointer must be 16-byte aligned (ZGCM_ERR_ALIGNMENT otherwise).
 *   - Ownership: the caller owns every buffer.  The library keeps no state between calls
 *     and allocates no device memory, with one exception: zgcm_attn_fwd takes its key
 *     scratch from the device's stream-ordered pool (see there); zgcm_attn_fwd_ws is the
 *     same call with caller-owned scratch.
 *   - Streams: every call is asynchronous on `cuda_stream` (a cudaStream_t, NULL = legacy
 *     default stream) and never synchronises the device.
 *   - Errors: arguments are checked on the host before anything is launched; a failed
 *     check returns a negative zgcm_status and launches nothing.  A failed launch returns
 *     ZGCM_ERR_CUDA.  No kernel traps.
 *   - Supported shapes: D == 128, Hq % Hkv == 0, Hq, Hkv >= 1, rope_dims even with
 *     0 <= rope_dims <= D, window >= 1, causal == 1, B >= 0, S >= 0, B*S*Hq*D < 2^40.
 *     B == 0 or S == 0 is a valid empty problem (backward still zeroes dgamma_*).
 *   - Positions are 0..S-1 in every sequence of the batch.
 *   - Thread-safe and re-entrant: no global mutable state.
 */
#ifndef ZGCM_ATTN_H
#define ZGCM_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ZGCM_OK = 0,
    ZGCM_ERR_INVALID_ARG = -1, /* null pointer, negative size, window < 1, eps < 0, ...   */
    ZGCM_ERR_UNSUPPORTED = -2, /* valid but not implemented: D != 128, causal == 0, ...   */
    ZGCM_ERR_ALIGNMENT = -3,   /* a tensor pointer is not 16-byte aligned                 */
    ZGCM_ERR_WORKSPACE = -4,   /* workspace null or smaller than the size query returns  */
    ZGCM_ERR_CUDA = -5,        /* a CUDA runtime call or a kernel launch failed          */
    ZGCM_ERR_TIMEOUT = -6,     /* a bounded device-side wait gave up                     */
    ZGCM_ERR_TOO_LARGE = -7    /* problem needs more scratch than zgcm_attn_bwd_noalloc has */
} zgcm_status;

/* Human-readable name of a zgcm_status value (static string, never NULL). */
const char* zgcm_status_string(int status);

/*
 * Forward of one gated attention layer.
 *
 *   q_hat = RoPE(gamma_q * q / sqrt(mean_d q^2 + eps))     per (b, s, query head)
 *   k_hat = RoPE(gamma_k * k / sqrt(mean_d k^2 + eps))     per (b, s, KV head)
 *   s_ij  = scale * q_hat_i . k_hat_j            for max(0, i-window+1) <= j <= i
 *   A_i   = sum_j softmax_j(s_ij) v_j ;  out_i = sigmoid(g_i) * A_i
 *   lse_i = log sum_j exp(s_ij)                  (natural log, kept for backward)
 *
 * RoPE rotates pairs (t, t + rope_dims/2) for t < rope_dims/2 by angle pos * theta_t,
 * theta_t = rope_base^(-2t/rope_dims); dims >= rope_dims pass through.
 *
 * In : q, g bf16 [B,S,Hq,D]; k, v bf16 [B,S,Hkv,D]; gamma_q, gamma_k fp32 [D].
 * Out: out bf16 [B,S,Hq,D] (rounded once, to nearest even); lse fp32 [B,Hq,S].
 * out/lse must not alias any input.
 * The tcgen05 kernels need device scratch for the normalised keys
 * (zgcm_attn_fwd_workspace_size bytes): this call takes it with cudaMallocAsync on
 * `cuda_stream` and returns it with cudaFreeAsync after the kernels, so it never
 * synchronises; callers that manage memory themselves use zgcm_attn_fwd_ws.
 */
int zgcm_attn_fwd(const void* q, const void* k, const void* v, const void* g,
                  const float* gamma_q, const float* gamma_k,
                  int B, int S, int Hq, int Hkv, int D, int rope_dims,
                  double rope_base, int window, int causal, float eps, float scale,
                  void* out, float* lse, void* cuda_stream);

/*
 * Bytes of device scratch the forward needs for this configuration.  0 for the sliding layer
 * with 4 query heads per KV head (window up to 128: the strip kernel normalises its key
 * chunks in shared memory, so zgcm_attn_fwd allocates nothing there), for an empty problem
 * and for invalid arguments.  Otherwise (wider windows, the global layer among them, and
 * sliding windows with another group size) B*S*Hkv*D*2 rounded up to 256: the fp16
 * normalised, rotated keys, written once per key tile by the preparation kernel
 * (fwd_prep_k_kernel) and read by every query block that sees the tile; zgcm_attn_fwd takes
 * them from the stream-ordered pool of the caller's stream (cudaMallocAsync / cudaFreeAsync).
 */
size_t zgcm_attn_fwd_workspace_size(int B, int S, int Hq, int Hkv, int D, int rope_dims, int window);

/*
 * zgcm_attn_fwd with caller-owned scratch: workspace must hold at least
 * zgcm_attn_fwd_workspace_size(...) bytes, 256-byte aligned (may be NULL when that is 0),
 * contents on entry irrelevant, not used by a concurrent call.  ZGCM_ERR_WORKSPACE if it
 * is missing or too small.
 */
int zgcm_attn_fwd_ws(const void* q, const void* k, const void* v, const void* g,
                     const float* gamma_q, const float* gamma_k,
                     int B, int S, int Hq, int Hkv, int D, int rope_dims,
                     double rope_base, int window, int causal, float eps, float scale,
                     void* out, float* lse, void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * Training-step pair: a forward that keeps the activations its backward would otherwise
 * recompute.  Both passes form the same fp16 q~ = RoPE(gamma_q * q / rms(q)) and k~ (times
 * the same power of two) and the same inverse RMS of every q and k row (RMSNorm backward);
 * zgcm_attn_fwd_save leaves them in a caller-owned store and zgcm_attn_bwd_saved reads them
 * there instead of converting q and k again (its preparation pass converts v alone).  The
 * results are bit-identical to zgcm_attn_fwd + zgcm_attn_bwd on the same inputs.
 *
 * zgcm_attn_saved_size: bytes of the store for this problem (every shape zgcm_attn_fwd
 *   accepts); 0 for an empty problem and for invalid arguments.
 * Layout (each part 256-byte aligned, in this order): q~ fp16 [B,S,Hq,D], q inverse RMS fp32
 *   [B,Hq,S], k~ fp16 [B,S,Hkv,D], k inverse RMS fp32 [B,Hkv,S].
 * zgcm_attn_fwd_save: zgcm_attn_fwd_ws with the store as its workspace (k~ is the forward's
 *   own key workspace).  `saved`: at least zgcm_attn_saved_size bytes, 256-byte aligned,
 *   owned by the caller; after the call (in stream order) it holds this forward's
 *   activations.  Returns ZGCM_ERR_WORKSPACE / ZGCM_ERR_ALIGNMENT for a store too
 *   small or misaligned; otherwise as zgcm_attn_fwd.
 * zgcm_attn_bwd_saved: zgcm_attn_bwd_timed given the store a zgcm_attn_fwd_save of the same
 *   inputs and arguments filled (`saved`, read only; NULL returns ZGCM_ERR_INVALID_ARG).
 *   Kernels: zgcm_attn_bwd_saved_kernel_name(i) (bwd_prep_v_kernel in place of the two
 *   preparation kernels).  The workspace is the same as zgcm_attn_bwd's.
 */
size_t zgcm_attn_saved_size(int B, int S, int Hq, int Hkv, int D, int rope_dims, int window);

int zgcm_attn_fwd_save(const void* q, const void* k, const void* v, const void* g,
                       const float* gamma_q, const float* gamma_k,
                       int B, int S, int Hq, int Hkv, int D, int rope_dims,
                       double rope_base, int window, int causal, float eps, float scale,
                       void* out, float* lse, void* saved, size_t saved_bytes, void* cuda_stream);

int zgcm_attn_bwd_saved(const void* q, const void* k, const void* v, const void* g,
                        const float* gamma_q, const float* gamma_k,
                        const void* out, const float* lse, const void* dout,
                        int B, int S, int Hq, int Hkv, int D, int rope_dims,
                        double rope_base, int window, int causal, float eps, float scale,
                        void* dq, void* dk, void* dv, void* dg,
                        float* dgamma_q, float* dgamma_k,
                        void* workspace, size_t workspace_bytes, const void* saved, size_t saved_bytes,
                        void* cuda_stream, void* const* events, int n_pairs);

const char* zgcm_attn_bwd_saved_kernel_name(int i, int S, int rope_dims, int window);

/*
 * Bytes of device workspace zgcm_attn_bwd needs for this problem (0 for an empty one).
 * Returns 0 as well for arguments zgcm_attn_bwd would reject.
 */
size_t zgcm_attn_bwd_workspace_size(int B, int S, int Hq, int Hkv, int D, int window);

/*
 * Backward of zgcm_attn_fwd: exact gradients of L = sum(dout * out) with respect to
 * q, k, v, g, gamma_q and gamma_k.
 *
 * In : the forward's inputs and arguments, its outputs `out` (bf16) and `lse` (fp32),
 *      and dout bf16 [B,S,Hq,D].  The backward forms the softmax probabilities from `lse`
 *      as exp(s_ij - lse_i), so `lse` must be the one zgcm_attn_fwd returned for these
 *      inputs: the tcgen05 kernels recompute the forward's scores bit for bit, and a
 *      log-sum-exp from elsewhere leaves the probabilities of a row summing to other than 1.
 * Out: dq, dg bf16 [B,S,Hq,D] — gradients w.r.t. the RAW q (before RMSNorm) and the gate
 *      logits; dk, dv bf16 [B,S,Hkv,D] — summed over the Hq/Hkv query heads that share
 *      each KV head; dgamma_q, dgamma_k fp32 [D] — overwritten (not accumulated).
 * workspace: device scratch of at least zgcm_attn_bwd_workspace_size(...) bytes, 256-byte
 *      aligned, owned by the caller, contents on entry irrelevant; it must not be used by
 *      another call that runs concurrently.
 * Outputs must not alias inputs or each other.
 */
int zgcm_attn_bwd(const void* q, const void* k, const void* v, const void* g,
                  const float* gamma_q, const float* gamma_k,
                  const void* out, const float* lse, const void* dout,
                  int B, int S, int Hq, int Hkv, int D, int rope_dims,
                  double rope_base, int window, int causal, float eps, float scale,
                  void* dq, void* dk, void* dv, void* dg,
                  float* dgamma_q, float* dgamma_k,
                  void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * Measurement variant of zgcm_attn_bwd: the same work on the same stream, and in addition
 * records events[2i] / events[2i+1] (cudaEvent_t created by the caller) immediately before
 * and after the i-th kernel the backward launches, for i < n_pairs, so each kernel can be
 * timed on its own.  zgcm_attn_bwd_kernel_name(i) names kernel i (NULL past the last).
 * n_pairs may be 0 (then `events` may be NULL).
 */
int zgcm_attn_bwd_timed(const void* q, const void* k, const void* v, const void* g,
                        const float* gamma_q, const float* gamma_k,
                        const void* out, const float* lse, const void* dout,
                        int B, int S, int Hq, int Hkv, int D, int rope_dims,
                        double rope_base, int window, int causal, float eps, float scale,
                        void* dq, void* dk, void* dv, void* dg,
                        float* dgamma_q, float* dgamma_k,
                        void* workspace, size_t workspace_bytes, void* cuda_stream,
                        void* const* events, int n_pairs);

/*
 * Query rows at the end of a longer key sequence: a shard of one sequence whose earlier key
 * and value rows (those its window reaches) were gathered from the ranks that own them.  The
 * layer on positions 0 .. S-1 (k, v: [B,S,Hkv,D], every position) restricted to the query
 * rows of positions q_off .. S-1, q_off = S - Sq: q, g, out, dout, dq, dg are [B,Sq,Hq,D],
 * lse [B,Hq,Sq]; row i of them is position q_off + i (its RoPE angle, its window).  The
 * rows before q_off cost nothing: no query block before them is computed.  (The shard
 * layout of the sequence-sharded long-context stage: shibing624 review, section
 * "数据与课程", the 256K stage; the global layers of the ZGCM-1 summary, section
 * "前置知识 / 滑动窗口注意力(SWA)与混合注意力", see every earlier key.)
 *
 * Arguments as zgcm_attn_fwd_ws / zgcm_attn_bwd, with Sq and S in place of S; outputs are the
 * rows zgcm_attn_fwd / zgcm_attn_bwd of the whole sequence would give for those positions,
 * and dk, dv (every key row), dgamma_q, dgamma_k the parts the given query rows contribute.
 * Workspace: zgcm_attn_fwd_workspace_size / zgcm_attn_bwd_workspace_size of (B, S, ...).
 * Requires 0 <= Sq <= S (else ZGCM_ERR_INVALID_ARG) and, when Sq < S, q_off a multiple of
 * 128 and window > 128 (else ZGCM_ERR_UNSUPPORTED: a window of at most 128 reaches 127 rows
 * back, which a caller covers by padding its query rows with zeros).  Sq == S is
 * zgcm_attn_fwd_ws / zgcm_attn_bwd.  Sq == 0: nothing to compute (the backward zeroes dk,
 * dv and dgamma_*).
 */
int zgcm_attn_fwd_rows(const void* q, const void* k, const void* v, const void* g,
                       const float* gamma_q, const float* gamma_k,
                       int B, int Sq, int S, int Hq, int Hkv, int D, int rope_dims,
                       double rope_base, int window, int causal, float eps, float scale,
                       void* out, float* lse, void* workspace, size_t workspace_bytes, void* cuda_stream);
int zgcm_attn_bwd_rows(const void* q, const void* k, const void* v, const void* g,
                       const float* gamma_q, const float* gamma_k,
                       const void* out, const float* lse, const void* dout,
                       int B, int Sq, int S, int Hq, int Hkv, int D, int rope_dims,
                       double rope_base, int window, int causal, float eps, float scale,
                       void* dq, void* dk, void* dv, void* dg,
                       float* dgamma_q, float* dgamma_k,
                       void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * zgcm_attn_bwd for callers that cannot allocate device memory.  (No counterpart in the
 * paper: this is an interface convenience of this library.)  A process that has reserved
 * the GPU's memory for its own pool, or a plugin given no allocator, cannot provide the
 * workspace zgcm_attn_bwd asks for, and cudaMalloc/cudaFree may synchronise the device.
 * This variant takes the same arguments minus the workspace and uses a fixed 64 MiB
 * scratch array that lives in the library's device image on every GPU that loads the
 * library, until the process exits.  It allocates nothing.
 *
 * Limit: problems whose zgcm_attn_bwd_workspace_size exceeds 64 MiB return
 * ZGCM_ERR_TOO_LARGE before anything runs; at 32 query / 8 KV heads, D = 128 and a
 * window of at most 128 that is B*S <= 3117 tokens (3118 is rejected).
 * Device: the array used is the calling thread's current device's, so q (and every other
 * tensor, and the stream) must be on the current device; a q that lives elsewhere returns
 * ZGCM_ERR_INVALID_ARG.  Null tensor pointers return ZGCM_ERR_INVALID_ARG.
 * The first call on a device looks up the array's device address (once per device).
 * All calls on a device share the array, which keeps the last call's contents; every
 * scratch word is written before it is read, so nothing needs clearing.  Calls whose
 * executions overlap on the GPU (other streams, other host threads) race on it.
 */
int zgcm_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* g,
                          const float* gamma_q, const float* gamma_k,
                          const void* out, const float* lse, const void* dout,
                          int B, int S, int Hq, int Hkv, int D, int rope_dims,
                          double rope_base, int window, int causal, float eps, float scale,
                          void* dq, void* dk, void* dv, void* dg,
                          float* dgamma_q, float* dgamma_k, void* cuda_stream);

/*
 * One decode step (inference): a single new token per sequence against a KV cache.  The
 * sliding layers keep a ring of `window` key/value slots per sequence (the constant-size
 * cache of the ZGCM-1 KV design: 128 tokens per sliding layer, ZGCM-1 summary section
 * "前置知识"); the global layers keep every token (a growing cache).
 *
 * For sequence b at position p = pos[b]: the new key k is RMS-normalised and rotated at p
 * (as in the forward) and stored with v in cache slot p mod cache_len; then
 *   out = sigmoid(g) * softmax_j(scale q~ . k~_j) v_j   over j = max(0, p-window+1) .. p,
 *   lse = log sum_j exp(scale q~ . k~_j),
 * the forward's row p for the same tokens (each key written by an earlier call).
 *
 * In : q, g bf16 [B,Hq,D] and k, v bf16 [B,Hkv,D]: the new token of each sequence (raw,
 *      before the norm); pos int32 [B], device: the token's position (0-based);
 *      gamma_q, gamma_k fp32 [D].
 * Cache (caller-owned, updated in place): k_cache fp16 [B,cache_len,Hkv,D] holds the
 *      normalised, rotated keys times the power of two the training kernels use for their
 *      fp16 keys (1 unless max|gamma| sqrt(D) > 16384); v_cache bf16 [B,cache_len,Hkv,D] the
 *      values.  Position j lives in slot j mod cache_len.  The window's keys must all still
 *      be there: cache_len >= min(window, p + 1) (a ring of cache_len = window slots for a
 *      sliding layer; cache_len > the longest position for a global one).  A row whose
 *      window is longer than the cache gets NaN (out and lse); its cache is not written.
 * Out: out bf16 [B,Hq,D]; lse fp32 [B,Hq].
 * workspace: at least zgcm_attn_decode_workspace_size(...) bytes, 16-byte aligned (split
 *      partial results).  Same checks, errors and stream behaviour as the forward.
 * Kernels: decode_split_kernel (one CTA per sequence, KV head and split of up to 512 keys),
 *      then decode_combine_kernel.
 */
int zgcm_attn_decode(const void* q, const void* k, const void* v, const void* g,
                     const float* gamma_q, const float* gamma_k, const int* pos,
                     int B, int Hq, int Hkv, int D, int rope_dims, double rope_base, int window,
                     float eps, float scale, void* k_cache, void* v_cache, int cache_len,
                     void* out, float* lse, void* workspace, size_t workspace_bytes, void* cuda_stream);

/* Bytes of workspace zgcm_attn_decode needs (0 for invalid arguments or B == 0). */
size_t zgcm_attn_decode_workspace_size(int B, int Hq, int window, int cache_len);

/*
 * Main kernel zgcm_attn_fwd launches for this configuration (static string), all of them
 * tcgen05 / TMEM / TMA kernels for any number of rotated dims: "fwd_strip_kernel" (windows
 * up to 128 with 4 query heads per KV head; in the training pair the Q and K preparation
 * kernels run before it), "fwd_tc_kernel" (windows up to 128, other group sizes) and
 * "fwd_glob_tc_kernel" (wider windows and the global layer), these two preceded by the key
 * preparation kernel fwd_prep_k_kernel.
 */
const char* zgcm_attn_fwd_kernel_name(int B, int S, int Hq, int Hkv, int rope_dims, int window);

/*
 * Device-side failure check.  Every wait inside the kernels is bounded; when one expires
 * the kernel records where, releases what it holds and returns early (its outputs are then
 * undefined).  This call synchronises the device, returns ZGCM_ERR_TIMEOUT if such a
 * record exists (and clears it), ZGCM_OK otherwise.
 */
int zgcm_attn_device_error(void);

/*
 * Test of the failure path above, without a fault: launches one CTA that waits on a barrier
 * nothing arrives on.  The bounded wait expires (about a second), the CTA records the site
 * as the attention kernels would and returns, so the next zgcm_attn_device_error() returns
 * ZGCM_ERR_TIMEOUT and the context stays usable.  Asynchronous on `cuda_stream`.
 */
int zgcm_attn_selftest_expired_wait(void* cuda_stream);

/* Name of the i-th kernel zgcm_attn_bwd launches for this configuration (static string),
 * or NULL when i is past the last one.  Windows up to 128 run the gate pass, the K/V and Q
 * preparation and the tcgen05 pair (bwd_gate_kernel, bwd_prep_kv_kernel, bwd_prep_q_kernel,
 * bwd_q_tc_kernel, bwd_kv_tc_kernel, then the two d_gamma reductions); wider windows (the
 * global layer among them) the same gate pass and preparation, then bwd_tile_stats_kernel,
 * bwd_q_glob_kernel, bwd_kv_tc_kernel and the two reductions.  Any number of rotated dims. */
const char* zgcm_attn_bwd_kernel_name(int i, int S, int rope_dims, int window);

#ifdef __cplusplus
}
#endif

#endif /* ZGCM_ATTN_H */
