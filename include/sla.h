/*
 * sla.h - C ABI of the SLA (Sparse-Linear Attention) hot path on B200 (sm_100a).
 *
 * What is computed.  "SLA: Beyond Sparsity in Diffusion Transformers via
 * Fine-Tunable Sparse-Linear Attention" (arXiv 2509.24006), abstract and the
 * technical-framework steps of its paper card: attention weights are sorted
 * into critical, marginal and negligible groups; critical pairs get exact
 * O(N^2) softmax attention, marginal pairs get O(N) linear attention, and
 * negligible pairs are skipped, in a forward and a backward pass.  The pages
 * leave the classifier, feature map, combination and backward open; this
 * library takes these readings:
 *   - classes are per (query block i, key block j) of `block` (64) tokens:
 *     pooled logits s_ij = mean(Q_i) . mean(K_j) * scale; per row the n_crit
 *     largest (ties: lower j first) are critical, the n_negl smallest are
 *     negligible, the rest marginal; n_crit = ceil(k_h*T - 1e-9),
 *     n_negl = min(floor(k_l*T + 1e-9), T - n_crit), T = N / block;
 *   - critical pairs: softmax attention with scale 1/sqrt(d) (or
 *     softmax_scale) over all tokens of the row's critical key blocks;
 *   - marginal pairs: phi(x) = elu(x) + 1; per key block
 *     h_j = phi(K_j)^T V_j and z_j = sum phi(K_j); per query block
 *     H_i = sum_{j marginal} h_j, Z_i likewise;
 *     O_l = phi(Q) H_i / (phi(Q) . Z_i)  (0 if row i has no marginal block);
 *   - O = O_s + O_l W_proj, W_proj one d x d matrix shared by all heads;
 *   - the backward treats the classes as constants.
 *
 * Conventions (all entry points).
 *   - Every data pointer is a DEVICE pointer, allocated and owned by the
 *     caller; the library never allocates or frees memory and keeps no
 *     state between calls (except the per-process cached TMA encoder entry
 *     point).  Sizes of caller buffers come from sla_query_sizes().
 *   - Q, K, V, O, dO: bf16, contiguous [B, H, N, d], 16-byte aligned.
 *     W_proj: bf16 row-major [d, d].  dQ, dK, dV, dW_proj: fp32.
 *   - Supported: block == 64, d in {64, 128}, N % 64 == 0, N >= 64,
 *     1 <= B*H, T = N/64 <= 4096, 0 <= k_h, 0 <= k_l, k_h + k_l <= 1.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     is asynchronous on it.  Argument errors are returned before anything is
 *     launched.  A failed launch returns SLA_ERR_CUDA.  Errors found on the
 *     device (a wait that timed out, an index out of range) are recorded in
 *     an error word inside the workspace and reported by sla_check().
 *   - Calls that share a workspace must not overlap on the device.
 *   - Nothing aborts the process and no C++ exception crosses this ABI.
 */
#ifndef SLA_H_
#define SLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SLA_API __attribute__((visibility("default")))
#else
#define SLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SLA_OK = 0,
  SLA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or fraction */
  SLA_ERR_UNSUPPORTED = 2, /* valid but not implemented (block != 64, d not 64/128) */
  SLA_ERR_WORKSPACE = 3,   /* workspace or buffer smaller than sla_query_sizes() */
  SLA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  SLA_ERR_TIMEOUT = 5,     /* a device-side wait gave up (reported by sla_check) */
  SLA_ERR_DEVICE = 6       /* a device-side invariant failed (reported by sla_check) */
} sla_status;

/* Problem shape.  softmax_scale <= 0 selects 1/sqrt(d).
 * n_valid: valid tokens per sequence (key padding); 0 means N.  Otherwise
 * N - block < n_valid <= N (only the last block may be partial).  Tokens at
 * t >= n_valid take no part: block means, softmax keys and key-block
 * summaries use valid tokens only; padded rows of o, o_s, den are 0 and of lse
 * +inf (exp(s - lse) = 0 for every key; -inf marks a real row without a
 * critical block); d_o at padded rows is ignored; dq, dk, dv there are 0.  With
 * n_valid = 0 padding tokens are ordinary tokens (the pages do not say how a
 * grid is padded to whole blocks; this is the optional exact handling). */
typedef struct {
  int B, H, N, d, block;
  double k_h, k_l;
  float softmax_scale;
  int n_valid;
} sla_shape;

/* Classification output (written by sla_classify*, read by forward/backward;
 * a mask may be reused across calls, e.g. across denoising steps).
 *   cls           int8  [B,H,T,T]   +1 critical, 0 marginal, -1 negligible
 *   crit_idx      int32 [B,H,T,n_crit]  critical key blocks, ascending
 *   marg_bits     uint32[B,H,T,ceil(T/32)]  bit j%32 of word j/32: j marginal
 *   crit_col_ptr  int32 [B,H,T+1]   CSR by key block (offsets per (b,h))
 *   crit_col_idx  int32 [B,H,T*n_crit]  query blocks with j critical, ascending
 *   pooled_logits fp32  [B,H,T,T]   optional (NULL: not written / not read) */
typedef struct {
  int8_t* cls;
  int32_t* crit_idx;
  uint32_t* marg_bits;
  int32_t* crit_col_ptr;
  int32_t* crit_col_idx;
  float* pooled_logits;
} sla_mask;

/* State saved by sla_forward for sla_backward.
 *   lse   fp32 [B,H,N]      log-sum-exp of the critical scores (-inf if none,
 *                           +inf on a padded row, see sla_shape.n_valid)
 *   o_s   fp32 [B,H,N,d]    sparse-branch output
 *   den   fp32 [B,H,N]      phi(Q).Z_i (0 if the row has no marginal block)
 *   hz_agg bf16 [2][B,H,T,d*d+d]  per query block: H_i (d x d, row-major) then
 *          Z_i (d), stored as a high plane followed by a low plane (value =
 *          hi + lo, about 16 significant bits); 4 bytes per element in all */
typedef struct {
  float* lse;
  float* o_s;
  float* den;
  void* hz_agg;
} sla_saved;

/* Sizes in bytes of every caller buffer for a shape. */
typedef struct {
  int T, n_crit, n_negl, n_marg;
  size_t cls_bytes, crit_idx_bytes, marg_bits_bytes, crit_col_ptr_bytes, crit_col_idx_bytes,
      pooled_logits_bytes;
  size_t lse_bytes, o_s_bytes, den_bytes, hz_agg_bytes;
  size_t workspace_bytes; /* one workspace serves classify, forward and backward */
} sla_sizes;

/* Fill *out for *shape.  Host only; no CUDA call. */
SLA_API sla_status sla_query_sizes(const sla_shape* shape, sla_sizes* out);

/* Pool Q and K per block, score the pooled rows and classify every
 * (query block, key block) pair into *mask.  q, k: bf16 [B,H,N,d].
 * Defined by: SLA paper card, "technical framework" step 1 and core point 2
 * (the weights split into critical, marginal and negligible), English
 * abstract; the pooled-score ranking is the reading above. */
SLA_API sla_status sla_classify(const sla_shape* shape, const void* q, const void* k,
                        const sla_mask* mask, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Classify from caller-given fp32 scores [B,H,T,T] (any values but NaN);
 * same ranking rule and outputs as sla_classify, pooled_logits untouched.
 * Lets a test feed identical scores to this library and to a reference. */
SLA_API sla_status sla_classify_from_scores(const sla_shape* shape, const float* logits,
                                    const sla_mask* mask, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* Same classification as sla_classify, for callers that cannot allocate
 * device memory when they classify (for example code running inside CUDA
 * graph capture, allocator-less embedded or real-time runtimes, or hosts
 * whose device memory comes from a pool they may not grow).  It takes no
 * workspace: its only scratch (pooled Q and K) is a fixed 16 MiB array built
 * into the library, present on every GPU that loads it until the process
 * exits, and it calls no allocating routine.  The paper has no counterpart;
 * this is a packaging variant.
 *   - Limit: 2 * B*H*T*d*4 bytes <= 16 MiB (B*H*T*d <= 2M); larger shapes get
 *     SLA_ERR_WORKSPACE.  Other arguments and outputs as sla_classify.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - Every call shares the one array: calls that overlap on the GPU (other
 *     streams, other threads) race on it and must be serialized by the caller.
 *   - The looked-up address is kept per device for the life of the process;
 *     after cudaDeviceReset() on a device it is stale, so do not call this
 *     entry point on that device again in the same process. */
SLA_API sla_status sla_classify_noalloc(const sla_shape* shape, const void* q, const void* k,
                                        const sla_mask* mask, void* stream);

/* Hierarchical selection for long sequences.  "Trainable Log-linear Sparse
 * Attention for Efficient Diffusion Transformers" (abstract): top-K is taken
 * on a coarse level first and the finer level only looks inside what the
 * coarse level kept.  Reading (the page gives no formulas):
 *   - super-block J = key blocks [J*group, min(T, (J+1)*group)); its key is
 *     Kc_J = the equal-weight mean of its blocks' mean keys; TG = ceil(T/group);
 *   - coarse scores sc_iJ = mean(Q_i) . Kc_J * scale; in the order
 *     (sc desc, J asc) the first c_hi super-blocks of row i hold its critical
 *     candidates, the last c_lo its negligible candidates;
 *   - c_hi = min(TG, max(top, f(n_crit))), c_lo = min(TG, max(bottom,
 *     f(n_negl))), f(0) = 0, f(n) = ceil(n/group) + (T % group ? 1 : 0), so
 *     the candidates always hold enough blocks; if c_hi + c_lo > TG both are
 *     TG and the result is exactly sla_classify's;
 *   - critical: the n_crit candidate blocks first in the order (s desc,
 *     j asc) of the pooled logits s_ij of sla_classify; negligible: the
 *     n_negl negligible candidates last in that order; the rest marginal.
 * Exactly n_crit critical and n_negl negligible blocks per row, as with
 * sla_classify, and the mask has the same layout and meaning.
 *   group >= 2; top, bottom >= 0 (minimum candidate counts). */
typedef struct {
  int group, top, bottom;
} sla_hierarchy;

/* TG, c_hi and c_lo of the reading above.  Host only; no CUDA call.  A flat
 * case (c_hi + c_lo > TG before the clamp) reports c_hi = c_lo = TG. */
SLA_API sla_status sla_hierarchy_counts(const sla_shape* shape, const sla_hierarchy* hier,
                                        int* n_super, int* c_hi, int* c_lo);

/* Hierarchical classification from q, k (bf16 [B,H,N,d]) into *mask, with
 * the crit_col CSR, like sla_classify.  mask->pooled_logits, if not NULL,
 * receives s_ij at the candidate blocks of each row (other entries are left
 * as they were); coarse_logits (fp32 [B,H,T,TG], 16-byte aligned, or NULL)
 * receives sc_iJ.  In a flat case the call is sla_classify: pooled_logits
 * gets every s_ij and coarse_logits is left untouched. */
SLA_API sla_status sla_classify_hierarchical(const sla_shape* shape, const void* q,
                                             const void* k, const sla_hierarchy* hier,
                                             const sla_mask* mask, float* coarse_logits,
                                             void* workspace, size_t workspace_bytes,
                                             void* stream);

/* The same selection from caller-given scores: logits fp32 [B,H,T,T] (only
 * the candidate entries are read) and coarse_logits fp32 [B,H,T,TG]; any
 * values but NaN.  mask->pooled_logits is not touched.  Lets a test feed
 * identical scores to this library and to a reference. */
SLA_API sla_status sla_classify_hierarchical_from_scores(const sla_shape* shape,
                                                         const float* logits,
                                                         const float* coarse_logits,
                                                         const sla_hierarchy* hier,
                                                         const sla_mask* mask, void* workspace,
                                                         size_t workspace_bytes, void* stream);

/* Forward with a given mask: writes o (bf16 [B,H,N,d]) and *saved.
 * Defined by: SLA English abstract and paper card "technical framework" steps
 * 2-4 (critical pairs: exact attention; marginal: linear attention; negligible:
 * skipped) and step 5 (one fused computation); the combination is the reading
 * above. */
SLA_API sla_status sla_forward(const sla_shape* shape, const void* q, const void* k, const void* v,
                       const void* w_proj, const sla_mask* mask, void* o,
                       const sla_saved* saved, void* workspace, size_t workspace_bytes,
                       void* stream);

/* Backward of sum(O * dO) with the mask held fixed.  Needs the *saved state
 * of the forward on the same inputs and mask.  Writes dq, dk, dv (fp32
 * [B,H,N,d]) and dw_proj (fp32 [d,d], summed over B, H, N; overwritten).
 * Defined by: SLA English abstract (the kernel supports the backward pass)
 * and paper card step 5; the gradients are those of the forward above. */
SLA_API sla_status sla_backward(const sla_shape* shape, const void* q, const void* k, const void* v,
                        const void* w_proj, const sla_mask* mask, const sla_saved* saved,
                        const void* d_o, float* dq, float* dk, float* dv, float* dw_proj,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Gate on the linear branch, after the page "SALAD: Achieve High-Sparsity
 * Attention via Efficient Linear Attention Tuning for Video Diffusion
 * Transformer", section "Methodologie: SALAD", items 2 (a global factor in
 * (0, 1) from a sigmoid scales the linear branch) and 3 (branches whose
 * factor is very low are dropped at inference):
 *   g = 1 / (1 + exp(-logit)),  O = O_s + g * O_l W_proj;
 *   g < skip_below: the branch is dropped, O = O_s, its kernels are not
 *   launched and neither the branch nor the logit gets a gradient.
 * logit = +inf gives g = 1 (the ungated forward, bit for bit). */
typedef struct {
  float logit;
  float skip_below;
} sla_gate;

/* sla_forward with a gate (gate must not be NULL; NaN fields are rejected).
 * A dropped branch leaves saved->hz_agg unwritten and saved->den untouched. */
SLA_API sla_status sla_forward_gated(const sla_shape* shape, const void* q, const void* k,
                                     const void* v, const void* w_proj, const sla_mask* mask,
                                     const sla_gate* gate, void* o, const sla_saved* saved,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* sla_backward with the same gate as the forward.  Also writes *d_logit
 * (device fp32 scalar, overwritten): g (1 - g) times the sum over B, H, N of
 * (O_l W_proj) . dO; 0 when the branch is dropped. */
SLA_API sla_status sla_backward_gated(const sla_shape* shape, const void* q, const void* k,
                                      const void* v, const void* w_proj, const sla_mask* mask,
                                      const sla_gate* gate, const sla_saved* saved,
                                      const void* d_o, float* dq, float* dk, float* dv,
                                      float* dw_proj, float* d_logit, void* workspace,
                                      size_t workspace_bytes, void* stream);

/* Zero the workspace's device error word (asynchronously on `stream`).  Call
 * once on a new workspace before its first use; sla_check() clears it
 * afterwards. */
SLA_API sla_status sla_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Synchronize `stream`, then return and clear the workspace's device error
 * word (SLA_OK if no device-side error was recorded). */
SLA_API sla_status sla_check(void* workspace, void* stream);

/* Test hook for the device-side failure paths.  Writes `what` into a word of
 * the workspace header that the kernels read at launch (asynchronously on
 * `stream`; sla_workspace_init() and what = 0 clear it):
 *   SLA_INJECT_WITHHOLD_LOADS  the sparse forward's copy warp issues none of
 *     its copies, so every wait on them runs out after its time limit
 *     (about 2 s); the kernel winds down with nothing in flight and
 *     sla_check() reports SLA_ERR_TIMEOUT.
 * No fault, trap or hang is involved; the CUDA context stays usable.  The
 * paper has no counterpart. */
#define SLA_INJECT_WITHHOLD_LOADS 1
SLA_API sla_status sla_debug_inject(void* workspace, int what, void* stream);

/* Static description of a status code. */
SLA_API const char* sla_strerror(sla_status status);

/* Per-kernel device time collected by the opt-in profiler. */
typedef struct {
  const char* name; /* static string, e.g. "fwd_sparse" */
  int launches;
  double total_ms;
} sla_kernel_stat;

/* Start recording: until sla_profile_end(), every kernel the library
 * launches is bracketed by two CUDA events on its stream (diagnostic only;
 * adds a few microseconds per launch).  Process-wide. */
SLA_API sla_status sla_profile_begin(void);

/* Stop recording, wait for the recorded launches, and write up to max_out
 * per-kernel totals (in first-launch order) to out; *n_out = entries written. */
SLA_API sla_status sla_profile_end(sla_kernel_stat* out, int max_out, int* n_out);

/* Library version, "major.minor.patch". */
SLA_API const char* sla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SLA_H_ */
