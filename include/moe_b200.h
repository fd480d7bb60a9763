/*
 * moe_b200.h -- C ABI of the single-GPU Mixture-of-Experts layer for B200
 * (sm_100a): router -> dispatch (permute) -> grouped SwiGLU expert MLP ->
 * combine, plus the backward of the grouped MLP.
 *
 * The stages follow the Transformer Engine documentation page "Mixture of
 * Experts" (sections Introduction, Router, Token dispatch, Token combine,
 * Token probabilities, Grouped GEMM, Grouped MLP and "Example: MoE layer on a
 * single device"). The expert MLP is the SwiGLU of the te_mixtral.py example
 * (_expert_ffn) and of torchtitan's GroupedExperts.
 *
 * Conventions, for every entry point:
 *  - Pointers. Every tensor pointer is DEVICE memory that the caller
 *    allocates and owns. Each must be 16-byte aligned, except routing_map.
 *    The library never allocates, frees or synchronises on these calls.
 *    Scratch memory is the caller's `workspace`; query its size with the
 *    matching *_workspace_size function.
 *  - Layouts are dense and row-major. bf16 tensors are passed as moe_bf16
 *    (the 16-bit pattern of a bfloat16).
 *  - Stream. Every call is asynchronous on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream). Results are valid once the stream reaches
 *    them.
 *  - Errors. Argument errors are reported before anything is launched, as
 *    MOE_ERR_INVALID_ARG (bad sizes or NULL pointers), MOE_ERR_UNSUPPORTED (a
 *    valid shape outside the kernels' limits) or MOE_ERR_WORKSPACE. A failed
 *    launch gives MOE_ERR_CUDA. Kernels report problems that they detect (an
 *    expert index outside [0,E), inconsistent offsets, a wait that timed out)
 *    in a device-side error word, and skip the offending row instead of
 *    trapping. moe_get_device_status reads and clears that word.
 *  - Limits. 1 <= E <= 256; 1 <= k <= min(E, 16); H and I are multiples of 8
 *    (rows of 16 bytes: the stride rule of the tensor-memory-access maps and of
 *    the 16-byte vector loads); T * k < 2^31.
 *  - Dropless routing. A = T * k routed rows, a static size: buffers never
 *    depend on the routing, so no device-to-host copy is needed (TE Token
 *    dispatch: num_out_tokens known statically).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16; /* bfloat16 bit pattern */

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_CUDA = 3,
    MOE_ERR_WORKSPACE = 4,
    MOE_ERR_DEVICE_CHECK = 5, /* a kernel found invalid data (index or offsets) */
    MOE_ERR_TIMEOUT = 6       /* a kernel gave up on a bounded wait */
} moe_status;

typedef enum moe_score_fn {
    MOE_SCORE_SOFTMAX = 0,
    MOE_SCORE_SIGMOID = 1
} moe_score_fn;

/*
 * Router options (TE "Mixture of Experts", Router):
 *  score_fn     MOE_SCORE_SOFTMAX or MOE_SCORE_SIGMOID.
 *  renormalize  softmax: 1 = softmax after top-k, so the k weights are a
 *               softmax over the chosen logits and sum to one; 0 = softmax
 *               over all E experts before top-k (use_pre_softmax).
 *               sigmoid: 1 = divide the k sigmoids by their sum; 0 = raw.
 *  scaling      multiplies every returned weight (scaling_factor); 1 = none.
 *  expert_bias  NULL, or device fp32 [E]. It is added to the sigmoid score for
 *               the choice of experts only, never to the weights (Load
 *               balancing section). Valid with MOE_SCORE_SIGMOID only.
 */
typedef struct moe_router_opts {
    int score_fn;
    int renormalize;
    float scaling;
    const float* expert_bias;
} moe_router_opts;

/* Human-readable name of a status code (static storage). */
const char* moe_status_string(moe_status status);

/* Synchronises `stream`, then reads and clears the device-side error word.
 * Returns MOE_OK, MOE_ERR_DEVICE_CHECK, MOE_ERR_TIMEOUT or MOE_ERR_CUDA. */
moe_status moe_get_device_status(void* stream);

/* Stage tracing. `events` points to n_events cudaEvent_t handles that the
 * caller created (with timing enabled) and owns; NULL or n_events = 0 turns
 * tracing off. While set, moe_layer_forward records them on its stream at its
 * stage boundaries, in this order:
 *   [0] start  [1] router + offsets  [2] permute  [3] gate_up + SwiGLU
 *   [4] down   [5] shared expert (recorded even without one)  [6] combine
 * (with the combine folded into the shared expert's down GEMM, see
 * moe_layer_forward, the stage [5]..[6] is empty and [4]..[5] holds it; with
 * gate_up and down in one launch, [3]..[4] is empty and [2]..[3] holds both;
 * with the permute done by the router kernel, [1]..[2] is empty);
 * moe_grouped_mlp_backward and moe_grouped_mlp_scaled_backward record:
 *   [0] start  [1] combine backward  [2] down dgrad + SwiGLU backward
 *   [3] gate_up dgrad  [4] token sum of dx  [5] down wgrad  [6] gate_up wgrad
 * Events beyond n_events are skipped. The elapsed time between consecutive
 * events is the device time of one stage. The setting is process-wide and
 * not thread-safe. Returns MOE_ERR_INVALID_ARG if n_events < 0. */
moe_status moe_trace_set(void* const* events, int n_events);

/* ------------------------------------------------------------------ router
 * moe_router_topk -- TE Router (fused_topk_with_score_function); te_mixtral.py
 * TEMixtralSparseMoeBlock.forward (fp32 softmax, top-k, renormalise).
 * All math runs in fp32. For each token t, the k experts with the largest
 * score are chosen (softmax ranks the logits; sigmoid ranks
 * sigmoid(logit) + expert_bias). Among equal scores the lower expert index
 * wins, and NaN ranks below every number.
 *  logits       in  fp32 [T, E]
 *  topk_idx     out int32 [T, k]  chosen experts, best first
 *  topk_prob    out fp32  [T, k]  routing weight of each chosen expert
 *  routing_map  out uint8 [T, E]  1 at the chosen experts, else 0 (NULL: skip)
 *  counts       out int32 [E]     tokens routed to each expert (column sums)
 *  offsets      out int32 [E+1]   offsets[0] = 0, offsets[e+1] = offsets[e] +
 *                                 counts[e]: the start of each expert block
 *                                 ("offsets are the cumulative per-expert
 *                                 counts", TE Expert parallelism, Receive buffer)
 *  workspace    scratch of moe_router_workspace_size(T, E, k) bytes
 * T = 0 is allowed: counts and offsets are zeroed. */
size_t moe_router_workspace_size(int64_t T, int E, int k);
moe_status moe_router_topk(const float* logits, int64_t T, int E, int k,
                           const moe_router_opts* opts, int32_t* topk_idx, float* topk_prob,
                           uint8_t* routing_map, int32_t* counts, int32_t* offsets,
                           void* workspace, size_t workspace_bytes, void* stream);

/* moe_router_backward -- TE Router, backward through the score function:
 * dlogits = dL/dlogits from dprob = dL/dtopk_prob, for the experts the
 * forward chose. The choice itself is piecewise constant in the logits and
 * passes no gradient; an expert_bias only moves the choice and is ignored.
 * With g_j = scaling * dprob[t,j], computed in fp32:
 *   softmax, renormalize=1: q = softmax over the chosen logits;
 *       dlogits[t, e_j] = q_j (g_j - sum_i q_i g_i), 0 at experts not chosen.
 *   softmax, renormalize=0: q = softmax over all E logits;
 *       dlogits[t, e] = q_e (G_e - sum_j q_{e_j} g_j), G_e = g_j at e = e_j, else 0.
 *   sigmoid, renormalize=0: dlogits[t, e_j] = g_j s_j (1 - s_j), s = sigmoid(logit).
 *   sigmoid, renormalize=1: r_j = s_j / S, S = sum_j s_j;
 *       dlogits[t, e_j] = (g_j - sum_i r_i g_i) / S * s_j (1 - s_j).
 *  logits    in  fp32 [T, E]   the forward's logits
 *  topk_idx  in  int32 [T, k]  the forward's choice (moe_router_topk)
 *  dprob     in  fp32 [T, k]
 *  dlogits   out fp32 [T, E]   every element written
 * opts as in the forward call. An index outside [0, E) is recorded as
 * MOE_ERR_DEVICE_CHECK (moe_get_device_status) and contributes nothing. */
moe_status moe_router_backward(const float* logits, int64_t T, int E, int k,
                               const moe_router_opts* opts, const int32_t* topk_idx,
                               const float* dprob, float* dlogits, void* stream);

/* moe_expert_bias_update -- auxiliary-loss-free load balancing between steps
 * (TE Router, Load balancing: lower the bias of overloaded experts, raise it
 * for under-used ones; torchtitan MoE._update_expert_bias). With the counts of
 * the last step (moe_router_topk's counts, on the device, no host sync):
 *   delta_e = coeff * sign(mean(counts) - counts[e]), decided exactly in
 *             integers; then delta_e -= mean(delta); expert_bias[e] += delta_e
 * in fp32. The bias is then passed to the next moe_router_topk (sigmoid score).
 *  counts       in     int32 [E]
 *  expert_bias  in/out fp32  [E]
 * E in [1, 256]. */
moe_status moe_expert_bias_update(const int32_t* counts, int E, float coeff, float* expert_bias,
                                  void* stream);

/* moe_aux_loss -- TE Mixture of Experts, Load balancing (fused_moe_aux_loss
 * on the dense scores of fused_compute_score_for_moe_aux_loss): the auxiliary
 * loss that penalises uneven token counts. The page names its inputs but
 * prints no formula; the reading implemented is the switch-style loss
 *   loss = coeff * E / (k T^2) * sum_e (sum_t s[t,e]) * counts[e],
 * which equals coeff when every expert has T k / E assignments and a mean
 * score of 1/E. The dense scores s are the softmax over all E logits
 * (MOE_SCORE_SOFTMAX) or the sigmoid of each logit (MOE_SCORE_SIGMOID), with
 * no expert bias, in fp32; the sums over tokens run in a fixed order (fp32
 * within a block, fp64 across blocks), so the result is the same on every run
 * on a given GPU.
 *  logits  in  fp32 [T, E]   the router's logits
 *  counts  in  int32 [E]     tokens per expert from the router's routing map
 *                            (moe_router_topk's counts)
 *  loss    out fp32 [1]      on the device
 *  scores  out fp32 [T, E]   the dense scores (NULL: not written)
 * T >= 1, E in [1, 256], 1 <= k <= min(E, 16). workspace of at least
 * moe_aux_loss_workspace_size(T, E) bytes, 16-byte aligned. */
size_t moe_aux_loss_workspace_size(int64_t T, int E);
moe_status moe_aux_loss(const float* logits, int64_t T, int E, int k, int score_fn,
                        const int32_t* counts, float coeff, float* loss, float* scores,
                        void* workspace, size_t workspace_bytes, void* stream);

/* moe_aux_loss_backward -- the gradient of grad_loss * loss (moe_aux_loss) with
 * respect to the logits, the counts held fixed (they come from the discrete
 * choice). With G_e = grad_loss * coeff * E * counts[e] / (k T^2):
 *   softmax: dlogits[t,i] = s[t,i] (G_i - sum_e s[t,e] G_e)
 *   sigmoid: dlogits[t,i] = G_i s[t,i] (1 - s[t,i])
 *  grad_loss  in  fp32 [1] on the device (NULL: 1)
 *  dlogits    out fp32 [T, E]; accumulate != 0 adds to it (for example to the
 *             router's own gradient from moe_router_backward), 0 overwrites.
 * Other arguments as in moe_aux_loss. */
moe_status moe_aux_loss_backward(const float* logits, int64_t T, int E, int k, int score_fn,
                                 const int32_t* counts, float coeff, const float* grad_loss,
                                 float* dlogits, int accumulate, void* stream);

/* moe_router_topk_noalloc -- the same routing as moe_router_topk, with no
 * workspace argument: for callers that cannot allocate device memory when they
 * route, such as a runtime that hands out all device memory from its own
 * pool before serving starts, or code running where allocation is forbidden.
 * The pages have no counterpart to it; it is an interface of this library.
 * Its scratch is one fixed array inside the library (a little over 3 MiB), which
 * every GPU that loads the library keeps until the process exits. It is
 * therefore limited to T <= MOE_NOALLOC_MAX_TOKENS and
 * T * k <= MOE_NOALLOC_MAX_ASSIGNMENTS; larger sizes return
 * MOE_ERR_UNSUPPORTED before anything is launched. Calls allocate nothing and
 * share that one array: two calls whose kernels overlap on the GPU (for
 * example on different streams without ordering) race and may return wrong
 * results. Calls that are ordered on one stream are safe. The first call on
 * a device looks up the array's device address and keeps it; make that first
 * call before any stream capture. If the lookup fails, the call returns
 * MOE_ERR_CUDA, nothing is kept, and the next call looks it up again.
 * Arguments, outputs and errors are otherwise those of moe_router_topk. */
#define MOE_NOALLOC_MAX_TOKENS 32768
#define MOE_NOALLOC_MAX_ASSIGNMENTS 262144
moe_status moe_router_topk_noalloc(const float* logits, int64_t T, int E, int k,
                                   const moe_router_opts* opts, int32_t* topk_idx,
                                   float* topk_prob, uint8_t* routing_map, int32_t* counts,
                                   int32_t* offsets, void* stream);

/* ----------------------------------------------------------------- dispatch
 * moe_permute -- TE Token dispatch: the rows of all tokens routed to the same
 * expert are stored back to back, in expert order. Inside an expert block,
 * rows are in ascending token order: the assignment (t, j) with
 * e = topk_idx[t, j] goes to row offsets[e] + #{t' < t routed to e}.
 *  x            in  bf16 [T, H]
 *  topk_idx     in  int32 [T, k]  (from moe_router_topk)
 *  offsets      in  int32 [E+1]   (from moe_router_topk)
 *  x_perm       out bf16 [T*k, H] expert-contiguous copy of the routed rows
 *  sorted_token out int32 [T*k]   token of each permuted row
 *  row_of       out int32 [T, k]  permuted row of each assignment (the map
 *                                 that combine uses to restore token order)
 *  workspace    scratch of moe_permute_workspace_size(T, E, k) bytes */
size_t moe_permute_workspace_size(int64_t T, int E, int k);
moe_status moe_permute(const moe_bf16* x, int64_t T, int H, const int32_t* topk_idx, int k,
                       const int32_t* offsets, int E, moe_bf16* x_perm, int32_t* sorted_token,
                       int32_t* row_of, void* workspace, size_t workspace_bytes, void* stream);

/* moe_permute_padded -- TE Token permutation, Padding and alignment
 * (moe_permute_and_pad_with_probs): the dispatch of moe_permute with each
 * expert's block rounded up to a multiple of align rows, for grouped GEMM
 * back ends that want aligned blocks. An empty block stays empty; the tokens
 * keep their moe_permute order inside a block, and the rows past an expert's
 * tokens are padding:
 *   padded_offsets[e+1] = padded_offsets[e] + align * ceil(counts[e] / align)
 *   assignment (t, j), e = topk_idx[t,j]: row padded_offsets[e] + #{t' < t routed to e}
 * Pad rows are zeros in x_perm, -1 in sorted_token and 0 in prob_perm. The
 * combine needs no padding information: row_of points at the real rows.
 *  x, topk_idx, k, E       as in moe_permute
 *  offsets         in  int32 [E+1]  unpadded, from moe_router_topk
 *  topk_prob       in  fp32 [T, k]  (needed only with prob_perm)
 *  align           in  1 .. 65536
 *  padded_offsets  out int32 [E+1]
 *  x_perm          out bf16 [R, H]  R = moe_permute_padded_max_rows(T, E, k, align)
 *                      = T*k + E*(align-1), the bound that needs no host sync;
 *                      rows past padded_offsets[E] are untouched
 *  prob_perm       out fp32 [R]     routing weight of each row (NULL: skip);
 *                      the weights for moe_grouped_mlp_scaled
 *  sorted_token    out int32 [R]
 *  row_of          out int32 [T, k]
 *  workspace       moe_permute_workspace_size(T, E, k) bytes */
int64_t moe_permute_padded_max_rows(int64_t T, int E, int k, int align);
moe_status moe_permute_padded(const moe_bf16* x, int64_t T, int H, const int32_t* topk_idx,
                              const float* topk_prob, int k, const int32_t* offsets, int E, int align,
                              int32_t* padded_offsets, moe_bf16* x_perm, float* prob_perm,
                              int32_t* sorted_token, int32_t* row_of, void* workspace,
                              size_t workspace_bytes, void* stream);

/* -------------------------------------------------------------- grouped MLP
 * moe_grouped_mlp -- TE Grouped GEMM (Y_i = X_i W_i^T per expert block,
 * Y = concat(Y_i)) and Grouped MLP (FC1 with the activation fused, then FC2).
 * For the rows r of expert e, [offsets[e], offsets[e+1]):
 *   g = x_perm[r] . w_gate_up[e][:, 0:I]   u = x_perm[r] . w_gate_up[e][:, I:2I]
 *   h[r] = bf16(silu(g) * u)               y_perm[r] = bf16(h[r] . w_down[e])
 * in fp32 accumulation. Experts may have any number of rows, zero included.
 *  x_perm       in  bf16 [A, H]
 *  offsets      in  int32 [E+1]   offsets[E] <= A; rows past offsets[E] untouched
 *  w_gate_up    in  bf16 [E, H, 2I]  (gate columns first, then up)
 *  w_down       in  bf16 [E, I, H]
 *  y_perm       out bf16 [A, H]
 *  gu_save      out bf16 [A, 2I]  g and u, kept for the backward (NULL: skip)
 *  h_save       out bf16 [A, I]   h (NULL: h goes to the workspace)
 *  workspace    moe_grouped_mlp_workspace_size(A, E, H, I) bytes; 0 when
 *               h_save is given */
size_t moe_grouped_mlp_workspace_size(int64_t A, int E, int H, int I);
moe_status moe_grouped_mlp(const moe_bf16* x_perm, int64_t A, const int32_t* offsets, int E,
                           int H, int I, const moe_bf16* w_gate_up, const moe_bf16* w_down,
                           moe_bf16* y_perm, moe_bf16* gu_save, moe_bf16* h_save,
                           void* workspace, size_t workspace_bytes, void* stream);

/* moe_grouped_mlp_scaled -- TE Grouped MLP with ScaledSwiGLU: moe_grouped_mlp
 * with the routing weight of each row applied to the activation before FC2,
 *   h[r] = bf16(silu(g) * u * row_scale[r]),  y_perm[r] = bf16(h[r] . w_down[e]),
 * so y_perm is already weighted ((p h) W2 = p (h W2), the page's identity for
 * FC2 without bias) and moe_unpermute_combine must then run with topk_prob
 * NULL. gu_save keeps the unscaled g and u. row_scale fp32 [A] (for example
 * moe_permute_padded's prob_perm; NULL: 1). moe_grouped_mlp_scaled_backward
 * is its backward. Other arguments as in moe_grouped_mlp. */
moe_status moe_grouped_mlp_scaled(const moe_bf16* x_perm, int64_t A, const int32_t* offsets, int E,
                                  int H, int I, const moe_bf16* w_gate_up, const moe_bf16* w_down,
                                  const float* row_scale, moe_bf16* y_perm, moe_bf16* gu_save,
                                  moe_bf16* h_save, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ combine
 * moe_unpermute_combine -- TE Token combine with merging_probs:
 *   out[t] = bf16( shared_out[t] + sum_{j<k} topk_prob[t,j] * y_perm[row_of[t,j]] )
 * summed in fp32, j ascending. Each output row has one writer, so the result
 * is deterministic. topk_prob NULL sums the rows unweighted. shared_out NULL
 * means no shared expert. The routing weights must be applied exactly once (TE
 * Token probabilities): pass NULL here if y_perm is already weighted.
 *  y_perm in bf16 [A, H]; row_of in int32 [T, k]; topk_prob in fp32 [T, k];
 *  shared_out in bf16 [T, H]; out out bf16 [T, H]. */
moe_status moe_unpermute_combine(const moe_bf16* y_perm, const int32_t* row_of,
                                 const float* topk_prob, int64_t T, int k, int H,
                                 const moe_bf16* shared_out, moe_bf16* out, void* stream);

/* moe_unpermute_combine_rows -- moe_unpermute_combine for a y_perm of y_rows
 * rows, such as the output of a padded dispatch (moe_permute_padded: rows
 * T*k + E*(align-1) at most, with row_of pointing at the real rows, so the pad
 * rows are never read). moe_unpermute_combine is this call with
 * y_rows = T*k. A row_of entry outside [0, y_rows) is recorded as
 * MOE_ERR_DEVICE_CHECK and skipped. */
moe_status moe_unpermute_combine_rows(const moe_bf16* y_perm, int64_t y_rows, const int32_t* row_of,
                                      const float* topk_prob, int64_t T, int k, int H,
                                      const moe_bf16* shared_out, moe_bf16* out, void* stream);

/* ------------------------------------------------------------ fused layer
 * moe_layer_forward -- the four stages on one stream (TE "Example: MoE layer
 * on a single device"):
 *   out[t] = shared(x[t]) + sum_j p[t,j] * MLP_{e[t,j]}(x[t])
 * shared_gate_up [H, 2I] and shared_down [I, H] are the dense SwiGLU shared
 * expert (torchtitan MoE.forward adds it to the routed output); pass NULL for
 * none. The optional outputs below keep the forward state for
 * moe_grouped_mlp_backward. Each may be NULL, in which case it lives in the
 * workspace: topk_idx [T,k], topk_prob [T,k], counts [E], offsets [E+1],
 * row_of [T,k], x_perm [A,H], gu [A,2I] (NULL: not computed), h [A,I],
 * y_perm [A,H].
 * With the folded permute forced (moe_testing_set_kernels, fold_permute = 1),
 * x_perm NULL and single-CTA GEMM tiles (experts averaging under 1024 rows, at
 * least 16), the permutation is folded into the
 * gate_up GEMM (TE Token permutation): its A rows are gathered from x by token,
 * and no permuted copy of x is written (x_perm in the workspace is left
 * unwritten). The result is bit-identical to the default path, which
 * measures faster on B200.
 * With a shared expert whose GEMMs run on CTA-pair tiles (T > 16), the
 * combine is done in the shared expert's down GEMM epilogue: each output row
 * (one token) is the shared expert's fp32 result plus its k routed rows,
 * weighted, j ascending, rounded to bf16 once (TE Token combine; the shared
 * expert's output is then not stored as bf16 before the sum). Otherwise the
 * combine kernel adds the stored bf16 shared output.
 * For one token block (T <= 8) the router kernel also writes the counts and
 * offsets, and, when the permuted rows take at most 64 KB, the rows
 * themselves (no scan or permute launch).
 * With at most T <= 64 rows per expert on swap-AB tiles, where the experts
 * that can hold rows (min(E, T k)) have at least one gate_up tile (64 columns
 * of h) per SM, the gate_up and down GEMMs run as one launch: a down tile
 * loads its weights first and waits (bounded) on a device counter until its
 * expert's h is stored. The results are bit-identical to two launches.
 * The call records no device-to-host copy and no host synchronisation, so it
 * can be captured in a CUDA graph. */
size_t moe_layer_forward_workspace_size(int64_t T, int H, int I, int E, int k, int has_shared);
moe_status moe_layer_forward(const float* logits, const moe_bf16* x, int64_t T, int H, int I,
                             int E, int k, const moe_router_opts* opts,
                             const moe_bf16* w_gate_up, const moe_bf16* w_down,
                             const moe_bf16* shared_gate_up, const moe_bf16* shared_down,
                             moe_bf16* out, int32_t* topk_idx, float* topk_prob, int32_t* counts,
                             int32_t* offsets, int32_t* row_of, moe_bf16* x_perm, moe_bf16* gu,
                             moe_bf16* h, moe_bf16* y_perm, void* workspace,
                             size_t workspace_bytes, void* stream);

/* ----------------------------------------------------------------- backward
 * moe_grouped_mlp_backward -- gradients of out[t] = sum_j p[t,j] MLP_e(x[t])
 * with respect to x, w_gate_up, w_down and the routing weights p (TE Example:
 * every stage is differentiable; the logits do not receive a gradient here):
 *   dprob[t,j] = <dout[t], y_perm[row]>           dy[row] = p[t,j] * dout[t]
 *   dh = dy . w_down[e]^T     du = dh * silu(g)    dg = dh * u * silu'(g)
 *   dx_perm = [dg | du] . w_gate_up[e]^T           dx[t] = sum_j dx_perm[row_of[t,j]]
 *   dw_down[e] = h_e^T . dy_e                      dw_gate_up[e] = x_e^T . [dg | du]_e
 * with row = row_of[t,j] and the forward state saved by moe_layer_forward
 * (gu must have been saved). Accumulation is fp32. An expert with no rows
 * gets zero weight gradients.
 *  dout in bf16 [T,H]; dx out bf16 [T,H]; dw_gate_up out bf16 [E,H,2I];
 *  dw_down out bf16 [E,I,H]; dprob out fp32 [T,k];
 *  workspace of moe_grouped_mlp_backward_workspace_size(T, H, I, E, k) bytes. */
size_t moe_grouped_mlp_backward_workspace_size(int64_t T, int H, int I, int E, int k);
moe_status moe_grouped_mlp_backward(const moe_bf16* dout, int64_t T, int H, int I, int E, int k,
                                    const moe_bf16* w_gate_up, const moe_bf16* w_down,
                                    const int32_t* row_of, const float* topk_prob,
                                    const int32_t* offsets, const moe_bf16* x_perm,
                                    const moe_bf16* gu, const moe_bf16* h, const moe_bf16* y_perm,
                                    moe_bf16* dx, moe_bf16* dw_gate_up, moe_bf16* dw_down,
                                    float* dprob, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* moe_grouped_mlp_scaled_backward -- gradients of the ScaledSwiGLU layer (TE
 * Grouped MLP, the routing weight applied to the activation before FC2):
 *   out[t] = sum_j y_perm[row_of[t,j]],  y_perm[r] = bf16(p_r silu(g_r) u_r) . w_down[e]
 * i.e. moe_grouped_mlp_scaled followed by moe_unpermute_combine with
 * topk_prob NULL, with respect to x, w_gate_up, w_down and p:
 *   dy[r] = dout[t]   (r = row_of[t,j]; a pad row: 0)
 *   dh = dy . w_down[e]^T          dprob[t,j] = <dh, silu(g) * u>   (row r)
 *   ds = p_r * dh                  du = ds * silu(g)    dg = ds * u * silu'(g)
 *   dx_perm = [dg | du] . w_gate_up[e]^T       dx[t] = sum_j dx_perm[row_of[t,j]]
 *   dw_down[e] = h_e^T . dy_e                  dw_gate_up[e] = x_e^T . [dg | du]_e
 * The rows are those of the forward's dispatch, padded (moe_permute_padded)
 * or not (moe_permute), A of them with offsets (padded_offsets) [E+1].
 * Accumulation is fp32; dprob sums each 64-column group of dh * silu(g) * u
 * in column order, then the groups in order, so it is the same on every run.
 * An expert with no rows gets zero weight gradients.
 *  dout          in  bf16 [T,H]
 *  row_of        in  int32 [T,k]   row of each assignment
 *  sorted_token  in  int32 [A]     token of each row, -1 for a pad row
 *  row_scale     in  fp32 [A]      p of each row (prob_perm; 0 on pad rows)
 *  x_perm        in  bf16 [A,H]    the forward's rows (pad rows zero)
 *  gu            in  bf16 [A,2I]   the forward's unscaled g and u (gu_save)
 *  h             in  bf16 [A,I]    the forward's scaled h (h_save)
 *  dx out bf16 [T,H]; dw_gate_up out bf16 [E,H,2I]; dw_down out bf16 [E,I,H];
 *  dprob out fp32 [T,k], the gradient of the routing weights (it reaches the
 *  logits through the router's softmax or sigmoid, which is not done here);
 *  workspace of moe_grouped_mlp_scaled_backward_workspace_size(A, H, I) bytes.
 * A row index or token outside its range is recorded as MOE_ERR_DEVICE_CHECK. */
size_t moe_grouped_mlp_scaled_backward_workspace_size(int64_t A, int H, int I);
moe_status moe_grouped_mlp_scaled_backward(const moe_bf16* dout, int64_t T, int H, int I, int E, int k,
                                           const moe_bf16* w_gate_up, const moe_bf16* w_down,
                                           const int32_t* row_of, const int32_t* sorted_token,
                                           const float* row_scale, const int32_t* offsets, int64_t A,
                                           const moe_bf16* x_perm, const moe_bf16* gu, const moe_bf16* h,
                                           moe_bf16* dx, moe_bf16* dw_gate_up, moe_bf16* dw_down,
                                           float* dprob, void* workspace, size_t workspace_bytes,
                                           void* stream);

/* ------------------------------------------------------------ testing hooks
 * moe_testing_set_kernels -- forces one kernel variant for every later call in
 * this process, so that tests can run each variant on the same inputs. It is
 * not an operation of the pages. The variants compute identical results (the
 * tests compare them bit for bit, or against the oracle) and differ only in
 * speed; by default (MOE_TESTING_AUTO everywhere) the library chooses by the
 * shapes alone.
 *  gemm_tiles    group-M GEMMs on single-CTA 128-row tiles or CTA-pair tiles;
 *                or the forward GEMMs on swap-AB tiles (weights as the 128-row
 *                operand, 64 token rows per tile; the backward GEMMs then take
 *                single-CTA tiles); SWAP_UNFUSED: swap-AB tiles with the
 *                layer's gate_up and down GEMMs as two launches even where
 *                every expert holds at most 64 rows (by default one launch
 *                then computes both)
 *  router        the warp-per-token or the lane-per-token router kernel (the
 *                lane kernel where it applies: E a multiple of 32, k <= 8,
 *                renormalised softmax or sigmoid)
 *  permute       the token-range (rows up to 4096 wide) or the warp-per-token
 *                permute kernel
 *  fold_permute  1: moe_layer_forward without a requested x_perm gathers the
 *                gate_up GEMM's A rows from x by token id (single-CTA tiles),
 *                so the permuted copy of x is never written; it measures
 *                slower on B200 than TMA tiles of x_perm
 * Returns MOE_ERR_INVALID_ARG for a value out of range. Not synchronised with
 * calls issued from other threads. */
#define MOE_TESTING_AUTO 0
#define MOE_TESTING_GEMM_SINGLE 1
#define MOE_TESTING_GEMM_PAIR 2
#define MOE_TESTING_GEMM_SWAP 3
#define MOE_TESTING_GEMM_SWAP_UNFUSED 4
#define MOE_TESTING_ROUTER_WARP 1
#define MOE_TESTING_ROUTER_LANE 2
#define MOE_TESTING_PERMUTE_TOKENS 1
#define MOE_TESTING_PERMUTE_WARP 2
moe_status moe_testing_set_kernels(int gemm_tiles, int router, int permute, int fold_permute);

/* moe_testing_wait_timeout -- launches one block whose thread waits, with the
 * same bounded wait as the GEMM kernels' pipeline barriers but a limit of
 * limit_ns nanoseconds (1 .. 1e9), on a shared-memory barrier that nothing
 * arrives on. The wait runs out, the kernel records MOE_ERR_TIMEOUT in the
 * device error word and returns, so the next moe_get_device_status returns
 * MOE_ERR_TIMEOUT (and clears it) and the context stays usable. It tests
 * failure detection without a GPU fault; it is not an operation of the pages.
 * Returns MOE_ERR_INVALID_ARG for a limit out of range. */
moe_status moe_testing_wait_timeout(int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
