// moe_internal.h -- launchers shared between the kernel files and the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

using bf16 = __nv_bfloat16;

// Whether the kernels that this host thread launches for its current call are
// chained (programmatic dependent launch). Chaining hides each kernel's launch
// and prologue behind the end of the kernel before it, which pays in calls of
// a few rows, where those fixed costs are most of the time (measured on B200:
// a one-token layer forward 60 -> 49 us). In large calls it cost 2.5-4 %, so
// the entry points turn it on by the call's size (ChainScope, kChainMaxRows).
bool& chained_launches();   // thread-local, moe_api.cu
constexpr int64_t kChainMaxRows = 4096;
struct ChainScope {
    bool prev;
    explicit ChainScope(bool on) : prev(chained_launches()) { chained_launches() = on; }
    ~ChainScope() { chained_launches() = prev; }
};

// Launches a kernel of a layer call, chained when chained_launches() says so:
// it may then be scheduled before the previous kernel in the stream has
// finished, and it calls pdl_wait() (moe_common.cuh) before it touches data
// that other kernels write or read (without a chain pdl_wait returns at once).
template <class... KArgs, class... Args>
cudaError_t launch_chained(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                           Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = chained_launches() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Tokens handled by one block of the router / rank kernels (a power of two,
// 8..64). Ranks inside an expert block are counted per such token block, then
// offset by a scan. Small batches use small token blocks so that every SM gets
// work; large ones use 64 to keep the per-block counts ([E][blocks]) small.
constexpr int kMaxTokensPerRouteBlock = 64;

inline int route_tokens_per_block(int64_t T) {
    if (T <= 8192) return 8;
    if (T <= 32768) return 16;
    if (T <= 131072) return 32;
    return 64;
}

inline int64_t route_blocks(int64_t T) {
    const int tpb = route_tokens_per_block(T);
    return (T + tpb - 1) / tpb;
}

// Scratch of the routing path, carved from the caller's workspace.
struct RouteScratch {
    int32_t* block_base;  // [E][nb]: per-(expert, token block) counts, then exclusive prefix
    int32_t* local_rank;  // [T][k]: rank of the assignment inside its token block
    unsigned* ticket;     // last-block-done counter of the scan kernel
};
size_t route_scratch_bytes(int64_t T, int E, int k);
RouteScratch carve_route_scratch(void* base, int64_t T, int E, int k);

// With counts and offsets given and a single token block (T <= 8 tokens), the
// router also writes the counts and offsets and sets *scanned; otherwise
// launch_expert_scan must follow. Whichever writes the offsets also sets
// zero[0 .. n_zero) to 0 (the fused expert MLP's schedule counters; NULL: none).
// When the router writes them, x, x_perm, sorted_token, row_of and permuted
// are given and the permuted rows take at most 64 KB, it also does the permute
// (x [T][H] into x_perm [T k][H]) and sets *permuted; otherwise
// launch_permute must follow.
cudaError_t launch_router_topk(const float* logits, int64_t T, int E, int k,
                               const moe_router_opts& opts, int32_t* topk_idx, float* topk_prob,
                               uint8_t* routing_map, const RouteScratch& rs, cudaStream_t st,
                               unsigned* err, int32_t* counts = nullptr, int32_t* offsets = nullptr,
                               bool* scanned = nullptr, int32_t* zero = nullptr, int n_zero = 0,
                               const bf16* x = nullptr, int H = 0, bf16* x_perm = nullptr,
                               int32_t* sorted_token = nullptr, int32_t* row_of = nullptr, bool* permuted = nullptr);
cudaError_t launch_router_backward(const float* logits, int64_t T, int E, int k, const moe_router_opts& opts,
                                   const int32_t* topk_idx, const float* dprob, float* dlogits,
                                   cudaStream_t st, unsigned* err);
cudaError_t launch_expert_bias_update(const int32_t* counts, int E, float coeff, float* bias, cudaStream_t st);

// Auxiliary load-balancing loss (aux_loss.cu).
size_t aux_loss_workspace_bytes(int64_t T, int E);
cudaError_t launch_aux_loss(const float* logits, int64_t T, int E, int k, int score_fn, const int32_t* counts,
                            float coeff, float* loss, float* scores, void* ws, cudaStream_t st);
cudaError_t launch_aux_loss_backward(const float* logits, int64_t T, int E, int k, int score_fn,
                                     const int32_t* counts, float coeff, const float* grad_loss, float* dlogits,
                                     int accumulate, cudaStream_t st);
cudaError_t launch_rank_from_indices(const int32_t* topk_idx, int64_t T, int E, int k,
                                     const RouteScratch& rs, cudaStream_t st, unsigned* err);
// Turns block counts into exclusive prefixes; writes counts/offsets if given,
// and then sets zero[0 .. n_zero) to 0 (NULL: none).
cudaError_t launch_expert_scan(int64_t T, int E, const RouteScratch& rs, int32_t* counts,
                               int32_t* offsets, cudaStream_t st, int32_t* zero = nullptr, int n_zero = 0);
// Padded dispatch (Token permutation, Padding and alignment).
cudaError_t launch_pad_offsets(const int32_t* offsets, int E, int align, int32_t* padded_offsets, cudaStream_t st);
cudaError_t launch_pad_fill(const int32_t* offsets, const int32_t* padded_offsets, int E, int H, bf16* x_perm,
                            int32_t* sorted_token, float* prob_perm, cudaStream_t st);
cudaError_t launch_prob_perm(const float* topk_prob, const int32_t* row_of, int64_t n, float* prob_perm,
                             cudaStream_t st);
// row_bound: rows of x_perm and sorted_token (<= 0: T*k, the unpadded dispatch)
cudaError_t launch_permute(const bf16* x, int64_t T, int H, const int32_t* topk_idx, int k,
                           const int32_t* offsets, int E, const RouteScratch& rs, bf16* x_perm,
                           int32_t* sorted_token, int32_t* row_of, cudaStream_t st, unsigned* err,
                           int64_t row_bound = 0);

// The fixed scratch array behind moe_router_topk_noalloc (routing.cu).
size_t router_noalloc_capacity();
cudaError_t router_noalloc_scratch(void** ptr);

cudaError_t launch_combine(const bf16* y_perm, const int32_t* row_of, const float* probs,
                           int64_t T, int k, int H, int64_t A, const bf16* shared, bf16* out,
                           cudaStream_t st, unsigned* err);
cudaError_t launch_combine_backward(const bf16* dout, const bf16* y_perm, const int32_t* row_of,
                                    const float* probs, int64_t T, int k, int H, int64_t A,
                                    bf16* dy_perm, float* dprob, cudaStream_t st, unsigned* err);
// dy[r] = dout[sorted_token[r]] for r < offsets[E] (-1: a zero row).
cudaError_t launch_gather_rows(const bf16* dout, const int32_t* sorted_token, int64_t T, const int32_t* offsets,
                               int E, int64_t A, int H, bf16* dy, cudaStream_t st, unsigned* err);
// dprob[i] = sum_{q < nq} row_dot[row_of[i] * nq + q], q ascending.
cudaError_t launch_row_dot_sum(const float* row_dot, int nq, const int32_t* row_of, int64_t n, int64_t A,
                               float* dprob, cudaStream_t st, unsigned* err);

// ---------------------------------------------------------------- GEMMs
// Grouped GEMMs on tcgen05. Each returns cudaErrorInvalidValue if a tensor
// map cannot be encoded (bad alignment or extent).
// gate_up + SwiGLU: h[r] = silu(x[r] Wg[e]) * (x[r] Wu[e]); optionally gu[r] = [g | u].
// offsets NULL: one group of `rows` rows using the weights of group 0.
// max_group_rows: an upper bound on the rows of any group (0: rows), which
// lets small batches take narrower swap-AB tiles (a layer call passes T: a
// token is routed to an expert at most once).
cudaError_t gemm_gate_up_swiglu(const bf16* x, int64_t rows, const int32_t* offsets, int E, int H,
                                int I, const bf16* w_gate_up, bf16* h, bf16* gu_save,
                                cudaStream_t st, unsigned* err, const float* row_scale = nullptr,
                                int64_t max_group_rows = 0);
// gate_up + SwiGLU with A row r gathered from x: row sorted_token[r] (-1: a
// zero row) of x [T][H], so no permuted copy of x is needed. Single-CTA tiles
// only; H a multiple of 8 and x 16-byte aligned.
cudaError_t gemm_gate_up_swiglu_gather(const bf16* x, int64_t T, const int32_t* sorted_token, int64_t rows,
                                       const int32_t* offsets, int E, int H, int I, const bf16* w_gate_up, bf16* h,
                                       bf16* gu_save, cudaStream_t st, unsigned* err,
                                       const float* row_scale = nullptr);
// The expert MLP of a small batch in one launch (gemm_swap_mlp_kernel):
// h = SwiGLU(x W_gate_up) (and gu = [g | u] if gu_save), then y = h W_down,
// on swap-AB tiles. Every expert must hold at most max_group_rows <= 64 rows
// (a layer call passes T). sched: E + 1 int32 that are zero when the launch
// starts (the router or the scan zeroes them). use_fused_mlp says whether a
// call of this many rows, groups and columns of h takes it.
bool use_fused_mlp(int64_t rows, int groups, int64_t max_group_rows, int I);
cudaError_t gemm_expert_mlp_fused(const bf16* x, int64_t rows, const int32_t* offsets, int E, int H, int I,
                                  const bf16* w_gate_up, const bf16* w_down, bf16* h, bf16* gu_save, bf16* y,
                                  int32_t* sched, int64_t max_group_rows, cudaStream_t st, unsigned* err);
// Whether the forward gate_up GEMM runs on single-CTA 128-row tiles (not CTA
// pairs, not swap-AB tiles) for this many rows and groups.
bool grouped_gemm_single_tiles(int64_t rows, int groups);
// Whether a group-M GEMM of this many rows and groups runs on CTA-pair tiles.
bool grouped_gemm_pair_tiles(int64_t rows, int groups);
// The shared expert's down GEMM with the token combine folded into its
// epilogue: out[t] = bf16(h[t] Wd + sum_j probs[t,j] y_perm[row_of[t,j]]), the
// sum in fp32 after the product, j ascending. CTA-pair tiles only
// (cudaErrorNotSupported when grouped_gemm_pair_tiles(T, 1) is false).
cudaError_t gemm_down_combine(const bf16* h, int64_t T, int H, int I, const bf16* w_down, const bf16* y_perm,
                              int64_t y_rows, const int32_t* row_of, const float* probs, int k, bf16* out,
                              cudaStream_t st, unsigned* err);
// down: y[r] = h[r] Wd[e]
cudaError_t gemm_down(const bf16* h, int64_t rows, const int32_t* offsets, int E, int H, int I,
                      const bf16* w_down, bf16* y, cudaStream_t st, unsigned* err, int64_t max_group_rows = 0);
// dgrad of down with SwiGLU backward: dh = dy Wd[e]^T, then dgu = [dg | du].
// ScaledSwiGLU (row_dot non-NULL): the forward's h[r] was scaled by
// row_scale[r], so [dg | du] is taken from row_scale[r] * dh, and
// row_dot [rows][ceil(I/64)] gets each 64-column group's sum of
// dh * silu(g) * u (the routing weight's gradient, in parts).
cudaError_t gemm_down_dgrad_swiglu(const bf16* dy, int64_t rows, const int32_t* offsets, int E,
                                   int H, int I, const bf16* w_down, const bf16* gu, bf16* dgu,
                                   cudaStream_t st, unsigned* err, const float* row_scale = nullptr,
                                   float* row_dot = nullptr);
// dgrad of gate_up: dx_perm = dgu Wgu[e]^T
cudaError_t gemm_gate_up_dgrad(const bf16* dgu, int64_t rows, const int32_t* offsets, int E, int H,
                               int I, const bf16* w_gate_up, bf16* dx_perm, cudaStream_t st,
                               unsigned* err);
// wgrad: dW[e] = X_e^T D_e over the rows of group e (ragged reduction);
// X [rows, M], D [rows, N], dW [E, M, N]. Empty groups get dW[e] = 0.
cudaError_t gemm_wgrad(const bf16* X, const bf16* D, int64_t rows, const int32_t* offsets, int E,
                       int M, int N, bf16* dW, cudaStream_t st, unsigned* err);

int sm_count();

// Kernel variants forced by moe_testing_set_kernels (MOE_TESTING_AUTO: the
// library's own choice by shape).
struct KernelOverride {
    int gemm_tiles = MOE_TESTING_AUTO;
    int router = MOE_TESTING_AUTO;
    int permute = MOE_TESTING_AUTO;
    int fold_permute = 0;
};
const KernelOverride& kernel_override();

}  // namespace moe
