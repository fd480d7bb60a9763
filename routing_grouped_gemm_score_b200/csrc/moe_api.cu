// moe_api.cu -- the extern "C" entry points declared in include/moe_b200.h:
// argument checks (before any CUDA call), workspace layout, the device error
// word, and the stage order of the fused forward and of the backward.
#include <cstring>
#include <mutex>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

__device__ unsigned g_device_error;

constexpr int kMaxDevices = 64;

int current_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return -1;
    return d;
}

struct DeviceInfo {
    std::once_flag once;
    int sms = 148;
    unsigned* err = nullptr;
};
DeviceInfo g_info[kMaxDevices];

DeviceInfo* info() {
    const int d = current_device();
    if (d < 0 || d >= kMaxDevices) return nullptr;
    DeviceInfo* di = &g_info[d];
    std::call_once(di->once, [di, d] {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d) == cudaSuccess && sms > 0)
            di->sms = sms;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess)
            di->err = static_cast<unsigned*>(p);
    });
    return di;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Stage tracing (moe_trace_set): caller-owned events recorded at stage ends.
constexpr int kMaxTraceEvents = 16;
cudaEvent_t g_trace[kMaxTraceEvents];
int g_trace_n = 0;

cudaError_t trace_mark(int i, cudaStream_t st) {
    if (i >= g_trace_n) return cudaSuccess;
    return cudaEventRecord(g_trace[i], st);
}

// Bump allocator over the caller's workspace; every piece is 256-byte aligned.
struct Carver {
    char* base;
    size_t used = 0;
    explicit Carver(void* b) : base(static_cast<char*>(b)) {}
    template <class T>
    T* take(size_t count) {
        used = (used + 255) & ~size_t(255);
        T* p = reinterpret_cast<T*>(base ? base + used : nullptr);
        used += count * sizeof(T);
        return p;
    }
    size_t bytes() const { return (used + 255) & ~size_t(255); }
};

bool shape_ok(int64_t T, int E, int k) {
    return T >= 0 && E >= 1 && E <= 256 && k >= 1 && k <= 16 && k <= E &&
           T * (int64_t)k < (int64_t(1) << 31);
}

// H and I multiples of 8: 16-byte rows, the stride rule of the TMA maps and of
// the 16-byte vector loads and stores (pytorch/ao pull request 2600, the
// alignment of grouped-GEMM operands).
bool dims_ok(int H, int I) { return H > 0 && I > 0 && H % 8 == 0 && I % 8 == 0; }

moe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe_router_opts default_opts() {
    moe_router_opts o;
    o.score_fn = MOE_SCORE_SOFTMAX;
    o.renormalize = 1;
    o.scaling = 1.0f;
    o.expert_bias = nullptr;
    return o;
}

moe_status check_opts(const moe_router_opts& o) {
    if (o.score_fn != MOE_SCORE_SOFTMAX && o.score_fn != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (o.expert_bias && o.score_fn != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (!(o.scaling == o.scaling)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// Layout of the fused forward's workspace. Pieces the caller supplies are
// still reserved, so the size depends on the shape only.
struct FwdLayout {
    RouteScratch rs;
    int32_t *topk_idx, *counts, *offsets, *row_of, *sorted_token;
    int32_t* sched;   // [E + 1]: the fused small-batch MLP's tile counter and per-expert h counts
    float* topk_prob;
    bf16 *x_perm, *h, *y_perm, *shared_h, *shared_out;
    size_t bytes;
};

FwdLayout fwd_layout(void* ws, int64_t T, int H, int I, int E, int k, int has_shared) {
    const int64_t A = T * k;
    Carver c(ws);
    FwdLayout L;
    char* route = c.take<char>(route_scratch_bytes(T, E, k));
    L.rs = carve_route_scratch(route, T, E, k);
    L.topk_idx = c.take<int32_t>((size_t)A);
    L.topk_prob = c.take<float>((size_t)A);
    L.counts = c.take<int32_t>((size_t)E);
    L.offsets = c.take<int32_t>((size_t)E + 1);
    L.sched = c.take<int32_t>((size_t)E + 1);
    L.row_of = c.take<int32_t>((size_t)A);
    L.sorted_token = c.take<int32_t>((size_t)A);
    L.x_perm = c.take<bf16>((size_t)A * H);
    L.h = c.take<bf16>((size_t)A * I);
    L.y_perm = c.take<bf16>((size_t)A * H);
    L.shared_h = has_shared ? c.take<bf16>((size_t)T * I) : nullptr;
    L.shared_out = has_shared ? c.take<bf16>((size_t)T * H) : nullptr;
    L.bytes = c.bytes();
    return L;
}

struct BwdLayout {
    bf16 *dy, *dgu, *dx_perm;
    size_t bytes;
};

BwdLayout bwd_layout(void* ws, int64_t T, int H, int I, int k) {
    const int64_t A = T * k;
    Carver c(ws);
    BwdLayout L;
    L.dy = c.take<bf16>((size_t)A * H);
    L.dgu = c.take<bf16>((size_t)A * 2 * I);
    L.dx_perm = c.take<bf16>((size_t)A * H);
    L.bytes = c.bytes();
    return L;
}

struct ScaledBwdLayout {
    bf16 *dy, *dgu, *dx_perm;
    float* row_dot;
    size_t bytes;
};

ScaledBwdLayout scaled_bwd_layout(void* ws, int64_t A, int H, int I) {
    Carver c(ws);
    ScaledBwdLayout L;
    L.dy = c.take<bf16>((size_t)A * H);
    L.dgu = c.take<bf16>((size_t)A * 2 * I);
    L.dx_perm = c.take<bf16>((size_t)A * H);
    L.row_dot = c.take<float>((size_t)A * ((I + 63) / 64));
    L.bytes = c.bytes();
    return L;
}

}  // namespace

unsigned* device_error_word() {
    DeviceInfo* di = info();
    return di ? di->err : nullptr;
}

int sm_count() {
    DeviceInfo* di = info();
    return di ? di->sms : 148;
}

KernelOverride g_override;

bool& chained_launches() {
    thread_local bool on = false;
    return on;
}

// One thread waits, with the given limit, on an mbarrier that nothing arrives
// on: the bounded wait of the GEMM kernels (mbar_wait_limit) running out.
// It records kErrTimeout in the device error word and returns.
__global__ void wait_on_nothing_kernel(unsigned long long limit_ns, unsigned* err) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, &abort_flag, err, limit_ns);
    __syncthreads();
}

const KernelOverride& kernel_override() { return g_override; }

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape outside the kernels' limits";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or launch failed";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace too small or missing";
        case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK: a kernel found invalid routing data";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a kernel gave up on a bounded wait";
    }
    return "unknown moe_status";
}

moe_status moe_get_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (v) {
        const unsigned zero = 0;
        if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    if (v & kErrTimeout) return MOE_ERR_TIMEOUT;
    if (v & kErrDeviceCheck) return MOE_ERR_DEVICE_CHECK;
    return MOE_OK;
}

moe_status moe_testing_set_kernels(int gemm_tiles, int router, int permute, int fold_permute) {
    if (gemm_tiles < 0 || gemm_tiles > 4 || router < 0 || router > 2 || permute < 0 || permute > 2 ||
        fold_permute < 0 || fold_permute > 1)
        return MOE_ERR_INVALID_ARG;
    moe::g_override.gemm_tiles = gemm_tiles;
    moe::g_override.router = router;
    moe::g_override.permute = permute;
    moe::g_override.fold_permute = fold_permute;
    return MOE_OK;
}

moe_status moe_testing_wait_timeout(int64_t limit_ns, void* stream) {
    if (limit_ns <= 0 || limit_ns > 1000000000) return MOE_ERR_INVALID_ARG;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    moe::wait_on_nothing_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)limit_ns, err);
    return from_cuda(cudaGetLastError());
}

moe_status moe_trace_set(void* const* events, int n_events) {
    if (n_events < 0) return MOE_ERR_INVALID_ARG;
    if (!events) n_events = 0;
    if (n_events > kMaxTraceEvents) n_events = kMaxTraceEvents;
    for (int i = 0; i < n_events; ++i) g_trace[i] = static_cast<cudaEvent_t>(events[i]);
    g_trace_n = n_events;
    return MOE_OK;
}

size_t moe_router_workspace_size(int64_t T, int E, int k) {
    if (!shape_ok(T, E, k)) return 0;
    return route_scratch_bytes(T, E, k);
}

moe_status moe_router_topk(const float* logits, int64_t T, int E, int k,
                           const moe_router_opts* opts_in, int32_t* topk_idx, float* topk_prob,
                           uint8_t* routing_map, int32_t* counts, int32_t* offsets,
                           void* workspace, size_t workspace_bytes, void* stream) {
    const ChainScope chain(T * (int64_t)k <= kChainMaxRows);
    if (!shape_ok(T, E, k)) return MOE_ERR_INVALID_ARG;
    const moe_router_opts opts = opts_in ? *opts_in : default_opts();
    if (check_opts(opts) != MOE_OK) return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets || !aligned16(counts) || !aligned16(offsets)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !topk_idx || !topk_prob || !aligned16(logits) ||
                  !aligned16(topk_idx) || !aligned16(topk_prob)))
        return MOE_ERR_INVALID_ARG;
    if (opts.expert_bias && !aligned16(opts.expert_bias)) return MOE_ERR_INVALID_ARG;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st) != cudaSuccess) return MOE_ERR_CUDA;
        return from_cuda(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st));
    }
    if (!workspace || workspace_bytes < route_scratch_bytes(T, E, k)) return MOE_ERR_WORKSPACE;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const RouteScratch rs = carve_route_scratch(workspace, T, E, k);
    bool scanned = false;
    cudaError_t e = launch_router_topk(logits, T, E, k, opts, topk_idx, topk_prob, routing_map, rs,
                                       st, err, counts, offsets, &scanned);
    if (e == cudaSuccess && !scanned) e = launch_expert_scan(T, E, rs, counts, offsets, st);
    return from_cuda(e);
}

moe_status moe_router_backward(const float* logits, int64_t T, int E, int k,
                               const moe_router_opts* opts_in, const int32_t* topk_idx,
                               const float* dprob, float* dlogits, void* stream) {
    if (!shape_ok(T, E, k)) return MOE_ERR_INVALID_ARG;
    const moe_router_opts opts = opts_in ? *opts_in : default_opts();
    if (check_opts(opts) != MOE_OK) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !topk_idx || !dprob || !dlogits || !aligned16(logits) ||
                  !aligned16(topk_idx) || !aligned16(dprob) || !aligned16(dlogits)))
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    return from_cuda(launch_router_backward(logits, T, E, k, opts, topk_idx, dprob, dlogits,
                                            static_cast<cudaStream_t>(stream), err));
}

moe_status moe_expert_bias_update(const int32_t* counts, int E, float coeff, float* expert_bias,
                                  void* stream) {
    if (E < 1 || E > 256 || !counts || !expert_bias || !aligned16(counts) || !aligned16(expert_bias))
        return MOE_ERR_INVALID_ARG;
    if (!(coeff == coeff)) return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_expert_bias_update(counts, E, coeff, expert_bias, static_cast<cudaStream_t>(stream)));
}

size_t moe_aux_loss_workspace_size(int64_t T, int E) {
    if (T < 1 || E < 1 || E > 256) return 0;
    return aux_loss_workspace_bytes(T, E);
}

namespace {
bool aux_args_ok(const float* logits, int64_t T, int E, int k, int score_fn, const int32_t* counts) {
    return T >= 1 && shape_ok(T, E, k) && (score_fn == MOE_SCORE_SOFTMAX || score_fn == MOE_SCORE_SIGMOID) &&
           logits && counts && aligned16(logits) && aligned16(counts);
}
}  // namespace

moe_status moe_aux_loss(const float* logits, int64_t T, int E, int k, int score_fn,
                        const int32_t* counts, float coeff, float* loss, float* scores,
                        void* workspace, size_t workspace_bytes, void* stream) {
    if (!aux_args_ok(logits, T, E, k, score_fn, counts) || !loss || !(coeff == coeff))
        return MOE_ERR_INVALID_ARG;
    if (scores && !aligned16(scores)) return MOE_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return MOE_ERR_INVALID_ARG;
    if (workspace_bytes < aux_loss_workspace_bytes(T, E)) return MOE_ERR_WORKSPACE;
    return from_cuda(launch_aux_loss(logits, T, E, k, score_fn, counts, coeff, loss, scores, workspace,
                                     static_cast<cudaStream_t>(stream)));
}

moe_status moe_aux_loss_backward(const float* logits, int64_t T, int E, int k, int score_fn,
                                 const int32_t* counts, float coeff, const float* grad_loss,
                                 float* dlogits, int accumulate, void* stream) {
    if (!aux_args_ok(logits, T, E, k, score_fn, counts) || !dlogits || !aligned16(dlogits) || !(coeff == coeff))
        return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_aux_loss_backward(logits, T, E, k, score_fn, counts, coeff, grad_loss, dlogits,
                                              accumulate, static_cast<cudaStream_t>(stream)));
}

moe_status moe_router_topk_noalloc(const float* logits, int64_t T, int E, int k,
                                   const moe_router_opts* opts_in, int32_t* topk_idx,
                                   float* topk_prob, uint8_t* routing_map, int32_t* counts,
                                   int32_t* offsets, void* stream) {
    const ChainScope chain(T * (int64_t)k <= kChainMaxRows);
    if (!shape_ok(T, E, k)) return MOE_ERR_INVALID_ARG;
    const moe_router_opts opts = opts_in ? *opts_in : default_opts();
    if (check_opts(opts) != MOE_OK) return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets || !aligned16(counts) || !aligned16(offsets)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !topk_idx || !topk_prob || !aligned16(logits) ||
                  !aligned16(topk_idx) || !aligned16(topk_prob)))
        return MOE_ERR_INVALID_ARG;
    if (opts.expert_bias && !aligned16(opts.expert_bias)) return MOE_ERR_INVALID_ARG;
    if (T > MOE_NOALLOC_MAX_TOKENS || T * (int64_t)k > MOE_NOALLOC_MAX_ASSIGNMENTS ||
        route_scratch_bytes(T, E, k) > router_noalloc_capacity())
        return MOE_ERR_UNSUPPORTED;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st) != cudaSuccess) return MOE_ERR_CUDA;
        return from_cuda(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st));
    }
    void* scratch = nullptr;
    if (router_noalloc_scratch(&scratch) != cudaSuccess || !scratch) return MOE_ERR_CUDA;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    // The router kernel resets the scan's ticket counter itself, and every
    // other scratch word is written before it is read, so the previous call's
    // contents need no clearing.
    const RouteScratch rs = carve_route_scratch(scratch, T, E, k);
    bool scanned = false;
    cudaError_t e = launch_router_topk(logits, T, E, k, opts, topk_idx, topk_prob, routing_map, rs,
                                       st, err, counts, offsets, &scanned);
    if (e == cudaSuccess && !scanned) e = launch_expert_scan(T, E, rs, counts, offsets, st);
    return from_cuda(e);
}

size_t moe_permute_workspace_size(int64_t T, int E, int k) {
    if (!shape_ok(T, E, k)) return 0;
    return route_scratch_bytes(T, E, k);
}

moe_status moe_permute(const moe_bf16* x, int64_t T, int H, const int32_t* topk_idx, int k,
                       const int32_t* offsets, int E, moe_bf16* x_perm, int32_t* sorted_token,
                       int32_t* row_of, void* workspace, size_t workspace_bytes, void* stream) {
    const ChainScope chain(T * (int64_t)k <= kChainMaxRows);
    if (!shape_ok(T, E, k) || H <= 0 || H % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !topk_idx || !offsets || !x_perm || !sorted_token || !row_of) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm) || !aligned16(topk_idx) || !aligned16(offsets) ||
        !aligned16(sorted_token) || !aligned16(row_of))
        return MOE_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < route_scratch_bytes(T, E, k)) return MOE_ERR_WORKSPACE;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const RouteScratch rs = carve_route_scratch(workspace, T, E, k);
    cudaError_t e = launch_rank_from_indices(topk_idx, T, E, k, rs, st, err);
    if (e == cudaSuccess) e = launch_expert_scan(T, E, rs, nullptr, nullptr, st);
    if (e == cudaSuccess)
        e = launch_permute(reinterpret_cast<const bf16*>(x), T, H, topk_idx, k, offsets, E, rs,
                           reinterpret_cast<bf16*>(x_perm), sorted_token, row_of, st, err);
    return from_cuda(e);
}

int64_t moe_permute_padded_max_rows(int64_t T, int E, int k, int align) {
    if (!shape_ok(T, E, k) || align < 1 || align > 65536) return 0;
    const int64_t m = T * k + (int64_t)E * (align - 1);
    return m < (int64_t(1) << 31) ? m : 0;
}

moe_status moe_permute_padded(const moe_bf16* x, int64_t T, int H, const int32_t* topk_idx,
                              const float* topk_prob, int k, const int32_t* offsets, int E, int align,
                              int32_t* padded_offsets, moe_bf16* x_perm, float* prob_perm,
                              int32_t* sorted_token, int32_t* row_of, void* workspace,
                              size_t workspace_bytes, void* stream) {
    const ChainScope chain(T * (int64_t)k <= kChainMaxRows);
    if (!shape_ok(T, E, k) || H <= 0 || H % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (moe_permute_padded_max_rows(T, E, k, align) <= 0 && T > 0) return MOE_ERR_INVALID_ARG;
    if (align < 1 || align > 65536 || !offsets || !padded_offsets || !aligned16(offsets) ||
        !aligned16(padded_offsets))
        return MOE_ERR_INVALID_ARG;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) return from_cuda(cudaMemsetAsync(padded_offsets, 0, sizeof(int32_t) * (E + 1), st));
    if (!x || !topk_idx || !x_perm || !sorted_token || !row_of) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm) || !aligned16(topk_idx) || !aligned16(sorted_token) ||
        !aligned16(row_of) || (prob_perm && (!topk_prob || !aligned16(prob_perm) || !aligned16(topk_prob))))
        return MOE_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < route_scratch_bytes(T, E, k)) return MOE_ERR_WORKSPACE;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const RouteScratch rs = carve_route_scratch(workspace, T, E, k);
    cudaError_t e = launch_pad_offsets(offsets, E, align, padded_offsets, st);
    if (e == cudaSuccess) e = launch_rank_from_indices(topk_idx, T, E, k, rs, st, err);
    if (e == cudaSuccess) e = launch_expert_scan(T, E, rs, nullptr, nullptr, st);
    if (e == cudaSuccess)
        e = launch_permute(reinterpret_cast<const bf16*>(x), T, H, topk_idx, k, padded_offsets, E, rs,
                           reinterpret_cast<bf16*>(x_perm), sorted_token, row_of, st, err,
                           moe_permute_padded_max_rows(T, E, k, align));
    if (e == cudaSuccess)
        e = launch_pad_fill(offsets, padded_offsets, E, H, reinterpret_cast<bf16*>(x_perm), sorted_token,
                            prob_perm, st);
    if (e == cudaSuccess && prob_perm) e = launch_prob_perm(topk_prob, row_of, T * k, prob_perm, st);
    return from_cuda(e);
}

size_t moe_grouped_mlp_workspace_size(int64_t A, int E, int H, int I) {
    if (A < 0 || E < 1 || E > 256 || !dims_ok(H, I)) return 0;
    Carver c(nullptr);
    c.take<bf16>((size_t)A * I);
    return c.bytes();
}

moe_status moe_grouped_mlp(const moe_bf16* x_perm, int64_t A, const int32_t* offsets, int E,
                           int H, int I, const moe_bf16* w_gate_up, const moe_bf16* w_down,
                           moe_bf16* y_perm, moe_bf16* gu_save, moe_bf16* h_save,
                           void* workspace, size_t workspace_bytes, void* stream) {
    return moe_grouped_mlp_scaled(x_perm, A, offsets, E, H, I, w_gate_up, w_down, nullptr, y_perm, gu_save,
                                  h_save, workspace, workspace_bytes, stream);
}

moe_status moe_grouped_mlp_scaled(const moe_bf16* x_perm, int64_t A, const int32_t* offsets, int E,
                                  int H, int I, const moe_bf16* w_gate_up, const moe_bf16* w_down,
                                  const float* row_scale, moe_bf16* y_perm, moe_bf16* gu_save,
                                  moe_bf16* h_save, void* workspace, size_t workspace_bytes, void* stream) {
    const ChainScope chain(A <= kChainMaxRows);
    if (row_scale && !aligned16(row_scale)) return MOE_ERR_INVALID_ARG;
    if (A < 0 || A >= (int64_t(1) << 31) || E < 1 || E > 256) return MOE_ERR_INVALID_ARG;
    if (H <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
    if (!dims_ok(H, I)) return MOE_ERR_UNSUPPORTED;
    if (A == 0) return MOE_OK;
    if (!x_perm || !offsets || !w_gate_up || !w_down || !y_perm) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_perm) || !aligned16(offsets) || !aligned16(w_gate_up) || !aligned16(w_down) ||
        !aligned16(y_perm) || (gu_save && !aligned16(gu_save)) || (h_save && !aligned16(h_save)))
        return MOE_ERR_INVALID_ARG;
    bf16* h = reinterpret_cast<bf16*>(h_save);
    if (!h) {
        if (!workspace || workspace_bytes < moe_grouped_mlp_workspace_size(A, E, H, I))
            return MOE_ERR_WORKSPACE;
        h = Carver(workspace).take<bf16>((size_t)A * I);
    }
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = gemm_gate_up_swiglu(reinterpret_cast<const bf16*>(x_perm), A, offsets, E, H, I,
                                        reinterpret_cast<const bf16*>(w_gate_up), h,
                                        reinterpret_cast<bf16*>(gu_save), st, err, row_scale);
    if (e == cudaSuccess)
        e = gemm_down(h, A, offsets, E, H, I, reinterpret_cast<const bf16*>(w_down),
                      reinterpret_cast<bf16*>(y_perm), st, err);
    return from_cuda(e);
}

moe_status moe_unpermute_combine(const moe_bf16* y_perm, const int32_t* row_of,
                                 const float* topk_prob, int64_t T, int k, int H,
                                 const moe_bf16* shared_out, moe_bf16* out, void* stream) {
    return moe_unpermute_combine_rows(y_perm, T * (int64_t)k, row_of, topk_prob, T, k, H, shared_out, out,
                                      stream);
}

moe_status moe_unpermute_combine_rows(const moe_bf16* y_perm, int64_t y_rows, const int32_t* row_of,
                                      const float* topk_prob, int64_t T, int k, int H,
                                      const moe_bf16* shared_out, moe_bf16* out, void* stream) {
    const ChainScope chain(T * (int64_t)k <= kChainMaxRows);
    if (T < 0 || k < 1 || k > 16 || H <= 0 || H % 8 != 0 || T * (int64_t)k >= (int64_t(1) << 31))
        return MOE_ERR_INVALID_ARG;
    if (y_rows < 0 || y_rows >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y_perm || !row_of || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y_perm) || !aligned16(row_of) || !aligned16(out) ||
        (topk_prob && !aligned16(topk_prob)) || (shared_out && !aligned16(shared_out)))
        return MOE_ERR_INVALID_ARG;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    return from_cuda(launch_combine(reinterpret_cast<const bf16*>(y_perm), row_of, topk_prob, T, k,
                                    H, y_rows, reinterpret_cast<const bf16*>(shared_out),
                                    reinterpret_cast<bf16*>(out), static_cast<cudaStream_t>(stream),
                                    err));
}

size_t moe_layer_forward_workspace_size(int64_t T, int H, int I, int E, int k, int has_shared) {
    if (!shape_ok(T, E, k) || !dims_ok(H, I)) return 0;
    return fwd_layout(nullptr, T, H, I, E, k, has_shared).bytes;
}

moe_status moe_layer_forward(const float* logits, const moe_bf16* x, int64_t T, int H, int I,
                             int E, int k, const moe_router_opts* opts_in,
                             const moe_bf16* w_gate_up, const moe_bf16* w_down,
                             const moe_bf16* shared_gate_up, const moe_bf16* shared_down,
                             moe_bf16* out, int32_t* topk_idx, float* topk_prob, int32_t* counts,
                             int32_t* offsets, int32_t* row_of, moe_bf16* x_perm, moe_bf16* gu,
                             moe_bf16* h, moe_bf16* y_perm, void* workspace,
                             size_t workspace_bytes, void* stream) {
    const ChainScope chain(T * (int64_t)k <= kChainMaxRows);
    if (!shape_ok(T, E, k) || H <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
    if (!dims_ok(H, I)) return MOE_ERR_UNSUPPORTED;
    const moe_router_opts opts = opts_in ? *opts_in : default_opts();
    if (check_opts(opts) != MOE_OK) return MOE_ERR_INVALID_ARG;
    if ((shared_gate_up == nullptr) != (shared_down == nullptr)) return MOE_ERR_INVALID_ARG;
    const void* must[] = {logits, x, w_gate_up, w_down, out};
    for (const void* p : must)
        if (T > 0 && (!p || !aligned16(p))) return MOE_ERR_INVALID_ARG;
    const void* opt[] = {shared_gate_up, shared_down, topk_idx, topk_prob, counts, offsets,
                         row_of, x_perm, gu, h, y_perm, opts.expert_bias};
    for (const void* p : opt)
        if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
    const int has_shared = shared_gate_up != nullptr;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        cudaError_t e = cudaSuccess;
        if (counts) e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st);
        if (e == cudaSuccess && offsets) e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st);
        return from_cuda(e);
    }
    const FwdLayout L0 = fwd_layout(nullptr, T, H, I, E, k, has_shared);
    if (!workspace || workspace_bytes < L0.bytes) return MOE_ERR_WORKSPACE;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    FwdLayout L = fwd_layout(workspace, T, H, I, E, k, has_shared);
    if (topk_idx) L.topk_idx = topk_idx;
    if (topk_prob) L.topk_prob = topk_prob;
    if (counts) L.counts = counts;
    if (offsets) L.offsets = offsets;
    if (row_of) L.row_of = row_of;
    if (x_perm) L.x_perm = reinterpret_cast<bf16*>(x_perm);
    if (h) L.h = reinterpret_cast<bf16*>(h);
    if (y_perm) L.y_perm = reinterpret_cast<bf16*>(y_perm);
    const int64_t A = T * k;
    const bf16* xb = reinterpret_cast<const bf16*>(x);

    // Folded permute (moe_testing_set_kernels): without a requested x_perm, on
    // single-CTA tiles, the gate_up GEMM gathers its A rows from x by token
    // (the permute computes the rows only), so the permuted copy of x is never
    // written or read. Off by default: on B200 the cp.async row gather feeds
    // the tensor cores more slowly than TMA tiles of x_perm (508 against 412 us
    // for the Qwen3-30B-A3B forward), more than the permute's copy costs.
    const bool gather = x_perm == nullptr && grouped_gemm_single_tiles(A, E) && (H % 8) == 0 &&
                        kernel_override().fold_permute != 0;
    // A small batch (an expert gets at most T <= 64 rows, and the experts that
    // can hold rows have as many gate_up tiles as there are SMs) runs gate_up
    // and down as one launch; the router or the scan zeroes its counters.
    const bool fused_mlp = !gather && use_fused_mlp(A, E, T, I);
    int32_t* zero = fused_mlp ? L.sched : nullptr;
    const int n_zero = fused_mlp ? E + 1 : 0;

    cudaError_t e = trace_mark(0, st);
    bool scanned = false, permuted = false;
    // one token block (T <= 8): the router also writes the counts and offsets
    // (no scan launch), and for at most 64 KB of rows the permuted rows too (no
    // permute launch)
    if (e == cudaSuccess)
        e = launch_router_topk(logits, T, E, k, opts, L.topk_idx, L.topk_prob, nullptr, L.rs, st,
                               err, L.counts, L.offsets, &scanned, zero, n_zero, xb, H, gather ? nullptr : L.x_perm,
                               L.sorted_token, L.row_of, gather ? nullptr : &permuted);
    if (e == cudaSuccess && !scanned) e = launch_expert_scan(T, E, L.rs, L.counts, L.offsets, st, zero, n_zero);
    if (e == cudaSuccess) e = trace_mark(1, st);
    if (e == cudaSuccess && !permuted)
        e = launch_permute(xb, T, H, L.topk_idx, k, L.offsets, E, L.rs, gather ? nullptr : L.x_perm,
                           L.sorted_token, L.row_of, st, err);
    if (e == cudaSuccess) e = trace_mark(2, st);
    if (e == cudaSuccess && fused_mlp)
        e = gemm_expert_mlp_fused(L.x_perm, A, L.offsets, E, H, I, reinterpret_cast<const bf16*>(w_gate_up),
                                  reinterpret_cast<const bf16*>(w_down), L.h, reinterpret_cast<bf16*>(gu), L.y_perm,
                                  L.sched, T, st, err);   // the down stage's trace mark follows at once
    else if (e == cudaSuccess)
        e = gather ? gemm_gate_up_swiglu_gather(xb, T, L.sorted_token, A, L.offsets, E, H, I,
                                                reinterpret_cast<const bf16*>(w_gate_up), L.h,
                                                reinterpret_cast<bf16*>(gu), st, err)
                   : gemm_gate_up_swiglu(L.x_perm, A, L.offsets, E, H, I,
                                         reinterpret_cast<const bf16*>(w_gate_up), L.h,
                                         reinterpret_cast<bf16*>(gu), st, err, nullptr, T);
    if (e == cudaSuccess) e = trace_mark(3, st);
    if (e == cudaSuccess && !fused_mlp)
        e = gemm_down(L.h, A, L.offsets, E, H, I, reinterpret_cast<const bf16*>(w_down), L.y_perm,
                      st, err, T);   // an expert gets at most T rows
    if (e == cudaSuccess) e = trace_mark(4, st);
    // With a shared expert on CTA-pair tiles, the combine runs in its down
    // GEMM's epilogue: that GEMM's rows are the tokens in order, so each output
    // row adds its token's k routed rows (j ascending) to the shared expert's
    // fp32 result and is written once; the combine stage is then empty.
    const bool fused = has_shared && grouped_gemm_pair_tiles(T, 1);
    if (e == cudaSuccess && has_shared) {
        e = gemm_gate_up_swiglu(xb, T, nullptr, 1, H, I,
                                reinterpret_cast<const bf16*>(shared_gate_up), L.shared_h, nullptr,
                                st, err);
        if (e == cudaSuccess && fused)
            e = gemm_down_combine(L.shared_h, T, H, I, reinterpret_cast<const bf16*>(shared_down), L.y_perm, A,
                                  L.row_of, L.topk_prob, k, reinterpret_cast<bf16*>(out), st, err);
        else if (e == cudaSuccess)
            e = gemm_down(L.shared_h, T, nullptr, 1, H, I,
                          reinterpret_cast<const bf16*>(shared_down), L.shared_out, st, err);
    }
    if (e == cudaSuccess) e = trace_mark(5, st);
    if (e == cudaSuccess && !fused)
        e = launch_combine(L.y_perm, L.row_of, L.topk_prob, T, k, H, A, L.shared_out,
                           reinterpret_cast<bf16*>(out), st, err);
    if (e == cudaSuccess) e = trace_mark(6, st);
    return from_cuda(e);
}

size_t moe_grouped_mlp_backward_workspace_size(int64_t T, int H, int I, int E, int k) {
    if (!shape_ok(T, E, k) || !dims_ok(H, I)) return 0;
    return bwd_layout(nullptr, T, H, I, k).bytes;
}

moe_status moe_grouped_mlp_backward(const moe_bf16* dout, int64_t T, int H, int I, int E, int k,
                                    const moe_bf16* w_gate_up, const moe_bf16* w_down,
                                    const int32_t* row_of, const float* topk_prob,
                                    const int32_t* offsets, const moe_bf16* x_perm,
                                    const moe_bf16* gu, const moe_bf16* h, const moe_bf16* y_perm,
                                    moe_bf16* dx, moe_bf16* dw_gate_up, moe_bf16* dw_down,
                                    float* dprob, void* workspace, size_t workspace_bytes,
                                    void* stream) {
    const ChainScope chain(T * (int64_t)k <= kChainMaxRows);
    if (!shape_ok(T, E, k) || H <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
    if (!dims_ok(H, I)) return MOE_ERR_UNSUPPORTED;
    const void* must[] = {dout, w_gate_up, w_down, row_of, topk_prob, offsets, x_perm, gu, h,
                          y_perm, dx, dw_gate_up, dw_down, dprob};
    for (const void* p : must)
        if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
    const BwdLayout L0 = bwd_layout(nullptr, T, H, I, k);
    if (!workspace || workspace_bytes < L0.bytes) return MOE_ERR_WORKSPACE;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const BwdLayout L = bwd_layout(workspace, T, H, I, k);
    const int64_t A = T * k;
    auto B = [](const moe_bf16* p) { return reinterpret_cast<const bf16*>(p); };
    cudaError_t e = trace_mark(0, st);
    if (T > 0) {
        if (e == cudaSuccess)
            e = launch_combine_backward(B(dout), B(y_perm), row_of, topk_prob, T, k, H, A, L.dy,
                                        dprob, st, err);
        if (e == cudaSuccess) e = trace_mark(1, st);
        if (e == cudaSuccess)
            e = gemm_down_dgrad_swiglu(L.dy, A, offsets, E, H, I, B(w_down), B(gu), L.dgu, st, err);
        if (e == cudaSuccess) e = trace_mark(2, st);
        if (e == cudaSuccess)
            e = gemm_gate_up_dgrad(L.dgu, A, offsets, E, H, I, B(w_gate_up), L.dx_perm, st, err);
        if (e == cudaSuccess) e = trace_mark(3, st);
        if (e == cudaSuccess)
            e = launch_combine(L.dx_perm, row_of, nullptr, T, k, H, A, nullptr,
                               reinterpret_cast<bf16*>(dx), st, err);
        if (e == cudaSuccess) e = trace_mark(4, st);
    }
    if (e == cudaSuccess)
        e = gemm_wgrad(B(h), L.dy, A, offsets, E, I, H, reinterpret_cast<bf16*>(dw_down), st, err);
    if (e == cudaSuccess) e = trace_mark(5, st);
    if (e == cudaSuccess)
        e = gemm_wgrad(B(x_perm), L.dgu, A, offsets, E, H, 2 * I,
                       reinterpret_cast<bf16*>(dw_gate_up), st, err);
    if (e == cudaSuccess) e = trace_mark(6, st);
    return from_cuda(e);
}

size_t moe_grouped_mlp_scaled_backward_workspace_size(int64_t A, int H, int I) {
    if (A < 0 || A >= (int64_t(1) << 31) || !dims_ok(H, I)) return 0;
    return scaled_bwd_layout(nullptr, A, H, I).bytes;
}

moe_status moe_grouped_mlp_scaled_backward(const moe_bf16* dout, int64_t T, int H, int I, int E, int k,
                                           const moe_bf16* w_gate_up, const moe_bf16* w_down,
                                           const int32_t* row_of, const int32_t* sorted_token,
                                           const float* row_scale, const int32_t* offsets, int64_t A,
                                           const moe_bf16* x_perm, const moe_bf16* gu, const moe_bf16* h,
                                           moe_bf16* dx, moe_bf16* dw_gate_up, moe_bf16* dw_down,
                                           float* dprob, void* workspace, size_t workspace_bytes,
                                           void* stream) {
    const ChainScope chain(A <= kChainMaxRows);
    if (!shape_ok(T, E, k) || H <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
    if (A < T * (int64_t)k || A >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;   // each assignment has a row
    if (!dims_ok(H, I)) return MOE_ERR_UNSUPPORTED;
    const void* must[] = {dout, w_gate_up, w_down, row_of, sorted_token, row_scale, offsets, x_perm, gu, h,
                          dx, dw_gate_up, dw_down, dprob};
    for (const void* p : must)
        if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
    const ScaledBwdLayout L0 = scaled_bwd_layout(nullptr, A, H, I);
    if (!workspace || workspace_bytes < L0.bytes) return MOE_ERR_WORKSPACE;
    unsigned* err = device_error_word();
    if (!err) return MOE_ERR_CUDA;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const ScaledBwdLayout L = scaled_bwd_layout(workspace, A, H, I);
    auto B = [](const moe_bf16* p) { return reinterpret_cast<const bf16*>(p); };
    cudaError_t e = trace_mark(0, st);
    if (A > 0) {
        if (e == cudaSuccess)
            e = launch_gather_rows(B(dout), sorted_token, T, offsets, E, A, H, L.dy, st, err);
        if (e == cudaSuccess) e = trace_mark(1, st);
        if (e == cudaSuccess)
            e = gemm_down_dgrad_swiglu(L.dy, A, offsets, E, H, I, B(w_down), B(gu), L.dgu, st, err, row_scale,
                                       L.row_dot);
        if (e == cudaSuccess)
            e = launch_row_dot_sum(L.row_dot, (I + 63) / 64, row_of, T * (int64_t)k, A, dprob, st, err);
        if (e == cudaSuccess) e = trace_mark(2, st);
        if (e == cudaSuccess)
            e = gemm_gate_up_dgrad(L.dgu, A, offsets, E, H, I, B(w_gate_up), L.dx_perm, st, err);
        if (e == cudaSuccess) e = trace_mark(3, st);
        if (e == cudaSuccess && T > 0)
            e = launch_combine(L.dx_perm, row_of, nullptr, T, k, H, A, nullptr, reinterpret_cast<bf16*>(dx), st,
                               err);
        if (e == cudaSuccess) e = trace_mark(4, st);
    }
    if (e == cudaSuccess)
        e = gemm_wgrad(B(h), L.dy, A, offsets, E, I, H, reinterpret_cast<bf16*>(dw_down), st, err);
    if (e == cudaSuccess) e = trace_mark(5, st);
    if (e == cudaSuccess)
        e = gemm_wgrad(B(x_perm), L.dgu, A, offsets, E, H, 2 * I, reinterpret_cast<bf16*>(dw_gate_up), st, err);
    if (e == cudaSuccess) e = trace_mark(6, st);
    return from_cuda(e);
}

}  // extern "C"
