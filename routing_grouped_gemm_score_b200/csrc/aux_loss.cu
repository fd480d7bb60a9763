// aux_loss.cu -- the router's auxiliary load-balancing loss and its gradient
// to the logits.
//
// Transformer Engine "Mixture of Experts", Load balancing
// (fused_compute_score_for_moe_aux_loss, fused_moe_aux_loss). The loss takes
// the dense scores s[t,e] -- the softmax over all E experts, or the sigmoid of
// each logit, with no expert bias -- and the per-expert token counts c[E] of
// the router's routing map. The page prints no formula; the reading used here
// is the switch-style loss that its inputs name,
//   loss = coeff * E / (k T^2) * sum_e (sum_t s[t,e]) * c_e,
// which is coeff when the load is balanced. The gradient holds the counts
// fixed: with G_e = grad * coeff * E * c_e / (k T^2),
//   softmax: dlogits[t,i] = s[t,i] (G_i - sum_e s[t,e] G_e),
//   sigmoid: dlogits[t,i] = G_i s[t,i] (1 - s[t,i]).
//
// Both kernels give each token to one warp (grid-stride over tokens); a lane
// holds the logits of experts lane, lane + 32, ... in registers. The forward
// reads the logits once, with one 1024-thread block per SM: each lane sums the
// scores of its experts over the warp's tokens in order, a block adds its 32
// warps' sums in warp order into one fp32 value per expert (stored expert-
// major), and the last block to finish (an atomic ticket) adds those in fp64:
// a few threads per expert each take every tpe-th block in order, then the
// expert's threads combine in order. Every order is fixed, so the loss is the
// same on every run on a given GPU.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kAuxThreads = 1024;                 // forward: one block per SM
constexpr int kAuxWarps = kAuxThreads / 32;
constexpr int kAuxBwdThreads = 256;
constexpr int kAuxBwdWarps = kAuxBwdThreads / 32;
constexpr int kAuxMaxE = 256;
constexpr int kAuxBwdBlocksPerSm = 4;

// Tokens a warp loads before it scores the first of them: U rows of logits in
// flight per warp instead of one.
constexpr int kAuxUnroll = 4;

// The lane's logits of one token (experts lane + 32 j); -inf past E.
template <int SLOTS>
__device__ __forceinline__ void load_logits(const float* __restrict__ lrow, int E, int lane, float (&lv)[SLOTS]) {
#pragma unroll
    for (int j = 0; j < SLOTS; ++j) {
        const int e = lane + 32 * j;
        lv[j] = e < E ? __ldg(lrow + e) : -INFINITY;
    }
}

// Dense scores of one token from the lane's logits; 0 past E.
template <int SLOTS>
__device__ __forceinline__ void token_scores(const float (&lv)[SLOTS], int E, int score_fn, int lane,
                                             float (&s)[SLOTS]) {
    if (score_fn == MOE_SCORE_SOFTMAX) {
        float m = lv[0];
#pragma unroll
        for (int j = 1; j < SLOTS; ++j) m = fmaxf(m, lv[j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
        float sum = 0.0f;
#pragma unroll
        for (int j = 0; j < SLOTS; ++j) {
            s[j] = lane + 32 * j < E ? expf(lv[j] - m) : 0.0f;
            sum += s[j];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
        // one correctly rounded reciprocal per token instead of SLOTS divisions:
        // 1.5 ulp per score instead of 0.5
        const float inv = __frcp_rn(sum);
#pragma unroll
        for (int j = 0; j < SLOTS; ++j) s[j] = s[j] * inv;
    } else {
#pragma unroll
        for (int j = 0; j < SLOTS; ++j) s[j] = lane + 32 * j < E ? 1.0f / (1.0f + expf(-lv[j])) : 0.0f;
    }
}

template <int SLOTS>
__global__ void __launch_bounds__(kAuxThreads)
    aux_loss_kernel(const float* __restrict__ logits, int64_t T, int E, int k, int score_fn,
                    const int32_t* __restrict__ counts, float coeff, float* __restrict__ loss,
                    float* __restrict__ scores, float* __restrict__ partial, unsigned* __restrict__ ticket) {
    __shared__ float red[kAuxWarps][kAuxMaxE];     // 32 KB
    __shared__ double dpart[kAuxThreads];
    __shared__ double dred[kAuxMaxE];
    __shared__ bool last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float acc[SLOTS];
#pragma unroll
    for (int j = 0; j < SLOTS; ++j) acc[j] = 0.0f;
    const int64_t nw = (int64_t)gridDim.x * kAuxWarps;
    for (int64_t t0 = (int64_t)blockIdx.x * kAuxWarps + warp; t0 < T; t0 += kAuxUnroll * nw) {
        float lv[kAuxUnroll][SLOTS];
#pragma unroll
        for (int u = 0; u < kAuxUnroll; ++u) {
            const int64_t t = t0 + u * nw;
            if (t < T) load_logits<SLOTS>(logits + t * E, E, lane, lv[u]);
        }
#pragma unroll
        for (int u = 0; u < kAuxUnroll; ++u) {
            const int64_t t = t0 + u * nw;
            if (t >= T) break;
            float s[SLOTS];
            token_scores<SLOTS>(lv[u], E, score_fn, lane, s);
#pragma unroll
            for (int j = 0; j < SLOTS; ++j) {
                acc[j] += s[j];
                const int e = lane + 32 * j;
                if (scores && e < E) scores[t * E + e] = s[j];
            }
        }
    }
#pragma unroll
    for (int j = 0; j < SLOTS; ++j) {
        const int e = lane + 32 * j;
        if (e < E) red[warp][e] = acc[j];
    }
    __syncthreads();
    const int nb = (int)gridDim.x;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kAuxWarps; ++w) v += red[w][e];
        partial[(int64_t)e * nb + blockIdx.x] = v;     // expert-major
    }
    __threadfence();   // this block's row is visible before its ticket
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(ticket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    // tpe threads per expert: thread j of expert e sums blocks j, j + tpe, ...
    const int tpe = kAuxThreads / E;   // >= 4
    {
        const int e = threadIdx.x / tpe, j = threadIdx.x - e * tpe;
        double P = 0.0;
        if (e < E) {
            const float* row = partial + (int64_t)e * nb;
#pragma unroll 4
            for (int b = j; b < nb; b += tpe) P += (double)__ldcg(row + b);
        }
        dpart[threadIdx.x] = P;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        double P = 0.0;
        for (int j = 0; j < tpe; ++j) P += dpart[e * tpe + j];
        dred[e] = P * (double)__ldg(counts + e);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double tot = 0.0;
        for (int e = 0; e < E; ++e) tot += dred[e];
        *loss = (float)((double)coeff * (double)E / ((double)k * (double)T * (double)T) * tot);
    }
}

template <int SLOTS>
__global__ void __launch_bounds__(kAuxBwdThreads)
    aux_loss_backward_kernel(const float* __restrict__ logits, int64_t T, int E, int k, int score_fn,
                             const int32_t* __restrict__ counts, float coeff, const float* __restrict__ grad_loss,
                             float* __restrict__ dlogits, int accumulate) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const double scale = (grad_loss ? (double)__ldg(grad_loss) : 1.0) * (double)coeff * (double)E /
                         ((double)k * (double)T * (double)T);
    float G[SLOTS];
#pragma unroll
    for (int j = 0; j < SLOTS; ++j) {
        const int e = lane + 32 * j;
        G[j] = e < E ? (float)(scale * (double)__ldg(counts + e)) : 0.0f;
    }
    const int64_t nw = (int64_t)gridDim.x * kAuxBwdWarps;
    for (int64_t t0 = (int64_t)blockIdx.x * kAuxBwdWarps + warp; t0 < T; t0 += kAuxUnroll * nw) {
        float lv[kAuxUnroll][SLOTS];
#pragma unroll
        for (int u = 0; u < kAuxUnroll; ++u) {
            const int64_t t = t0 + u * nw;
            if (t < T) load_logits<SLOTS>(logits + t * E, E, lane, lv[u]);
        }
#pragma unroll
        for (int u = 0; u < kAuxUnroll; ++u) {
            const int64_t t = t0 + u * nw;
            if (t >= T) break;
            float s[SLOTS], dl[SLOTS];
            token_scores<SLOTS>(lv[u], E, score_fn, lane, s);
            if (score_fn == MOE_SCORE_SOFTMAX) {
                float dot = 0.0f;
#pragma unroll
                for (int j = 0; j < SLOTS; ++j) dot += s[j] * G[j];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(kFull, dot, off);
#pragma unroll
                for (int j = 0; j < SLOTS; ++j) dl[j] = s[j] * (G[j] - dot);
            } else {
#pragma unroll
                for (int j = 0; j < SLOTS; ++j) dl[j] = G[j] * s[j] * (1.0f - s[j]);
            }
#pragma unroll
            for (int j = 0; j < SLOTS; ++j) {
                const int e = lane + 32 * j;
                if (e >= E) continue;
                float* d = dlogits + t * E + e;
                *d = accumulate ? *d + dl[j] : dl[j];
            }
        }
    }
}

// Blocks of the forward: one warp per token, up to one block per SM, and never
// more than kAuxMaxBlocks, which bounds the workspace whatever the GPU.
constexpr int64_t kAuxMaxBlocks = 1024;

int64_t aux_max_blocks(int64_t T) {
    const int64_t need = (T + kAuxWarps - 1) / kAuxWarps;
    const int64_t b = need < kAuxMaxBlocks ? need : kAuxMaxBlocks;
    return b < 1 ? 1 : b;
}

int64_t aux_blocks(int64_t T) {
    const int64_t cap = sm_count();
    const int64_t b = aux_max_blocks(T);
    return b < cap ? b : cap;
}

int64_t aux_bwd_blocks(int64_t T) {
    const int64_t cap = (int64_t)sm_count() * kAuxBwdBlocksPerSm;
    const int64_t need = (T + kAuxBwdWarps - 1) / kAuxBwdWarps;
    const int64_t b = need < cap ? need : cap;
    return b < 1 ? 1 : b;
}

template <template <int> class K, class... Args>
cudaError_t launch_slots(int E, int64_t blocks, cudaStream_t st, Args... args) {
    const int slots = (E + 31) / 32;
    if (slots <= 1) K<1>::launch(blocks, st, args...);
    else if (slots <= 2) K<2>::launch(blocks, st, args...);
    else if (slots <= 4) K<4>::launch(blocks, st, args...);
    else K<8>::launch(blocks, st, args...);
    return cudaGetLastError();
}

template <int SLOTS>
struct AuxFwd {
    template <class... Args>
    static void launch(int64_t blocks, cudaStream_t st, Args... args) {
        aux_loss_kernel<SLOTS><<<(unsigned)blocks, kAuxThreads, 0, st>>>(args...);
    }
};

template <int SLOTS>
struct AuxBwd {
    template <class... Args>
    static void launch(int64_t blocks, cudaStream_t st, Args... args) {
        aux_loss_backward_kernel<SLOTS><<<(unsigned)blocks, kAuxBwdThreads, 0, st>>>(args...);
    }
};

}  // namespace

size_t aux_loss_workspace_bytes(int64_t T, int E) {
    const size_t rows = (size_t)aux_max_blocks(T) * (size_t)E * sizeof(float);
    return ((rows + 255) & ~size_t(255)) + 256;
}

cudaError_t launch_aux_loss(const float* logits, int64_t T, int E, int k, int score_fn, const int32_t* counts,
                            float coeff, float* loss, float* scores, void* ws, cudaStream_t st) {
    const int64_t blocks = aux_blocks(T);
    float* partial = static_cast<float*>(ws);
    const size_t rows = ((size_t)blocks * (size_t)E * sizeof(float) + 255) & ~size_t(255);
    unsigned* ticket = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + rows);
    cudaError_t e = cudaMemsetAsync(ticket, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return e;
    return launch_slots<AuxFwd>(E, blocks, st, logits, T, E, k, score_fn, counts, coeff, loss, scores, partial,
                                ticket);
}

cudaError_t launch_aux_loss_backward(const float* logits, int64_t T, int E, int k, int score_fn,
                                     const int32_t* counts, float coeff, const float* grad_loss, float* dlogits,
                                     int accumulate, cudaStream_t st) {
    return launch_slots<AuxBwd>(E, aux_bwd_blocks(T), st, logits, T, E, k, score_fn, counts, coeff, grad_loss,
                                dlogits, accumulate);
}

}  // namespace moe
