// combine.cu -- token combine (unpermute + weighted sum) and its backward.
//
// Transformer Engine "Mixture of Experts", sections Token combine and Token
// probabilities:
//   out[t] = shared[t] + sum_j p[t,j] * y_perm[row_of[t,j]]
//   dy_perm[row_of[t,j]] = bf16(p[t,j] * dout[t])
//   dprob[t,j] = sum_h dout[t,h] * y_perm[row_of[t,j], h]   (fp32)
// One warp owns one token, so each output row and each dprob has a single
// writer and a fixed order of operations (shared first, then j ascending,
// fp32). The results are the same on every run, unlike a scatter-add with
// atomics. Rows move as 16-byte vectors of 8 bf16; a lane issues the k loads
// of its column chunks together. Also the two steps of the ScaledSwiGLU
// backward around its GEMMs: the row gather of the output gradient and the
// sum of the routing-weight gradient's partials.
#include <cstdlib>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kWarpKernelThreads = 128;   // 4 tokens in flight per block, one per warp

__device__ __forceinline__ void add_scaled(float (&acc)[8], const uint4& v, float p) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = unpack_bf16x2(w[i]);
        acc[2 * i] += p * f.x;
        acc[2 * i + 1] += p * f.y;
    }
}

// dot += <d, y> (in element order); s = p * d
__device__ __forceinline__ void dot_and_scale(const uint4& d, const uint4& yv, float p, float& dot,
                                              float (&s)[8]) {
    const uint32_t dw[4] = {d.x, d.y, d.z, d.w};
    const uint32_t yw[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 df = unpack_bf16x2(dw[i]);
        const float2 yf = unpack_bf16x2(yw[i]);
        dot += df.x * yf.x;
        dot += df.y * yf.y;
        s[2 * i] = p * df.x;
        s[2 * i + 1] = p * df.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float (&acc)[8]) {
    return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                      pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
}

// Backward of the weighted combine (dy_perm and dprob), one warp per token.
// The warp's lanes cover the row in 16-byte chunks, CH chunks per lane
// per step, each with its k row loads issued together; the next token's
// routing is loaded while the current token is processed. Each lane sums its
// products for every j over its chunks in order, and a warp butterfly then
// gives dprob; the order is fixed, so the result is the same on every run.
template <int KB, int CH>
__global__ void __launch_bounds__(kWarpKernelThreads, KB > 8 ? 2 : 4)
    combine_backward_warp_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ y,
                                 const int32_t* __restrict__ row_of, const float* __restrict__ probs,
                                 int64_t T, int k, int H8, int64_t A, uint4* __restrict__ dy,
                                 float* __restrict__ dprob, unsigned* err) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int32_t r_next = -1;
    float p_next = 0.0f;
    if (t < T && lane < k) {
        r_next = __ldg(row_of + t * k + lane);
        p_next = __ldg(probs + t * k + lane);
    }
    for (; t < T; t += nwarps) {
        int32_t r = r_next;
        const float p = p_next;
        if (lane < k && (r < 0 || r >= A)) {
            raise_error(err, kErrDeviceCheck);
            r = -1;
        }
        const int64_t tn = t + nwarps;   // the next token's routing, one token ahead
        r_next = -1;
        p_next = 0.0f;
        if (tn < T && lane < k) {
            r_next = __ldg(row_of + tn * k + lane);
            p_next = __ldg(probs + tn * k + lane);
        }
        int64_t off[KB];   // first chunk of row j in y and dy; -1: no row
        float ps[KB], dot[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            const int32_t rj = __shfl_sync(kFull, r, j);
            off[j] = (j < k && rj >= 0) ? (int64_t)rj * H8 : -1;
            ps[j] = __shfl_sync(kFull, p, j);
            dot[j] = 0.0f;
        }
        const uint4* drow = dout + t * H8;
        for (int c0 = 0; c0 < H8; c0 += 32 * CH) {
            uint4 d[CH], v[CH][KB];
#pragma unroll
            for (int h = 0; h < CH; ++h) {
                const int c = c0 + 32 * h + lane;
                if (c < H8) d[h] = __ldg(drow + c);
#pragma unroll
                for (int j = 0; j < KB; ++j)
                    if (off[j] >= 0 && c < H8) v[h][j] = __ldg(y + off[j] + c);
            }
#pragma unroll
            for (int h = 0; h < CH; ++h) {
                const int c = c0 + 32 * h + lane;
                if (c >= H8) continue;
#pragma unroll
                for (int j = 0; j < KB; ++j) {
                    if (off[j] < 0) continue;
                    float sc[8];
                    dot_and_scale(d[h], v[h][j], ps[j], dot[j], sc);
                    dy[off[j] + c] = pack8(sc);
                }
            }
        }
        float mine = 0.0f;
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            float v = dot[j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
            if (lane == j) mine = v;
        }
        if (lane < k) dprob[t * k + lane] = mine;
    }
}

// Combine, one warp per token: the warp's lanes cover the output row in
// 16-byte chunks, CH chunks per lane per step, each with its k row loads (and
// the shared row's chunk) issued together; the next token's routing is loaded
// while the current token is summed. The sum runs in a fixed order: shared
// first, then j ascending, fp32.
// A warp's unit of work is one 2^lg_parts-th of a token's row (the whole row
// but for small batches, where one warp per token would leave the GPU idle);
// each output element is summed the same way whatever the split.
template <int KB, int CH>
__global__ void __launch_bounds__(kWarpKernelThreads, KB > 8 ? 2 : 4)
    combine_warp_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ row_of,
                        const float* __restrict__ probs, int64_t T, int k, int H8, int64_t A,
                        const uint4* __restrict__ shared, uint4* __restrict__ out, unsigned* err, int lg_parts) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t units = T << lg_parts;
    const int span = (H8 + (1 << lg_parts) - 1) >> lg_parts;   // chunks of a part
    int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int32_t r_next = -1;
    float p_next = 1.0f;
    if (u < units && lane < k) {
        const int64_t t = u >> lg_parts;
        r_next = __ldg(row_of + t * k + lane);
        if (probs) p_next = __ldg(probs + t * k + lane);
    }
    for (; u < units; u += nwarps) {
        const int64_t t = u >> lg_parts;
        const int c_begin = (int)(u & ((1 << lg_parts) - 1)) * span;
        const int c_end = min(H8, c_begin + span);
        int32_t r = r_next;
        const float p = p_next;
        if (lane < k && (r < 0 || r >= A)) {
            raise_error(err, kErrDeviceCheck);
            r = -1;
        }
        const int64_t un = u + nwarps;   // the next unit's routing, one unit ahead
        r_next = -1;
        p_next = 1.0f;
        if (un < units && lane < k) {
            const int64_t tn = un >> lg_parts;
            r_next = __ldg(row_of + tn * k + lane);
            if (probs) p_next = __ldg(probs + tn * k + lane);
        }
        int64_t off[KB];   // first chunk of row j in y; -1: no row
        float ps[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            const int32_t rj = __shfl_sync(kFull, r, j);
            off[j] = (j < k && rj >= 0) ? (int64_t)rj * H8 : -1;
            ps[j] = __shfl_sync(kFull, p, j);
        }
        for (int c0 = c_begin; c0 < c_end; c0 += 32 * CH) {
            uint4 v[CH][KB], sh[CH];
#pragma unroll
            for (int h = 0; h < CH; ++h) {
                const int c = c0 + 32 * h + lane;
                if (c >= c_end) continue;
                if (shared) sh[h] = __ldg(shared + t * H8 + c);
#pragma unroll
                for (int j = 0; j < KB; ++j)
                    if (off[j] >= 0) v[h][j] = __ldg(y + off[j] + c);
            }
#pragma unroll
            for (int h = 0; h < CH; ++h) {
                const int c = c0 + 32 * h + lane;
                if (c >= c_end) continue;
                float acc[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
                if (shared) add_scaled(acc, sh[h], 1.0f);
#pragma unroll
                for (int j = 0; j < KB; ++j)
                    if (off[j] >= 0) add_scaled(acc, v[h][j], ps[j]);
                out[t * H8 + c] = pack8(acc);
            }
        }
    }
}

// Blocks for a warp-per-token kernel: as many warps as are resident on the
// GPU at once, or one per token if there are fewer tokens; each warp then
// loops over tokens.
template <class K>
int64_t warp_kernel_blocks(K kern, int64_t T) {
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kWarpKernelThreads, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t cap = (int64_t)sm_count() * per_sm * (kWarpKernelThreads / 32);
    const int64_t warps = T < cap ? T : cap;
    return (warps + kWarpKernelThreads / 32 - 1) / (kWarpKernelThreads / 32);
}

// ScaledSwiGLU backward, the combine's gradient: the combine adds the rows
// unweighted, so each row's gradient is its token's output gradient,
// dy[r] = dout[sorted_token[r]], and a pad row (sorted_token -1) gets zeros.
// One warp per row, rows [0, offsets[E]) -- one writer per row, in row order.
__global__ void __launch_bounds__(kWarpKernelThreads)
    gather_rows_kernel(const uint4* __restrict__ dout, const int32_t* __restrict__ sorted_token, int64_t T,
                       const int32_t* __restrict__ offsets, int E, int64_t A, int H8, uint4* __restrict__ dy,
                       unsigned* err) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int64_t rows = __ldg(offsets + E);
    if (rows > A || rows < 0) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(err, kErrDeviceCheck);
        rows = rows < 0 ? 0 : A;
    }
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nwarps) {
        int64_t t = __ldg(sorted_token + r);
        if (t >= T) {
            if (lane == 0) raise_error(err, kErrDeviceCheck);
            t = -1;
        }
        for (int c = lane; c < H8; c += 32)
            dy[r * H8 + c] = t >= 0 ? __ldg(dout + t * H8 + c) : make_uint4(0, 0, 0, 0);
    }
}

// dprob[i] = sum_q row_dot[row_of[i] * nq + q], q ascending: the gradient of
// each routing weight from the per-64-column partial sums that the ScaledSwiGLU
// backward epilogue wrote. One thread per assignment; a fixed order, so the
// result is the same on every run.
__global__ void __launch_bounds__(256)
    row_dot_sum_kernel(const float* __restrict__ row_dot, int nq, const int32_t* __restrict__ row_of, int64_t n,
                       int64_t A, float* __restrict__ dprob, unsigned* err) {
    pdl_wait();
    pdl_launch_dependents();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = __ldg(row_of + i);
        if (r < 0 || r >= A) {
            raise_error(err, kErrDeviceCheck);
            dprob[i] = 0.0f;
            continue;
        }
        const float* src = row_dot + r * nq;
        float sum = 0.0f;
#pragma unroll 8
        for (int q = 0; q < nq; ++q) sum += __ldg(src + q);
        dprob[i] = sum;
    }
}

}  // namespace

cudaError_t launch_gather_rows(const bf16* dout, const int32_t* sorted_token, int64_t T, const int32_t* offsets,
                               int E, int64_t A, int H, bf16* dy, cudaStream_t st, unsigned* err) {
    if (A == 0) return cudaSuccess;
    const int64_t blocks = warp_kernel_blocks(gather_rows_kernel, A);
    return launch_chained(gather_rows_kernel, dim3((unsigned)blocks), dim3(kWarpKernelThreads), 0, st,
                          reinterpret_cast<const uint4*>(dout), sorted_token, T, offsets, E, A, H / 8,
                          reinterpret_cast<uint4*>(dy), err);
}

cudaError_t launch_row_dot_sum(const float* row_dot, int nq, const int32_t* row_of, int64_t n, int64_t A,
                               float* dprob, cudaStream_t st, unsigned* err) {
    if (n == 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    return launch_chained(row_dot_sum_kernel, dim3((unsigned)blocks), dim3(256), 0, st, row_dot, nq, row_of, n, A,
                          dprob, err);
}

cudaError_t launch_combine(const bf16* y_perm, const int32_t* row_of, const float* probs,
                           int64_t T, int k, int H, int64_t A, const bf16* shared, bf16* out,
                           cudaStream_t st, unsigned* err) {
    if (T == 0) return cudaSuccess;
    auto kern = k <= 2 ? combine_warp_kernel<2, 4>
              : k <= 4 ? combine_warp_kernel<4, 2>
              : k <= 8 ? combine_warp_kernel<8, 2> : combine_warp_kernel<16, 1>;
    // small batches: split each token's row over up to 8 warps (whole 16-byte
    // chunks per lane step), so that more SMs share the few rows
    const int H8 = H / 8;
    const int64_t cap = warp_kernel_blocks(kern, (int64_t)1 << 40) * (kWarpKernelThreads / 32);
    int lg = 0;
    while (lg < 3 && (T << (lg + 1)) <= cap && (H8 >> (lg + 1)) >= 64) ++lg;
    const int64_t blocks = warp_kernel_blocks(kern, T << lg);
    return launch_chained(kern, dim3((unsigned)blocks), dim3(kWarpKernelThreads), 0, st,
                          reinterpret_cast<const uint4*>(y_perm), row_of, probs, T, k, H8, A,
                          reinterpret_cast<const uint4*>(shared), reinterpret_cast<uint4*>(out), err, lg);
}

cudaError_t launch_combine_backward(const bf16* dout, const bf16* y_perm, const int32_t* row_of,
                                    const float* probs, int64_t T, int k, int H, int64_t A,
                                    bf16* dy_perm, float* dprob, cudaStream_t st, unsigned* err) {
    if (T == 0) return cudaSuccess;
    auto kern = k <= 2 ? combine_backward_warp_kernel<2, 2>
              : k <= 4 ? combine_backward_warp_kernel<4, 2>
              : k <= 8 ? combine_backward_warp_kernel<8, 2> : combine_backward_warp_kernel<16, 1>;
    const int64_t blocks = warp_kernel_blocks(kern, T);
    return launch_chained(kern, dim3((unsigned)blocks), dim3(kWarpKernelThreads), 0, st,
                          reinterpret_cast<const uint4*>(dout), reinterpret_cast<const uint4*>(y_perm), row_of,
                          probs, T, k, H / 8, A, reinterpret_cast<uint4*>(dy_perm), dprob, err);
}

}  // namespace moe
