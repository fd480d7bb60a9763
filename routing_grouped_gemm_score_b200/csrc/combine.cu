// combine.cu -- token combine (unpermute + weighted sum) and its backward.
//
// Transformer Engine "Mixture of Experts", sections Token combine and Token
// probabilities:
//   out[t] = shared[t] + sum_j p[t,j] * y_perm[row_of[t,j]]
// One warp owns one output row, so the sum has a single writer and a fixed
// order (shared first, then j ascending, fp32). The result is the same on
// every run, unlike a scatter-add with atomics. Rows move as 16-byte vectors
// of 8 bf16.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

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

__global__ void __launch_bounds__(256)
    combine_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ row_of,
                   const float* __restrict__ probs, int64_t T, int k, int H8, int64_t A,
                   const uint4* __restrict__ shared, uint4* __restrict__ out, unsigned* err) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T;
         t += warps) {
        int64_t my_row = -1;
        float my_p = 0.0f;
        if (lane < k) {
            const int32_t r = row_of[t * k + lane];
            if (r >= 0 && r < A) {
                my_row = r;
                my_p = probs ? probs[t * k + lane] : 1.0f;
            } else {
                raise_error(err, kErrDeviceCheck);
            }
        }
        // two 16-byte column chunks per lane and pass, so that 2k loads are in flight
        for (int c0 = lane; c0 < H8; c0 += 64) {
            const int c1 = c0 + 32;
            const bool two = c1 < H8;
            float a0[8], a1[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) a0[i] = a1[i] = 0.0f;
            if (shared) {
                add_scaled(a0, __ldg(shared + t * H8 + c0), 1.0f);
                if (two) add_scaled(a1, __ldg(shared + t * H8 + c1), 1.0f);
            }
#pragma unroll 4
            for (int j = 0; j < k; ++j) {
                const int64_t r = __shfl_sync(kFull, my_row, j);
                const float pj = __shfl_sync(kFull, my_p, j);
                if (r < 0) continue;
                const uint4 v0 = __ldg(y + r * H8 + c0);
                const uint4 v1 = two ? __ldg(y + r * H8 + c1) : make_uint4(0, 0, 0, 0);
                add_scaled(a0, v0, pj);
                add_scaled(a1, v1, pj);
            }
            out[t * H8 + c0] = pack8(a0);
            if (two) out[t * H8 + c1] = pack8(a1);
        }
    }
}

// Backward of the weighted combine, one warp per token:
//   dy_perm[row_of[t,j]] = bf16(p[t,j] * dout[t])
//   dprob[t,j] = sum_h dout[t,h] * y_perm[row_of[t,j], h]   (fp32)
// Each lane sums its own columns in order; the warp then reduces in a fixed
// butterfly, so dprob is the same on every run. The dout row is read once per
// assignment; after the first pass it comes from L1.
__global__ void __launch_bounds__(256)
    combine_backward_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ y,
                            const int32_t* __restrict__ row_of, const float* __restrict__ probs,
                            int64_t T, int k, int H8, int64_t A, uint4* __restrict__ dy,
                            float* __restrict__ dprob, unsigned* err) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T;
         t += warps) {
        int64_t my_row = -1;
        float my_p = 0.0f;
        if (lane < k) {
            const int32_t r = row_of[t * k + lane];
            if (r >= 0 && r < A) my_row = r;
            else raise_error(err, kErrDeviceCheck);
            my_p = probs[t * k + lane];
        }
        for (int j = 0; j < k; ++j) {
            const int64_t r = __shfl_sync(kFull, my_row, j);
            const float pj = __shfl_sync(kFull, my_p, j);
            float dot = 0.0f;
            if (r >= 0) {
                for (int c0 = lane; c0 < H8; c0 += 64) {
                    const int c1 = c0 + 32;
                    const bool two = c1 < H8;
                    const uint4 d0 = __ldg(dout + t * H8 + c0);
                    const uint4 y0 = __ldg(y + r * H8 + c0);
                    const uint4 d1 = two ? __ldg(dout + t * H8 + c1) : make_uint4(0, 0, 0, 0);
                    const uint4 y1 = two ? __ldg(y + r * H8 + c1) : make_uint4(0, 0, 0, 0);
                    float s0[8], s1[8];
                    dot_and_scale(d0, y0, pj, dot, s0);
                    dot_and_scale(d1, y1, pj, dot, s1);
                    dy[r * H8 + c0] = pack8(s0);
                    if (two) dy[r * H8 + c1] = pack8(s1);
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(kFull, dot, off);
            if (lane == 0) dprob[t * k + j] = dot;
        }
    }
}

int64_t grid_for_warps(int64_t warps) {
    int64_t blocks = (warps + 7) / 8;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return blocks;
}

}  // namespace

cudaError_t launch_combine(const bf16* y_perm, const int32_t* row_of, const float* probs,
                           int64_t T, int k, int H, int64_t A, const bf16* shared, bf16* out,
                           cudaStream_t st, unsigned* err) {
    combine_kernel<<<(unsigned)grid_for_warps(T), 256, 0, st>>>(
        reinterpret_cast<const uint4*>(y_perm), row_of, probs, T, k, H / 8, A,
        reinterpret_cast<const uint4*>(shared), reinterpret_cast<uint4*>(out), err);
    return cudaGetLastError();
}

cudaError_t launch_combine_backward(const bf16* dout, const bf16* y_perm, const int32_t* row_of,
                                    const float* probs, int64_t T, int k, int H, int64_t A,
                                    bf16* dy_perm, float* dprob, cudaStream_t st, unsigned* err) {
    combine_backward_kernel<<<(unsigned)grid_for_warps(T), 256, 0, st>>>(
        reinterpret_cast<const uint4*>(dout), reinterpret_cast<const uint4*>(y_perm), row_of, probs,
        T, k, H / 8, A, reinterpret_cast<uint4*>(dy_perm), dprob, err);
    return cudaGetLastError();
}

}  // namespace moe
