// combine.cu -- token combine (unpermute + weighted sum) and its backward.
//
// Transformer Engine "Mixture of Experts", sections Token combine and Token
// probabilities:
//   out[t] = shared[t] + sum_j p[t,j] * y_perm[row_of[t,j]]
// One block owns one output row, so the sum has a single writer and a fixed
// order (shared first, then j ascending, fp32). The result is the same on
// every run, unlike a scatter-add with atomics. Rows move as 16-byte vectors
// of 8 bf16, and each thread issues the k loads of its column chunk together.
#include <cstdlib>

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

// Backward of the weighted combine, one block per token:
//   dy_perm[row_of[t,j]] = bf16(p[t,j] * dout[t])
//   dprob[t,j] = sum_h dout[t,h] * y_perm[row_of[t,j], h]   (fp32)
// Each thread keeps its dout chunk in registers and sums its products for
// every j; the block then reduces the k partial sums in a fixed tree (warp
// butterfly, then warps in order), so dprob is the same on every run.
__global__ void __launch_bounds__(256)
    combine_backward_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ y,
                            const int32_t* __restrict__ row_of, const float* __restrict__ probs,
                            int64_t T, int k, int H8, int64_t A, uint4* __restrict__ dy,
                            float* __restrict__ dprob, unsigned* err) {
    __shared__ int64_t rows[16];
    __shared__ float ps[16];
    __shared__ float part[8][16];   // per warp, per j
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        if (threadIdx.x < (unsigned)k) {
            const int j = threadIdx.x;
            const int32_t r = row_of[t * k + j];
            const bool ok = r >= 0 && r < A;
            if (!ok) raise_error(err, kErrDeviceCheck);
            rows[j] = ok ? r : -1;
            ps[j] = probs[t * k + j];
        }
        __syncthreads();
        float dot[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) dot[j] = 0.0f;
        for (int c = threadIdx.x; c < H8; c += blockDim.x) {
            const uint4 d = __ldg(dout + t * H8 + c);
#pragma unroll
            for (int j0 = 0; j0 < 16; j0 += 8) {      // up to 8 row loads in flight
                if (j0 >= k) break;
                uint4 v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (j0 + j < k && rows[j0 + j] >= 0) v[j] = __ldg(y + rows[j0 + j] * H8 + c);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (j0 + j >= k || rows[j0 + j] < 0) continue;
                    float sc[8];
                    dot_and_scale(d, v[j], ps[j0 + j], dot[j0 + j], sc);
                    dy[rows[j0 + j] * H8 + c] = pack8(sc);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (j >= k) break;
            float v = dot[j];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
            if (lane == 0) part[warp][j] = v;
        }
        __syncthreads();
        if (threadIdx.x < (unsigned)k) {
            float sum = 0.0f;
            for (int w = 0; w < nw; ++w) sum += part[w][threadIdx.x];
            dprob[t * k + threadIdx.x] = sum;
        }
        __syncthreads();
    }
}

// Backward of the weighted combine, one warp per token (same definition as
// above). The warp's lanes cover the row in 16-byte chunks, CH chunks per lane
// per step, each with its k row loads issued together; the next token's
// routing is loaded while the current token is processed. Each lane sums its
// products for every j over its chunks in order, and a warp butterfly then
// gives dprob; the order is fixed, so the result is the same on every run.
template <int KB, int CH>
__global__ void __launch_bounds__(128, KB > 8 ? 2 : 4)
    combine_backward_warp_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ y,
                                 const int32_t* __restrict__ row_of, const float* __restrict__ probs,
                                 int64_t T, int k, int H8, int64_t A, uint4* __restrict__ dy,
                                 float* __restrict__ dprob, unsigned* err) {
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
// while the current token is summed. The sum runs in the fixed order of the
// other combine kernels: shared first, then j ascending, fp32.
template <int KB, int CH>
__global__ void __launch_bounds__(128, KB > 8 ? 2 : 4)
    combine_warp_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ row_of,
                        const float* __restrict__ probs, int64_t T, int k, int H8, int64_t A,
                        const uint4* __restrict__ shared, uint4* __restrict__ out, unsigned* err) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int32_t r_next = -1;
    float p_next = 1.0f;
    if (t < T && lane < k) {
        r_next = __ldg(row_of + t * k + lane);
        if (probs) p_next = __ldg(probs + t * k + lane);
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
        p_next = 1.0f;
        if (tn < T && lane < k) {
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
        for (int c0 = 0; c0 < H8; c0 += 32 * CH) {
            uint4 v[CH][KB], sh[CH];
#pragma unroll
            for (int h = 0; h < CH; ++h) {
                const int c = c0 + 32 * h + lane;
                if (c >= H8) continue;
                if (shared) sh[h] = __ldg(shared + t * H8 + c);
#pragma unroll
                for (int j = 0; j < KB; ++j)
                    if (off[j] >= 0) v[h][j] = __ldg(y + off[j] + c);
            }
#pragma unroll
            for (int h = 0; h < CH; ++h) {
                const int c = c0 + 32 * h + lane;
                if (c >= H8) continue;
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

// Combine over contiguous token ranges, on plain 16-byte loads. A block owns
// tokens [t_begin, t_end). Its threads stage the range's source rows and
// weights in shared memory (kStageTokens at a time, one coalesced load), so no
// token waits on an index load. Each thread owns one 16-byte column chunk
// (blockDim = H/8 rounded up to a warp, H <= 4096), loads that chunk of the token's k rows
// together (KB >= k registers), and issues the next token's loads before it
// sums the current one (for KB <= 8), so loads stay in flight across tokens.
constexpr int kStageEntries = 2048;   // staged assignments (rows + weights: 16 KB)

template <int KB>
__device__ __forceinline__ void combine_issue(const uint4* __restrict__ y, const int32_t* s_row, int k,
                                              int H8, int c, int tt, uint4 (&dst)[KB]) {
#pragma unroll
    for (int j = 0; j < KB; ++j) {
        if (j >= k) break;
        const int32_t r = s_row[tt * k + j];
        if (r >= 0) dst[j] = __ldg(y + (int64_t)r * H8 + c);
    }
}

template <int KB>
__device__ __forceinline__ void combine_finish(const uint4 (&v)[KB], const int32_t* s_row, const float* s_p,
                                               int k, int H8, int c, int tt, int64_t t,
                                               const uint4* __restrict__ shared, uint4* __restrict__ out) {
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
    if (shared) add_scaled(acc, __ldg(shared + t * H8 + c), 1.0f);
#pragma unroll
    for (int j = 0; j < KB; ++j) {
        if (j >= k) break;
        if (s_row[tt * k + j] >= 0) add_scaled(acc, v[j], s_p[tt * k + j]);
    }
    out[t * H8 + c] = pack8(acc);
}

template <int KB>
__global__ void __launch_bounds__(512)
    combine_tokens_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ row_of,
                          const float* __restrict__ probs, int64_t T, int k, int H8, int64_t A,
                          const uint4* __restrict__ shared, uint4* __restrict__ out, int64_t per_block,
                          unsigned* err) {
    __shared__ int32_t s_row[kStageEntries];
    __shared__ float s_p[kStageEntries];
    const int64_t t_begin = (int64_t)blockIdx.x * per_block;
    const int64_t t_end = t_begin + per_block < T ? t_begin + per_block : T;
    const int c = threadIdx.x;            // this thread's column chunk
    const bool active = c < H8;
    const int tok_per_stage = kStageEntries / k;
    for (int64_t s0 = t_begin; s0 < t_end; s0 += tok_per_stage) {
        const int ntok = (int)(t_end - s0 < tok_per_stage ? t_end - s0 : tok_per_stage);
        __syncthreads();   // the previous stage's rows are no longer read
        for (int i = threadIdx.x; i < ntok * k; i += blockDim.x) {
            const int32_t r = row_of[s0 * k + i];
            const bool ok = r >= 0 && r < A;
            if (!ok) raise_error(err, kErrDeviceCheck);
            s_row[i] = ok ? r : -1;
            s_p[i] = probs ? probs[s0 * k + i] : 1.0f;
        }
        __syncthreads();
        if (!active) continue;
        if (KB <= 8) {
            // two register sets: token tt+1's loads fly while token tt is summed
            uint4 va[KB], vb[KB];
            combine_issue<KB>(y, s_row, k, H8, c, 0, va);
            for (int tt = 0; tt < ntok; tt += 2) {
                if (tt + 1 < ntok) combine_issue<KB>(y, s_row, k, H8, c, tt + 1, vb);
                combine_finish<KB>(va, s_row, s_p, k, H8, c, tt, s0 + tt, shared, out);
                if (tt + 1 < ntok) {
                    if (tt + 2 < ntok) combine_issue<KB>(y, s_row, k, H8, c, tt + 2, va);
                    combine_finish<KB>(vb, s_row, s_p, k, H8, c, tt + 1, s0 + tt + 1, shared, out);
                }
            }
        } else {
            uint4 va[KB];
            for (int tt = 0; tt < ntok; ++tt) {
                combine_issue<KB>(y, s_row, k, H8, c, tt, va);
                combine_finish<KB>(va, s_row, s_p, k, H8, c, tt, s0 + tt, shared, out);
            }
        }
    }
}

// Threads per block for one row of H8 chunks: one chunk per thread up to 256.
int row_threads(int H8) {
    int th = 32;
    while (th < H8 && th < 256) th <<= 1;
    return th;
}

int64_t row_blocks(int64_t T) {
    const int64_t cap = (int64_t)sm_count() * 64;   // enough to fill the GPU; rows loop beyond
    return T < cap ? (T > 0 ? T : 1) : cap;
}

}  // namespace

cudaError_t launch_combine(const bf16* y_perm, const int32_t* row_of, const float* probs,
                           int64_t T, int k, int H, int64_t A, const bf16* shared, bf16* out,
                           cudaStream_t st, unsigned* err) {
    if (T == 0) return cudaSuccess;
    const int H8 = H / 8;
    const char* force = getenv("MOE_COMBINE");
    if (!force || force[0] == 'w') {
        auto kern = k <= 2 ? combine_warp_kernel<2, 4>
                  : k <= 4 ? combine_warp_kernel<4, 2>
                  : k <= 8 ? combine_warp_kernel<8, 2> : combine_warp_kernel<16, 1>;
        constexpr int kThreadsW = 128;
        int per_sm = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreadsW, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        const int64_t cap = (int64_t)sm_count() * per_sm * (kThreadsW / 32);
        const int64_t warps = T < cap ? T : cap;
        const int64_t blocks = (warps + kThreadsW / 32 - 1) / (kThreadsW / 32);
        kern<<<(unsigned)blocks, kThreadsW, 0, st>>>(reinterpret_cast<const uint4*>(y_perm), row_of, probs, T, k, H8,
                                                    A, reinterpret_cast<const uint4*>(shared),
                                                    reinterpret_cast<uint4*>(out), err);
        return cudaGetLastError();
    }
    // MOE_COMBINE=regs|bulk: the token-range register kernel or the bulk-copy one
    const bool regs = force[0] == 'r' && H8 <= 512;
    if (regs) {
        const int threads = (H8 + 31) / 32 * 32;
        // blocks resident per SM for this kernel and block size
        auto kern = k <= 2 ? combine_tokens_kernel<2>
                  : k <= 4 ? combine_tokens_kernel<4>
                  : k <= 8 ? combine_tokens_kernel<8> : combine_tokens_kernel<16>;
        int per_sm = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        const int64_t slots = (int64_t)sm_count() * per_sm;
        const int64_t per_block = (T + slots - 1) / slots;
        const int64_t blocks = (T + per_block - 1) / per_block;
        kern<<<(unsigned)blocks, threads, 0, st>>>(reinterpret_cast<const uint4*>(y_perm), row_of, probs, T, k,
                                                  H8, A, reinterpret_cast<const uint4*>(shared),
                                                  reinterpret_cast<uint4*>(out), per_block, err);
        return cudaGetLastError();
    }
    cudaError_t res = cudaSuccess;
    rows_combine(y_perm, row_of, probs, T, k, H, A, shared, out, st, err, &res);
    return res;
}

cudaError_t launch_combine_backward(const bf16* dout, const bf16* y_perm, const int32_t* row_of,
                                    const float* probs, int64_t T, int k, int H, int64_t A,
                                    bf16* dy_perm, float* dprob, cudaStream_t st, unsigned* err) {
    if (T == 0) return cudaSuccess;
    const char* force = getenv("MOE_COMBINE_BWD");
    if (force && force[0] == 'b') {
        combine_backward_kernel<<<(unsigned)row_blocks(T), row_threads(H / 8), 0, st>>>(
            reinterpret_cast<const uint4*>(dout), reinterpret_cast<const uint4*>(y_perm), row_of, probs,
            T, k, H / 8, A, reinterpret_cast<uint4*>(dy_perm), dprob, err);
        return cudaGetLastError();
    }
    auto kern = k <= 2 ? combine_backward_warp_kernel<2, 2>
              : k <= 4 ? combine_backward_warp_kernel<4, 2>
              : k <= 8 ? combine_backward_warp_kernel<8, 2> : combine_backward_warp_kernel<16, 1>;
    constexpr int kThreadsW = 128;
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreadsW, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int64_t warps = (T < (int64_t)sm_count() * per_sm * (kThreadsW / 32)) ? T
                                                                               : (int64_t)sm_count() * per_sm * (kThreadsW / 32);
    const int64_t blocks = (warps + kThreadsW / 32 - 1) / (kThreadsW / 32);
    kern<<<(unsigned)blocks, kThreadsW, 0, st>>>(
        reinterpret_cast<const uint4*>(dout), reinterpret_cast<const uint4*>(y_perm), row_of, probs,
        T, k, H / 8, A, reinterpret_cast<uint4*>(dy_perm), dprob, err);
    return cudaGetLastError();
}

}  // namespace moe
