// grouped_gemm.cu -- persistent grouped GEMM on the sm_100a tensor cores
// (tcgen05.mma, accumulators in tensor memory), fed by TMA.
//
// Transformer Engine "Mixture of Experts", section Grouped GEMM: for each
// expert block i, Y_i = X_i W_i^T, in one call over all blocks, with the
// per-expert token counts kept on the device. Section Grouped MLP: FC1 with
// the activation fused into it, then FC2 as a separate grouped GEMM that
// reads the intermediate from memory. The SwiGLU is that of te_mixtral.py
// (_expert_ffn) and torchtitan GroupedExperts: silu(x Wg) * (x Wu).
//
// One CTA per SM runs a static round-robin over output tiles of 128 x 256.
// Warp roles:
//   warp 0   one thread issues the TMA loads of the A and B tiles of each
//            64-deep K slice into a 4-stage shared-memory ring (128-byte
//            swizzle).
//   warp 1   allocates 512 TMEM columns (two 128 x 256 fp32 accumulators).
//            One thread issues tcgen05.mma (M=128, N=256, K=16, bf16 in,
//            fp32 accumulate) and tcgen05.commit, which frees a smem stage
//            or publishes a finished accumulator.
//   warps 2-5 epilogue: tcgen05.ld of the accumulator rows of their TMEM
//            lane quarter, the fused element-wise work, and 16-byte stores.
// The two accumulators let the epilogue of one tile overlap the MMAs of the
// next.
//
// Two schedules:
//   group-M (forward and dgrad): expert e owns rows [off[e], off[e+1]) of
//     A and of the output. Its tiles are ceil(rows/128) x n_blocks, in
//     expert order, then N block, then M block, so the M blocks that share a
//     weight tile run at about the same time and reuse it from L2. A tile
//     that crosses into the next expert's rows computes them too, and the
//     epilogue drops them. Past the end of A, TMA reads zeros. An expert
//     with no rows has no tiles.
//   group-K (weight gradients): dW[e] = X_e^T D_e. The reduction runs over
//     the rows of expert e. In the last K slice, the rows that belong to the
//     next expert are zeroed in shared memory before the MMA. An expert with
//     no rows writes a zero tile.
// Every wait is bounded (moe_common.cuh). On a timeout the kernel records an
// error, every role leaves its loop, and TMEM is still freed.
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int kThreads = 192;
constexpr int kChunkBytes = 64 * BK * 2;       // one 64-wide swizzle chunk x 64 rows: 8 KB
constexpr int kStageA = BM * BK * 2;           // 16 KB
constexpr int kStageB = BN * BK * 2;           // 32 KB
constexpr int kStageBytes = kStageA + kStageB;  // 48 KB
constexpr int kTmemCols = 512;
constexpr int kMaxGroups = 256;

enum Epi { kEpiStore = 0, kEpiSwiglu = 1, kEpiSwigluBwd = 2 };

struct Params {
    int groups;           // number of experts
    int rows;             // group-M: rows of A and of the output; group-K: rows of X and D
    int M;                // group-K: output rows per expert
    int N;                // output columns per expert (SwiGLU forward: I, the width of h)
    int K;                // group-M: reduction length
    int n_blocks;         // output tiles along N
    int m_blocks;         // group-K: output tiles along M
    const int32_t* offsets;  // [groups+1]; NULL: one group of `rows` rows
    bf16* out;
    int64_t ldo;
    int64_t out_group_stride;  // group-K: elements between experts' outputs
    bf16* out2;                // SwiGLU forward: [g | u] save (may be NULL)
    int64_t ldo2;
    const bf16* aux;           // SwiGLU backward: the saved [g | u]
    int64_t ld_aux;
    int I;                     // SwiGLU: offset of the up half in [g | u]
    unsigned* err;
};

struct __align__(1024) Smem {
    uint8_t stage[STAGES][kStageBytes];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int total_tiles;
    int tile_start[kMaxGroups + 1];
    int off[kMaxGroups + 1];
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;  // + alignment slack

// Shared-memory matrix descriptor: 128-byte swizzle, sm_100 version bit.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: bf16 A and B, fp32 D, M=128, N=256, majors as given.
template <bool A_MN, bool B_MN>
__device__ __forceinline__ constexpr uint32_t instr_desc() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((A_MN ? 1u : 0u) << 15) |
           ((B_MN ? 1u : 0u) << 16) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

struct Tile {
    int g, m_blk, n_blk;
    int row0;   // group-M: first A/output row of the tile; group-K: first X/D row of the expert
    int rows;   // group-M: valid rows of this tile; group-K: rows (K extent) of the expert
    int num_kb;
};

template <bool GROUP_K>
__device__ __forceinline__ Tile decode_tile(const Smem& s, const Params& p, int id) {
    Tile t;
    if (GROUP_K) {
        const int per = p.m_blocks * p.n_blocks;
        t.g = id / per;
        const int local = id - t.g * per;
        t.n_blk = local / p.m_blocks;
        t.m_blk = local - t.n_blk * p.m_blocks;
        t.row0 = s.off[t.g];
        t.rows = max(s.off[t.g + 1] - s.off[t.g], 0);
        t.num_kb = (t.rows + BK - 1) / BK;
    } else {
        int lo = 0, hi = p.groups - 1;  // last g with tile_start[g] <= id
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s.tile_start[mid] <= id) lo = mid;
            else hi = mid - 1;
        }
        t.g = lo;
        const int cnt = max(s.off[t.g + 1] - s.off[t.g], 0);
        const int mt = (cnt + BM - 1) / BM;
        const int local = id - s.tile_start[t.g];
        t.n_blk = local / mt;
        t.m_blk = local - t.n_blk * mt;
        t.row0 = s.off[t.g] + t.m_blk * BM;
        t.rows = min(BM, cnt - t.m_blk * BM);
        t.num_kb = (p.K + BK - 1) / BK;
    }
    return t;
}

template <int EPI, bool A_MN, bool B_MN, bool GROUP_K>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &s.abort;

    // ---- schedule: expert offsets and the tile prefix, in shared memory
    const int G = p.groups;
    for (int g = threadIdx.x; g <= G; g += blockDim.x) {
        int v;
        if (p.offsets) v = __ldg(p.offsets + g);
        else v = (g == 0) ? 0 : p.rows;
        s.off[g] = min(max(v, 0), p.rows);
    }
    __syncthreads();
    if (warp == 0) {
        // tile_start = exclusive prefix of tiles per expert; 8 experts per lane
        int local[8];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int g = lane * 8 + i;
            int tiles = 0;
            if (g < G) {
                if (GROUP_K) {
                    tiles = p.m_blocks * p.n_blocks;
                } else {
                    const int cnt = max(s.off[g + 1] - s.off[g], 0);
                    tiles = ((cnt + BM - 1) / BM) * p.n_blocks;
                }
            }
            local[i] = tiles;
            sum += tiles;
        }
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += o;
        }
        int run = incl - sum;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int g = lane * 8 + i;
            if (g <= G) s.tile_start[g] = run;
            run += local[i];
        }
        if (lane == 31) s.total_tiles = incl;
        if (lane == 0) {
            for (int i = 0; i < STAGES; ++i) {
                mbar_init(&s.full[i], 1);
                mbar_init(&s.empty[i], 1);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(&s.acc_full[i], 1);
                mbar_init(&s.acc_empty[i], 128);
            }
            mbar_init(&s.drain, 1);
            s.abort = 0;
            fence_mbar_init();
            prefetch_tensormap(&tmA);
            prefetch_tensormap(&tmB);
        }
    }
    if (warp == 1) {
        tmem_alloc(&s.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s.tmem_base;
    const int total = s.total_tiles;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued[STAGES] = {0, 0, 0, 0};
            bool ok = true;
            for (int id = blockIdx.x; id < total && ok; id += gridDim.x) {
                const Tile t = decode_tile<GROUP_K>(s, p, id);
                for (int kb = 0; kb < t.num_kb; ++kb) {
                    if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* a_s = s.stage[stage];
                    uint8_t* b_s = s.stage[stage] + kStageA;
                    uint64_t* bar = &s.full[stage];
                    mbar_arrive_expect_tx(bar, kStageBytes);
                    if (GROUP_K) {
                        const int krow = t.row0 + kb * BK;
                        const int m0 = t.m_blk * BM, n0 = t.n_blk * BN;
                        tma_load_2d(&tmA, bar, a_s, m0, krow);
                        tma_load_2d(&tmA, bar, a_s + kChunkBytes, m0 + 64, krow);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            tma_load_2d(&tmB, bar, b_s + c * kChunkBytes, n0 + 64 * c, krow);
                    } else {
                        tma_load_2d(&tmA, bar, a_s, kb * BK, t.row0);
                        if (B_MN) {
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                int col;
                                if (EPI == kEpiSwiglu) {
                                    const int n0 = t.n_blk * (BN / 2);
                                    col = (c < 2) ? n0 + 64 * c : p.I + n0 + 64 * (c - 2);
                                } else {
                                    col = t.n_blk * BN + 64 * c;
                                }
                                tma_load_3d(&tmB, bar, b_s + c * kChunkBytes, col, kb * BK, t.g);
                            }
                        } else {
                            tma_load_3d(&tmB, bar, b_s, kb * BK, t.n_blk * BN, t.g);
                        }
                    }
                    issued[stage] += 1;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // let every load still in flight land before the CTA may exit
            for (int i = 0; i < STAGES; ++i)
                if (issued[i]) mbar_wait(&s.full[i], (issued[i] - 1) & 1u, abort_flag, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = instr_desc<A_MN, B_MN>();
        int stage = 0;
        uint32_t phase = 0;
        int local_tile = 0;
        bool ok = true;
        bool any_mma = false;
        for (int id = blockIdx.x; id < total && ok; id += gridDim.x, ++local_tile) {
            const Tile t = decode_tile<GROUP_K>(s, p, id);
            const int buf = local_tile & 1;
            const uint32_t use = (uint32_t)(local_tile >> 1);
            if (!mbar_wait(&s.acc_empty[buf], (use & 1u) ^ 1u, abort_flag, p.err)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
            if (t.num_kb == 0) {
                if (lane == 0) mbar_arrive(&s.acc_full[buf]);
                __syncwarp();
                continue;
            }
            for (int kb = 0; kb < t.num_kb; ++kb) {
                if (!mbar_wait(&s.full[stage], phase, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(s.stage[stage]);
                const uint32_t b_addr = a_addr + kStageA;
                if (GROUP_K) {
                    const int valid = t.rows - kb * BK;
                    if (valid < BK) {
                        // rows [valid, 64) of every chunk belong to the next expert: zero them
                        const int nrows = BK - valid;
                        for (int i = lane; i < nrows * 6 * 8; i += 32) {
                            const int chunk = i / (nrows * 8);
                            const int rem = i - chunk * nrows * 8;
                            const int r = valid + rem / 8, q = rem % 8;
                            uint4* dst = reinterpret_cast<uint4*>(s.stage[stage] + chunk * kChunkBytes +
                                                                  r * 128) + q;
                            *dst = make_uint4(0, 0, 0, 0);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                    }
                }
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t adesc =
                            A_MN ? smem_desc(a_addr + kk * 2048, kChunkBytes, 1024)
                                 : smem_desc(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc =
                            B_MN ? smem_desc(b_addr + kk * 2048, kChunkBytes, 1024)
                                 : smem_desc(b_addr + kk * 32, 16, 1024);
                        umma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(&s.empty[stage]);
                    any_mma = true;
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(&s.acc_full[buf]);
            __syncwarp();
        }
        // wait until every MMA issued here has finished before TMEM is freed
        if (lane == 0 && any_mma) {
            umma_commit(&s.drain);
            mbar_wait(&s.drain, 0, abort_flag, p.err);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;          // row of the tile owned by this thread
        int local_tile = 0;
        for (int id = blockIdx.x; id < total; id += gridDim.x, ++local_tile) {
            const Tile t = decode_tile<GROUP_K>(s, p, id);
            const int buf = local_tile & 1;
            const uint32_t use = (uint32_t)(local_tile >> 1);
            if (!mbar_wait(&s.acc_full[buf], use & 1u, abort_flag, p.err)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
            if (EPI == kEpiSwiglu) {
                const int n0 = t.n_blk * (BN / 2);
                const bool valid = r < t.rows;
                const int64_t grow = (int64_t)t.row0 + r;
#pragma unroll 1
                for (int c0 = 0; c0 < BN / 2; c0 += 32) {
                    float g[32], u[32];
                    tmem_load_2x32(t_row + c0, t_row + BN / 2 + c0, g, u);
                    if (valid && n0 + c0 < p.N) {
                        uint32_t hv[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            hv[i] = pack_bf16x2(silu_f(g[2 * i]) * u[2 * i],
                                                silu_f(g[2 * i + 1]) * u[2 * i + 1]);
                        uint4* dst = reinterpret_cast<uint4*>(p.out + grow * p.ldo + n0 + c0);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            if (n0 + c0 + 8 * q < p.N)
                                dst[q] = make_uint4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
                        if (p.out2) {
                            uint4* dg = reinterpret_cast<uint4*>(p.out2 + grow * p.ldo2 + n0 + c0);
                            uint4* du = reinterpret_cast<uint4*>(p.out2 + grow * p.ldo2 + p.I + n0 + c0);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                if (n0 + c0 + 8 * q >= p.N) continue;
                                dg[q] = make_uint4(pack_bf16x2(g[8 * q], g[8 * q + 1]),
                                                   pack_bf16x2(g[8 * q + 2], g[8 * q + 3]),
                                                   pack_bf16x2(g[8 * q + 4], g[8 * q + 5]),
                                                   pack_bf16x2(g[8 * q + 6], g[8 * q + 7]));
                                du[q] = make_uint4(pack_bf16x2(u[8 * q], u[8 * q + 1]),
                                                   pack_bf16x2(u[8 * q + 2], u[8 * q + 3]),
                                                   pack_bf16x2(u[8 * q + 4], u[8 * q + 5]),
                                                   pack_bf16x2(u[8 * q + 6], u[8 * q + 7]));
                            }
                        }
                    }
                }
            } else if (EPI == kEpiSwigluBwd) {
                const int n0 = t.n_blk * BN;
                const bool valid = r < t.rows;
                const int64_t grow = (int64_t)t.row0 + r;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 64) {
                    float dh[64];
                    tmem_load_2x32(t_row + c0, t_row + c0 + 32, *reinterpret_cast<float(*)[32]>(dh),
                                   *reinterpret_cast<float(*)[32]>(dh + 32));
                    if (!valid) continue;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int col = n0 + c0 + 8 * q;
                        if (col >= p.N) continue;
                        const uint4 gv = *reinterpret_cast<const uint4*>(p.aux + grow * p.ld_aux + col);
                        const uint4 uv = *reinterpret_cast<const uint4*>(p.aux + grow * p.ld_aux + p.I + col);
                        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
                        const uint32_t uw[4] = {uv.x, uv.y, uv.z, uv.w};
                        uint32_t dgw[4], duw[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 gf = unpack_bf16x2(gw[i]);
                            const float2 uf = unpack_bf16x2(uw[i]);
                            const float d0 = dh[8 * q + 2 * i], d1 = dh[8 * q + 2 * i + 1];
                            const float s0 = 1.0f / (1.0f + expf(-gf.x));
                            const float s1 = 1.0f / (1.0f + expf(-gf.y));
                            const float du0 = d0 * gf.x * s0, du1 = d1 * gf.y * s1;
                            const float dg0 = d0 * uf.x * (s0 + gf.x * s0 * (1.0f - s0));
                            const float dg1 = d1 * uf.y * (s1 + gf.y * s1 * (1.0f - s1));
                            dgw[i] = pack_bf16x2(dg0, dg1);
                            duw[i] = pack_bf16x2(du0, du1);
                        }
                        *reinterpret_cast<uint4*>(p.out + grow * p.ldo + col) =
                            make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
                        *reinterpret_cast<uint4*>(p.out + grow * p.ldo + p.I + col) =
                            make_uint4(duw[0], duw[1], duw[2], duw[3]);
                    }
                }
            } else {
                const int n0 = t.n_blk * BN;
                bool valid;
                bf16* orow;
                if (GROUP_K) {
                    const int m = t.m_blk * BM + r;
                    valid = m < p.M;
                    orow = p.out + (int64_t)t.g * p.out_group_stride + (int64_t)m * p.ldo;
                } else {
                    valid = r < t.rows;
                    orow = p.out + ((int64_t)t.row0 + r) * p.ldo;
                }
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 64) {
                    float v[64];
                    if (t.num_kb > 0) {
                        tmem_load_2x32(t_row + c0, t_row + c0 + 32, *reinterpret_cast<float(*)[32]>(v),
                                       *reinterpret_cast<float(*)[32]>(v + 32));
                    } else {
#pragma unroll
                        for (int i = 0; i < 64; ++i) v[i] = 0.0f;
                    }
                    if (!valid) continue;
                    uint4* dst = reinterpret_cast<uint4*>(orow + n0 + c0);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (n0 + c0 + 8 * q >= p.N) continue;
                        dst[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]),
                                            pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                            pack_bf16x2(v[8 * q + 4], v[8 * q + 5]),
                                            pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&s.acc_empty[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2-D bf16 tensor [outer][inner] with row pitch `pitch` elements.
bool make_map_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t pitch,
                 uint32_t box_inner, uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 tensor [d2][d1][d0], densely packed.
bool make_map_3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint32_t box0, uint32_t box1) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, bool A_MN, bool B_MN, bool GROUP_K>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& b, const Params& p, int64_t max_tiles,
                   cudaStream_t st) {
    auto kern = grouped_gemm_kernel<EPI, A_MN, B_MN, GROUP_K>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    if (max_tiles <= 0) return cudaSuccess;
    int64_t grid = sm_count();
    if (grid > max_tiles) grid = max_tiles;
    kern<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(a, b, p);
    return cudaGetLastError();
}

Params base_params(int groups, int64_t rows, const int32_t* offsets, unsigned* err) {
    Params p{};
    p.groups = groups;
    p.rows = (int)rows;
    p.offsets = offsets;
    p.err = err;
    return p;
}

// Upper bound of group-M tiles without reading the device counts.
int64_t group_m_tile_bound(int64_t rows, int groups, int n_blocks) {
    return ((rows + BM - 1) / BM + groups) * (int64_t)n_blocks;
}

}  // namespace

cudaError_t gemm_gate_up_swiglu(const bf16* x, int64_t rows, const int32_t* offsets, int E, int H,
                                int I, const bf16* w_gate_up, bf16* h, bf16* gu_save,
                                cudaStream_t st, unsigned* err) {
    if (rows == 0) return cudaSuccess;
    CUtensorMap ta, tb;
    if (!make_map_2d(&ta, x, H, rows, H, BK, BM)) return cudaErrorInvalidValue;
    if (!make_map_3d(&tb, w_gate_up, 2 * (uint64_t)I, H, offsets ? E : 1, 64, BK))
        return cudaErrorInvalidValue;
    const int groups = offsets ? E : 1;
    Params p = base_params(groups, rows, offsets, err);
    p.N = I;
    p.K = H;
    p.I = I;
    p.n_blocks = (I + BN / 2 - 1) / (BN / 2);
    p.out = h;
    p.ldo = I;
    p.out2 = gu_save;
    p.ldo2 = 2 * (int64_t)I;
    return launch<kEpiSwiglu, false, true, false>(ta, tb, p,
                                                  group_m_tile_bound(rows, groups, p.n_blocks), st);
}

cudaError_t gemm_down(const bf16* h, int64_t rows, const int32_t* offsets, int E, int H, int I,
                      const bf16* w_down, bf16* y, cudaStream_t st, unsigned* err) {
    if (rows == 0) return cudaSuccess;
    CUtensorMap ta, tb;
    if (!make_map_2d(&ta, h, I, rows, I, BK, BM)) return cudaErrorInvalidValue;
    if (!make_map_3d(&tb, w_down, H, I, offsets ? E : 1, 64, BK)) return cudaErrorInvalidValue;
    const int groups = offsets ? E : 1;
    Params p = base_params(groups, rows, offsets, err);
    p.N = H;
    p.K = I;
    p.n_blocks = (H + BN - 1) / BN;
    p.out = y;
    p.ldo = H;
    return launch<kEpiStore, false, true, false>(ta, tb, p,
                                                 group_m_tile_bound(rows, groups, p.n_blocks), st);
}

cudaError_t gemm_down_dgrad_swiglu(const bf16* dy, int64_t rows, const int32_t* offsets, int E,
                                   int H, int I, const bf16* w_down, const bf16* gu, bf16* dgu,
                                   cudaStream_t st, unsigned* err) {
    if (rows == 0) return cudaSuccess;
    CUtensorMap ta, tb;
    if (!make_map_2d(&ta, dy, H, rows, H, BK, BM)) return cudaErrorInvalidValue;
    // B[n = i][k = h] = w_down[e][i][h]: K-major, box 64 (h) x 256 (i)
    if (!make_map_3d(&tb, w_down, H, I, E, BK, BN)) return cudaErrorInvalidValue;
    Params p = base_params(E, rows, offsets, err);
    p.N = I;
    p.K = H;
    p.I = I;
    p.n_blocks = (I + BN - 1) / BN;
    p.out = dgu;
    p.ldo = 2 * (int64_t)I;
    p.aux = gu;
    p.ld_aux = 2 * (int64_t)I;
    return launch<kEpiSwigluBwd, false, false, false>(ta, tb, p,
                                                      group_m_tile_bound(rows, E, p.n_blocks), st);
}

cudaError_t gemm_gate_up_dgrad(const bf16* dgu, int64_t rows, const int32_t* offsets, int E, int H,
                               int I, const bf16* w_gate_up, bf16* dx_perm, cudaStream_t st,
                               unsigned* err) {
    if (rows == 0) return cudaSuccess;
    CUtensorMap ta, tb;
    if (!make_map_2d(&ta, dgu, 2 * (uint64_t)I, rows, 2 * (uint64_t)I, BK, BM))
        return cudaErrorInvalidValue;
    // B[n = h][k = c] = w_gate_up[e][h][c]: K-major, box 64 (c) x 256 (h)
    if (!make_map_3d(&tb, w_gate_up, 2 * (uint64_t)I, H, E, BK, BN)) return cudaErrorInvalidValue;
    Params p = base_params(E, rows, offsets, err);
    p.N = H;
    p.K = 2 * I;
    p.n_blocks = (H + BN - 1) / BN;
    p.out = dx_perm;
    p.ldo = H;
    return launch<kEpiStore, false, false, false>(ta, tb, p,
                                                  group_m_tile_bound(rows, E, p.n_blocks), st);
}

cudaError_t gemm_wgrad(const bf16* X, const bf16* D, int64_t rows, const int32_t* offsets, int E,
                       int M, int N, bf16* dW, cudaStream_t st, unsigned* err) {
    CUtensorMap ta, tb;
    const uint64_t r = rows > 0 ? (uint64_t)rows : 1;  // an empty X still needs a valid map
    if (!make_map_2d(&ta, X, M, r, M, 64, BK)) return cudaErrorInvalidValue;
    if (!make_map_2d(&tb, D, N, r, N, 64, BK)) return cudaErrorInvalidValue;
    Params p = base_params(E, rows, offsets, err);
    p.M = M;
    p.N = N;
    p.m_blocks = (M + BM - 1) / BM;
    p.n_blocks = (N + BN - 1) / BN;
    p.out = dW;
    p.ldo = N;
    p.out_group_stride = (int64_t)M * N;
    return launch<kEpiStore, true, true, true>(ta, tb, p,
                                               (int64_t)E * p.m_blocks * p.n_blocks, st);
}

}  // namespace moe
