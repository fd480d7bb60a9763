// grouped_gemm.cu -- persistent grouped GEMMs on the sm_100a tensor cores
// (tcgen05.mma, accumulators in tensor memory), fed by TMA.
//
// Transformer Engine "Mixture of Experts", section Grouped GEMM: for each
// expert block i, Y_i = X_i W_i^T, in one call over all blocks, with the
// per-expert token counts kept on the device. Section Grouped MLP: FC1 with
// the activation fused into it, then FC2 as a separate grouped GEMM that
// reads the intermediate from memory. The SwiGLU is that of te_mixtral.py
// (_expert_ffn) and torchtitan GroupedExperts: silu(x Wg) * (x Wu).
//
// Three kernels share the schedule. The forward and dgrad GEMMs run on pair
// tiles when the average expert block is large (>= 1024 rows, or a single dense
// group), else on single-CTA 128-row tiles, which round ragged blocks up less
// (use_pair_tiles); the forward GEMMs of small batches (<= 16 rows per expert
// on average) run on swap-AB tiles (gemm_swap_kernel, use_swap_tiles), and a
// layer's gate_up and down GEMMs for at most 64 rows per expert can run as
// one launch of such tiles (gemm_swap_mlp_kernel, use_fused_mlp).
//
// gemm_pair_kernel (group-M: forward and dgrad). Clusters of two CTAs on two
// SMs compute 256 x 256 output tiles with tcgen05.mma.cta_group::2 (M=256,
// N=256, K=16). Each CTA loads 128 rows of A and 128 columns of B per
// 64-deep K slice (32 KB) into a 6-stage shared-memory ring, so a weight tile
// is read once per 256 rows. The leader CTA issues the MMAs. Its commits
// free both CTAs' stages and publish both CTAs' accumulators
// (tcgen05.commit ... multicast::cluster). The peer CTA's TMA loads complete
// on the leader's full barrier. Expert e owns rows [off[e], off[e+1]) of A and
// of the output. Its tiles are ceil(rows/256) x n_blocks, in expert order,
// then N block, then M block. A tile that crosses into the next expert's rows
// computes them too, and the epilogue drops them. Past the end of A, TMA reads
// zeros. An expert with no rows has no tiles.
//
// gemm_1cta_kernel (group-M with small expert blocks, and group-K: weight
// gradients, dW[e] = X_e^T D_e). One CTA
// per 128 x 256 tile, a 4-stage ring of 48 KB, tcgen05.mma.cta_group::1. The
// reduction runs over the rows of expert e. In the last K slice only the
// 16-row K steps that hold rows of expert e are issued, and the few rows of the
// last step that belong to the next expert are zeroed in shared memory first.
// An expert with no rows writes a zero tile.
//
// Warp roles, in both: warp 0 issues TMA loads (one thread); warp 1 owns
// TMEM (two 128 x 256 fp32 accumulators, 512 columns) and issues the MMAs
// (one thread); warps 2-9 are the epilogue, two per TMEM lane quarter, each
// on one half of the tile's columns (tcgen05.ld of their TMEM lane
// quarter, the fused element-wise work, then a transpose through a per-warp
// shared-memory buffer so that each store instruction writes whole 128- or
// 64-byte row segments; rows outside the expert's block are masked). The two
// accumulators let the epilogue of one tile overlap the MMAs of the next.
// Every wait is bounded (moe_common.cuh). On a timeout the kernel records an
// error, every role leaves its loop, and TMEM is still freed.
#include <cudaTypedefs.h>

#include <cstddef>
#include <cstdlib>
#include <mutex>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int BN = 256, BK = 64;
constexpr int kEpiWarps = 8;                  // two per TMEM lane quarter, one per column half
constexpr int kThreads = 64 + 32 * kEpiWarps;   // warp 0 TMA, warp 1 MMA, warps 2.. epilogue
constexpr int kThreadsK = kThreads + 32;        // group-K adds a fixup warp (ragged K slices)
constexpr int kChunkBytes = 64 * BK * 2;  // one 64-wide swizzle chunk x 64 rows: 8 KB
constexpr int kTmemCols = 512;
constexpr int kMaxGroups = 256;

// single CTA: 128 x 256 tile, 4 stages of 16 + 32 KB
constexpr int BM1 = 128, STAGES1 = 4;
constexpr int kStageA1 = BM1 * BK * 2, kStageB1 = BN * BK * 2, kStage1 = kStageA1 + kStageB1;
// CTA pair: 256 x 256 tile, each CTA 6 stages of 16 + 16 KB
constexpr int BMP = 256, STAGESP = 6;
constexpr int kStageAP = 128 * BK * 2, kStageBP = (BN / 2) * BK * 2, kStageP = kStageAP + kStageBP;
// CTA pair, 128-row tile (an expert block's last <= 128 rows): each CTA loads
// 64 rows of A and its usual half of B
constexpr int kStageHalfP = 64 * BK * 2 + kStageBP;

// kEpiStoreAdd: the store with the token combine folded in (the shared
// expert's down GEMM, whose output rows are the tokens in order).
enum Epi { kEpiStore = 0, kEpiSwiglu = 1, kEpiSwigluBwd = 2, kEpiStoreAdd = 3 };

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
    int tma_out, tma_out2;     // single-CTA kernel: out / out2 have TMA store maps
    const float* row_scale;    // SwiGLU forward: h[r] *= row_scale[r]; backward: ds = row_scale[r] * dh (NULL: 1)
    // SwiGLU backward with row_scale: row_dot[r * ld_row_dot + c / 64] = the sum
    // over the 64 columns c.. of dh * silu(g) * u, in column order (NULL: skip)
    float* row_dot;
    int64_t ld_row_dot;
    // group-M, single CTA: A row r is row gather_tok[r] of gather_x [gather_T][K]
    // (-1: a zero row) instead of a TMA tile of A (NULL: TMA)
    const bf16* gather_x;
    const int32_t* gather_tok;
    int64_t gather_T;
    // kEpiStoreAdd: output row r also gets sum_{j < add_k} add_prob[r * add_k + j]
    // * add_rows[add_row_of[r * add_k + j]], after the accumulator, j ascending, in
    // fp32 (a row index outside [0, add_nrows) is a device-check error and adds nothing)
    const bf16* add_rows;
    const int32_t* add_row_of;
    const float* add_prob;
    int add_k;
    int64_t add_nrows;
    // fused swap-AB expert MLP (gemm_swap_mlp_kernel): the down GEMM's tiles
    // follow the gate_up tiles in one launch; y [rows][N2] = h W_down, n_blocks2
    // tiles of 128 columns per expert, K = I. sched[0] hands out the tiles and
    // sched[1 + g] counts the epilogue warps that have stored their part of
    // expert g's h; all are zero before the launch
    bf16* y;
    int64_t ldy;
    int N2;
    int n_blocks2;
    int32_t* sched;
    unsigned* err;
};

// 16-byte asynchronous copy global -> shared, zero-filled past src_bytes
// (0 or 16), cached in L2 only.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// One arrival on `bar` once this thread's cp.async copies issued so far have
// landed (the arrival is counted in the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int STAGES, int STAGE_BYTES>
struct __align__(1024) Smem {
    uint8_t stage[STAGES][STAGE_BYTES];
    // per epilogue warp: 32 rows x 32 bf16 in the 64-byte swizzle of stage64_off
    // (row stores and TMA stores alike), each on a 512-byte boundary
    uint8_t epi[kEpiWarps][32 * 64];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t ready[STAGES];   // group-K: the stage's ragged rows are zeroed
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int total_tiles;
    int tile_start[kMaxGroups + 1];
    int off[kMaxGroups + 1];
};
using Smem1 = Smem<STAGES1, kStage1>;
using SmemP = Smem<STAGESP, kStageP>;
static_assert(offsetof(Smem1, epi) % 512 == 0 && offsetof(SmemP, epi) % 512 == 0 && (32 * 64) % 512 == 0,
              "64-byte-swizzled staging blocks start on 512-byte boundaries");
constexpr size_t kSmem1Bytes = sizeof(Smem1) + 1024;  // + alignment slack
constexpr size_t kSmemPBytes = sizeof(SmemP) + 1024;
static_assert(kSmem1Bytes <= 227 * 1024 && kSmemPBytes <= 227 * 1024, "shared memory per CTA");

// Shared-memory matrix descriptor: 128-byte swizzle, sm_100 version bit.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: bf16 A and B, fp32 D, the given M and N and majors.
template <int M, int N, bool A_MN, bool B_MN>
__device__ __forceinline__ constexpr uint32_t instr_desc() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((A_MN ? 1u : 0u) << 15) |
           ((B_MN ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

struct Tile {
    int g, m_blk, n_blk;
    int row0;   // group-M: first A/output row of the tile; group-K: first X/D row of the expert
    int rows;   // group-M: valid rows of this tile; group-K: rows (K extent) of the expert
    int num_kb;
};

// Expert offsets and the exclusive prefix of tiles per expert, in shared
// memory. Called by all threads of the CTA; ends with a __syncthreads.
template <bool GROUP_K, class S>
__device__ __forceinline__ void build_schedule(S& s, const Params& p, int bm) {
    const int G = p.groups;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int g = threadIdx.x; g <= G; g += blockDim.x) {
        int v;
        if (p.offsets) v = __ldg(p.offsets + g);
        else v = (g == 0) ? 0 : p.rows;
        s.off[g] = min(max(v, 0), p.rows);
    }
    __syncthreads();
    if (warp == 0) {
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
                    tiles = ((cnt + bm - 1) / bm) * p.n_blocks;
                }
            }
            local[i] = tiles;
            sum += tiles;
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int g = lane * 8 + i;
            if (g <= G) s.tile_start[g] = run;
            run += local[i];
        }
        if (lane == 31) s.total_tiles = incl;
    }
    __syncthreads();
}

template <bool GROUP_K, class S>
__device__ __forceinline__ Tile decode_tile(const S& s, const Params& p, int id, int bm) {
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
        const int mt = (cnt + bm - 1) / bm;
        const int local = id - s.tile_start[t.g];
        t.n_blk = local / mt;
        t.m_blk = local - t.n_blk * mt;
        t.row0 = s.off[t.g] + t.m_blk * bm;
        t.rows = min(bm, cnt - t.m_blk * bm);
        t.num_kb = (p.K + BK - 1) / BK;
    }
    return t;
}

// First column of chunk c (64 columns) of an N-major weight tile. The SwiGLU
// forward takes a tile's gate columns and the matching up columns, so that one
// accumulator holds both. Single CTA: chunks 0..3 of a 256-column tile (128
// gate columns, then their up columns). Pair: each CTA 64 gate columns and
// their up columns (CTA 0 the tile's first 64 columns of h, CTA 1 the next),
// for 256-row and 128-row tiles alike.
template <int EPI>
__device__ __forceinline__ int b_col_1cta(const Tile& t, const Params& p, int c) {
    if (EPI == kEpiSwiglu) {
        const int n0 = t.n_blk * (BN / 2);
        return (c < 2) ? n0 + 64 * c : p.I + n0 + 64 * (c - 2);
    }
    return t.n_blk * BN + 64 * c;
}

template <int EPI>
__device__ __forceinline__ int b_col_pair(const Tile& t, const Params& p, uint32_t rank, int c) {
    if (EPI == kEpiSwiglu) return (c == 0 ? 0 : p.I) + t.n_blk * (BN / 2) + 64 * (int)rank;
    return t.n_blk * BN + (int)rank * 128 + 64 * c;
}

// Byte offset of 16-byte chunk q (0..3) of row r in a 32 x 64-byte staging
// block that a TMA store reads through a 64-byte-swizzled tensor map: the
// chunk index is XORed with address bits 7-8, (r >> 1) & 3 for a block on a
// 512-byte boundary. The same permutation puts the eight rows that a
// quarter-warp writes at once on eight different groups of four banks.
__device__ __forceinline__ uint32_t stage64_off(int r, int q) {
    return (uint32_t)(r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
}

// Writes the 32 values of each lane's row, packed as bf16 pairs (16 words) --
// lane = row of the warp's 32-row group -- to rows [0, nvalid) and columns
// [0, ncols) at dst (row stride ld elements), through the warp's 2 KB staging
// block: each lane writes its row into shared memory, then the warp reads it
// back so that one store instruction covers whole 64-byte row segments. The
// block uses the 64-byte swizzle of stage64_off, so neither phase has bank
// conflicts. Warp-collective.
__device__ __forceinline__ void store_rows_packed32(uint8_t* buf, bf16* dst, int64_t ld, int nvalid, int ncols,
                                                    const uint32_t* w, int lane) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(buf + stage64_off(lane, q)) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    __syncwarp();
    // rows lane / 4 + 8 * pass: the same swizzle term ((row >> 1) & 3) in every pass
    const int chunk = lane % 4;
    const uint8_t* src = buf + stage64_off(lane / 4, chunk);
    bf16* out = dst + (int64_t)(lane / 4) * ld + chunk * 8;
    const bool col_ok = chunk * 8 < ncols;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + pass * 8 * 64);
        if (pass * 8 + lane / 4 < nvalid && col_ok) *reinterpret_cast<uint4*>(out + (int64_t)pass * 8 * ld) = v;
    }
    __syncwarp();   // the buffer is free again
}

// store_rows_packed32 for fp32 values (rounded to bf16).
__device__ __forceinline__ void store_rows32(uint8_t* buf, bf16* dst, int64_t ld, int nvalid, int ncols,
                                             const float* v, int lane) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    store_rows_packed32(buf, dst, ld, nvalid, ncols, w, lane);
}

// Writes a 32 x 32 block (lane = row) of bf16 at dst. With an output tensor
// map and all 32 rows valid, the block goes through the warp's buffer to one
// TMA store (x, y = its first column and row in the map); otherwise through
// store_rows, which masks rows >= nvalid. The buffer is reused only after the
// previous TMA store has read it.
__device__ __forceinline__ void put_block32(uint8_t* buf, bf16* dst, int64_t ld, int nvalid, int ncols,
                                            const float* v, int lane, const CUtensorMap* map, int x, int y) {
    if (map != nullptr) {
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
    }
    if (map != nullptr && nvalid == 32 && ncols == 32) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(buf + stage64_off(lane, q)) =
                make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                           pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(map, buf, x, y);
            bulk_commit_group();
        }
        __syncwarp();
    } else {
        store_rows32(buf, dst, ld, nvalid, ncols, v, lane);
    }
}

// The saved bf16 g and u of one row for 32 columns (16-byte vectors).
struct Aux32 {
    uint4 g[4], u[4];
};

// Loads a row's g and u for columns [col, col + 32) of the saved [g | u];
// does nothing when !ok. Issued a chunk ahead of use so that the loads'
// latency overlaps other work.
__device__ __forceinline__ void load_aux32(const Params& p, int64_t grow, int col, bool ok, Aux32& a) {
    if (!ok) return;
    const uint4* gs = reinterpret_cast<const uint4*>(p.aux + grow * p.ld_aux + col);
    const uint4* us = reinterpret_cast<const uint4*>(p.aux + grow * p.ld_aux + p.I + col);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const bool in = col + 8 * q < p.I;   // columns past I are not read (they are not stored either)
        a.g[q] = in ? __ldg(gs + q) : make_uint4(0, 0, 0, 0);
        a.u[q] = in ? __ldg(us + q) : make_uint4(0, 0, 0, 0);
    }
}

// put_block32 for values already packed as bf16 pairs.
__device__ __forceinline__ void put_block32_packed(uint8_t* buf, bf16* dst, int64_t ld, int nvalid, int ncols,
                                                   const uint32_t* w, int lane, const CUtensorMap* map, int x,
                                                   int y) {
    if (map != nullptr) {
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
    }
    if (map != nullptr && nvalid == 32 && ncols == 32) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(buf + stage64_off(lane, q)) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(map, buf, x, y);
            bulk_commit_group();
        }
        __syncwarp();
    } else {
        store_rows_packed32(buf, dst, ld, nvalid, ncols, w, lane);
    }
}

// SwiGLU backward for 32 columns: from dh and the saved g, u, the bf16 dg and
// du, packed in pairs (dg in dgp, du in dup). SCALED (ScaledSwiGLU, where the
// forward stored h = p * silu(g) * u): the gradient reaching silu(g) * u is
// ds = p * dh, and dot gains sum_c dh[c] * silu(g[c]) * u[c] (the gradient of
// p), in column order.
template <bool SCALED>
__device__ __forceinline__ void swiglu_bwd32(const float* dh, const Aux32& a, float p, float& dot, uint32_t* dgp,
                                             uint32_t* dup) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t gw[4] = {a.g[q].x, a.g[q].y, a.g[q].z, a.g[q].w};
        const uint32_t uw[4] = {a.u[q].x, a.u[q].y, a.u[q].z, a.u[q].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 gf = unpack_bf16x2(gw[i]);
            const float2 uf = unpack_bf16x2(uw[i]);
            const int c = 8 * q + 2 * i;
            // 1/x rounded once: the correctly rounded reciprocal, the same value
            // as the IEEE division 1.0f / x
            const float s0 = __frcp_rn(1.0f + expf(-gf.x));
            const float s1 = __frcp_rn(1.0f + expf(-gf.y));
            float d0 = dh[c], d1 = dh[c + 1];
            if (SCALED) {
                dot += d0 * (gf.x * s0 * uf.x);
                dot += d1 * (gf.y * s1 * uf.y);
                d0 *= p;
                d1 *= p;
            }
            dup[c / 2] = pack_bf16x2(d0 * gf.x * s0, d1 * gf.y * s1);
            dgp[c / 2] = pack_bf16x2(d0 * uf.x * (s0 + gf.x * s0 * (1.0f - s0)),
                                     d1 * uf.y * (s1 + gf.y * s1 * (1.0f - s1)));
        }
    }
}

// The part of a tile's accumulator that one epilogue warp writes out: rows
// [r0, r0 + 32) of the tile (lane = row) and `chunks` 32-column chunks from
// tile column c_lo (SwiGLU forward: columns of h). Column c of the part sits
// at TMEM column tm + (c - c_lo) of the warp's lane quarter; in the SwiGLU
// forward the gate value sits there and the matching up value `up` columns
// further on.
struct EpiMap {
    int r0, c_lo, chunks, tm, up;
};

// A 128-lane accumulator (single-CTA tiles, 256-row pair tiles): lane i holds
// row i; the two warps of a lane quarter split the columns in halves. SwiGLU
// forward: gate in columns [0, 128), up in [128, 256).
template <int EPI>
__device__ __forceinline__ EpiMap full_map(int warp_r0, int col_half) {
    if (EPI == kEpiSwiglu) return EpiMap{warp_r0, 64 * col_half, 2, 64 * col_half, BN / 2};
    return EpiMap{warp_r0, 128 * col_half, 4, 128 * col_half, 0};
}

// full_map for a 256-row pair tile: its SwiGLU accumulator holds
// [g 64 | u 64] of the tile's first 64 columns of h (CTA 0's weights), then
// the same for the next 64 (CTA 1's).
template <int EPI>
__device__ __forceinline__ EpiMap pair_full_map(int warp_r0, int col_half) {
    if (EPI == kEpiSwiglu) return EpiMap{warp_r0, 64 * col_half, 2, 128 * col_half, 64};
    return full_map<EPI>(warp_r0, col_half);
}

// A 128-row pair tile (M = 128 across the two CTAs): each CTA's accumulator
// holds its 64 rows twice over -- tile columns [0, 128) in lanes 0..63 and
// [128, 256) in lanes 64..127, both at TMEM columns 0..127. Quarter q thus
// holds rows 32 * (q & 1) .. +31 (from the CTA's first row) of column half
// q >> 1. The SwiGLU forward loads its B columns as [gate 64 | up 64] per CTA,
// so a lane holds 64 gate columns at TMEM 0..63 and their up values at 64..127.
template <int EPI>
__device__ __forceinline__ EpiMap half_map(uint32_t rank, int quarter, int col_half) {
    const int r0 = 64 * (int)rank + 32 * (quarter & 1);
    if (EPI == kEpiSwiglu) return EpiMap{r0, 64 * (quarter >> 1) + 32 * col_half, 1, 32 * col_half, 64};
    return EpiMap{r0, 128 * (quarter >> 1) + 64 * col_half, 2, 64 * col_half, 0};
}

// Epilogue of one tile for one epilogue warp, on the part `em` of the
// accumulator; t_row addresses TMEM column 0 of the tile's buffer in the warp's
// lane quarter. For group-M the rows count from the tile's first row, and only
// rows inside the expert's block are written. For group-K they count from the
// first output row of the M block.
template <int EPI, bool GROUP_K>
__device__ __forceinline__ void epilogue_tile(const Params& p, const Tile& t, uint32_t t_row,
                                              const EpiMap& em, int lane, int n_tile,
                                              uint8_t* buf, const CUtensorMap* tmC,
                                              const CUtensorMap* tmC2, Aux32* pre) {
    const int warp_r0 = em.r0;
    const int r = warp_r0 + lane;
    if (EPI == kEpiSwiglu) {
        const int n0 = t.n_blk * (n_tile / 2);
        const int nvalid = min(max(t.rows - warp_r0, 0), 32);
        const int64_t row0 = (int64_t)t.row0 + warp_r0;
        // ScaledSwiGLU: the routing weight of the lane's row, applied before FC2
        const float rs = (p.row_scale && lane < nvalid) ? __ldg(p.row_scale + row0 + lane) : 1.0f;
#pragma unroll 1
        for (int i = 0; i < em.chunks; ++i) {
            const int c0 = em.c_lo + 32 * i;
            const uint32_t tc = t_row + (uint32_t)(em.tm + 32 * i);
            float g[32], u[32];
            tmem_load_2x32(tc, tc + (uint32_t)em.up, g, u);
            if (n0 + c0 >= p.N) continue;
            // columns of the chunk inside the output (a multiple of 8): a partial chunk takes
            // masked row stores, since a TMA store of the g part would spill into the u columns
            const int ncols = min(32, p.N - (n0 + c0));
            if (p.out2) {
                put_block32(buf, p.out2 + row0 * p.ldo2 + n0 + c0, p.ldo2, nvalid, ncols, g, lane, tmC2, n0 + c0,
                            (int)row0);
                put_block32(buf, p.out2 + row0 * p.ldo2 + p.I + n0 + c0, p.ldo2, nvalid, ncols, u, lane, tmC2,
                            p.I + n0 + c0, (int)row0);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) g[i] = silu_f(g[i]) * u[i] * rs;     // h, in place
            put_block32(buf, p.out + row0 * p.ldo + n0 + c0, p.ldo, nvalid, ncols, g, lane, tmC, n0 + c0, (int)row0);
        }
    } else if (EPI == kEpiSwigluBwd) {
        // the first chunk's g and u were loaded before the accumulator was
        // ready (`pre`); each later chunk's load while the one before is stored
        const int n0 = t.n_blk * n_tile;
        const bool valid = r < t.rows;
        const int nvalid = min(max(t.rows - warp_r0, 0), 32);
        const int64_t grow = (int64_t)t.row0 + r;
        const int64_t row0 = (int64_t)t.row0 + warp_r0;
        Aux32& ax = *pre;   // reloaded in place for each later chunk
        // ScaledSwiGLU: the row's routing weight, and the partial gradient of
        // it over each 64-column group (em.c_lo is a multiple of 64)
        const float ps = (p.row_scale && valid) ? __ldg(p.row_scale + grow) : 1.0f;
        float dot = 0.0f;
#pragma unroll 1
        for (int ci = 0; ci < em.chunks; ++ci) {
            const int col = n0 + em.c_lo + 32 * ci;
            float dh[32];
            tmem_load_32(t_row + (uint32_t)(em.tm + 32 * ci), dh);
            if (col >= p.N) continue;
            const int ncols = min(32, p.N - col);
            uint32_t dgp[16], dup[16];
            if (valid) {
                if (p.row_dot) {
                    swiglu_bwd32<true>(dh, ax, ps, dot, dgp, dup);
                    if ((ci & 1) || col + 32 >= p.N) {   // the group's last chunk
                        p.row_dot[grow * p.ld_row_dot + (col >> 6)] = dot;
                        dot = 0.0f;
                    }
                } else {
                    swiglu_bwd32<false>(dh, ax, 1.0f, dot, dgp, dup);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) dgp[i] = dup[i] = 0u;   // rows past the block: not stored
            }
            // the next chunk's g and u load while this chunk is stored
            load_aux32(p, grow, col + 32, valid && ci + 1 < em.chunks && col + 32 < p.N, ax);
            put_block32_packed(buf, p.out + row0 * p.ldo + col, p.ldo, nvalid, ncols, dgp, lane, tmC, col,
                               (int)row0);
            put_block32_packed(buf, p.out + row0 * p.ldo + p.I + col, p.ldo, nvalid, ncols, dup, lane, tmC, p.I + col,
                               (int)row0);
        }
    } else if (GROUP_K) {
        // weight gradient: each warp stages 32 rows x 32 columns in shared
        // memory and one lane stores the block into dW[g] with a TMA store;
        // the tensor map drops rows past M and columns past N.
        const int n0 = t.n_blk * n_tile;
        const int m0 = t.m_blk * BM1 + warp_r0;
#pragma unroll 1
        for (int c0 = em.c_lo; c0 < em.c_lo + 32 * em.chunks; c0 += 32) {
            float v[32];
            if (t.num_kb > 0) {
                tmem_load_32(t_row + (uint32_t)(em.tm + c0 - em.c_lo), v);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.0f;
            }
            if (n0 + c0 >= p.N || m0 >= p.M) continue;
            if (lane == 0) bulk_wait_group_read0();   // the previous block has left the buffer
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4*>(buf + stage64_off(lane, q)) =
                    make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                               pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(tmC, buf, n0 + c0, m0, t.g);
                bulk_commit_group();
            }
            __syncwarp();
        }
    } else {
        const int n0 = t.n_blk * n_tile;
        int nvalid;
        bf16* row0;
        if (GROUP_K) {
            const int m0 = t.m_blk * BM1 + warp_r0;
            nvalid = min(max(p.M - m0, 0), 32);
            row0 = p.out + (int64_t)t.g * p.out_group_stride + (int64_t)m0 * p.ldo;
        } else {
            nvalid = min(max(t.rows - warp_r0, 0), 32);
            row0 = p.out + ((int64_t)t.row0 + warp_r0) * p.ldo;
        }
#pragma unroll 1
        for (int c0 = em.c_lo; c0 < em.c_lo + 32 * em.chunks; c0 += 64) {
            float v[64];
            if (t.num_kb > 0) {
                const uint32_t tc = t_row + (uint32_t)(em.tm + c0 - em.c_lo);
                tmem_load_2x32(tc, tc + 32, *reinterpret_cast<float(*)[32]>(v),
                               *reinterpret_cast<float(*)[32]>(v + 32));
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) v[i] = 0.0f;
            }
            if (EPI == kEpiStoreAdd && r < t.rows) {
                // the token's routed rows, weighted, j ascending (16-byte loads of 8 columns)
                const int64_t tok = (int64_t)t.row0 + r;
                for (int j = 0; j < p.add_k; ++j) {
                    const int64_t row = __ldg(p.add_row_of + tok * p.add_k + j);
                    const float pj = __ldg(p.add_prob + tok * p.add_k + j);
                    if (row < 0 || row >= p.add_nrows) {
                        raise_error(p.err, kErrDeviceCheck);
                        continue;
                    }
                    const bf16* src = p.add_rows + row * p.ldo + n0 + c0;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (n0 + c0 + 8 * q >= p.N) break;
                        const uint4 w = __ldg(reinterpret_cast<const uint4*>(src) + q);
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 f = unpack_bf16x2(ws[i]);
                            v[8 * q + 2 * i] += pj * f.x;
                            v[8 * q + 2 * i + 1] += pj * f.y;
                        }
                    }
                }
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (n0 + c0 + 32 * half >= p.N) continue;
                put_block32(buf, row0 + n0 + c0 + 32 * half, p.ldo, nvalid, min(32, p.N - (n0 + c0 + 32 * half)),
                            v + 32 * half, lane,
                            GROUP_K ? nullptr : tmC, n0 + c0 + 32 * half, t.row0 + warp_r0);
            }
        }
    }
}

// ===================================================================== pair
template <int EPI, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA64,
                     const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ CUtensorMap tmC2, const Params p) {
    static_assert(EPI != kEpiSwiglu || B_MN, "the SwiGLU forward reads its weight N-major");
    extern __shared__ uint8_t smem_raw[];
    SmemP& s = *reinterpret_cast<SmemP*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();      // 0: leader, 1: peer
    const int cluster = blockIdx.x >> 1, clusters = gridDim.x >> 1;
    volatile int* abort_flag = &s.abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGESP; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.acc_full[i], 1);
            mbar_init(&s.acc_empty[i], 2 * kEpiWarps);   // one arrival per epilogue warp of both CTAs
        }
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmA64);
        prefetch_tensormap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_pair(&s.tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    pdl_wait();                // the previous kernel's outputs (A, offsets) are complete
    build_schedule<false>(s, p, BMP);
    tc_fence_before();
    cluster_sync_all();        // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = s.tmem_base;
    const int total = s.total_tiles;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t keep = l2_policy_evict_last();   // A panels are read by every N block
            int stage = 0;
            uint32_t phase = 0;
            uint32_t loads = 0;   // stage loads issued; load j used stage j % STAGESP
            bool ok = true;
            for (int id = cluster; id < total && ok; id += clusters) {
                const Tile t = decode_tile<false>(s, p, id, BMP);
                const bool half = t.rows <= 128;   // M = 128 across the pair: 64 rows per CTA
                for (int kb = 0; kb < t.num_kb; ++kb) {
                    if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* a_s = s.stage[stage];
                    uint8_t* b_s = s.stage[stage] + kStageAP;
                    const uint32_t bar = mapa_shared(smem_u32(&s.full[stage]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&s.full[stage], 2 * (half ? kStageHalfP : kStageP));
                    if (half)
                        tma_load_2d_pair_hint(&tmA64, bar, a_s, kb * BK, t.row0 + (int)rank * 64, keep);
                    else
                        tma_load_2d_pair_hint(&tmA, bar, a_s, kb * BK, t.row0 + (int)rank * 128, keep);
                    if (B_MN) {
#pragma unroll
                        for (int c = 0; c < 2; ++c)
                            tma_load_3d_pair(&tmB, bar, b_s + c * kChunkBytes, b_col_pair<EPI>(t, p, rank, c),
                                             kb * BK, t.g);
                    } else {
                        tma_load_3d_pair(&tmB, bar, b_s, kb * BK, t.n_blk * BN + (int)rank * 128,
                                         t.g);
                    }
                    ++loads;
                    if (++stage == STAGESP) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // the leader waits for every load it armed to land before it may exit
            if (rank == 0)
                for (int i = 0; i < STAGESP; ++i)
                    if (loads > (uint32_t)i)   // the stage's last load is its ((loads - 1 - i) / S)-th use
                        mbar_wait(&s.full[i], ((loads - 1 - (uint32_t)i) / STAGESP) & 1u, abort_flag, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer (leader)
        if (rank == 0) {
            constexpr uint32_t idesc_full = instr_desc<BMP, BN, false, B_MN>();
            constexpr uint32_t idesc_half = instr_desc<128, BN, false, B_MN>();
            int stage = 0;
            uint32_t phase = 0;
            int local_tile = 0;
            bool ok = true;
            bool any_mma = false;
            for (int id = cluster; id < total && ok; id += clusters, ++local_tile) {
                const Tile t = decode_tile<false>(s, p, id, BMP);
                const int buf = local_tile & 1;
                const uint32_t use = (uint32_t)(local_tile >> 1);
                if (!mbar_wait_cluster(&s.acc_empty[buf], (use & 1u) ^ 1u, abort_flag, p.err)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
                const uint32_t idesc = t.rows <= 128 ? idesc_half : idesc_full;
                for (int kb = 0; kb < t.num_kb; ++kb) {
                    if (!mbar_wait(&s.full[stage], phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(s.stage[stage]);
                    const uint32_t b_addr = a_addr + kStageAP;
                    if (lane == 0) {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint64_t adesc = smem_desc(a_addr + kk * 32, 16, 1024);
                            const uint64_t bdesc = B_MN ? smem_desc(b_addr + kk * 2048, kChunkBytes, 1024)
                                                        : smem_desc(b_addr + kk * 32, 16, 1024);
                            umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                        umma_commit_pair_mc(&s.empty[stage], 0x3);
                        any_mma = true;
                    }
                    __syncwarp();
                    if (++stage == STAGESP) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) umma_commit_pair_mc(&s.acc_full[buf], 0x3);
                __syncwarp();
            }
            if (lane == 0 && any_mma) {
                umma_commit_pair_mc(&s.drain, 0x1);
                mbar_wait(&s.drain, 0, abort_flag, p.err);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------ epilogue (both CTAs)
        const int quarter = warp & 3;                           // TMEM lanes 32*quarter .. +31
        const int col_half = (warp - 2) / 4;
        const EpiMap em_full = pair_full_map<EPI>((int)rank * 128 + quarter * 32, col_half);
        const EpiMap em_half = half_map<EPI>(rank, quarter, col_half);
        // the leader's barrier of buffer b (computed, not indexed, so that it stays in registers)
        auto leader_acc_empty = [&](int b) { return mapa_shared(smem_u32(&s.acc_empty[b]), 0); };
        int local_tile = 0;
        for (int id = cluster; id < total; id += clusters, ++local_tile) {
            const Tile t = decode_tile<false>(s, p, id, BMP);
            const int buf = local_tile & 1;
            const uint32_t use = (uint32_t)(local_tile >> 1);
            const EpiMap em = t.rows <= 128 ? em_half : em_full;   // a copy: a reference would need memory
            Aux32 pre;
            if (EPI == kEpiSwigluBwd) {
                const int col = t.n_blk * BN + em.c_lo;
                load_aux32(p, (int64_t)t.row0 + em.r0 + lane, col, em.r0 + lane < t.rows && col < p.N, pre);
            }
            if (!mbar_wait(&s.acc_full[buf], use & 1u, abort_flag, p.err)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
            epilogue_tile<EPI, false>(p, t, t_row, em, lane, BN, s.epi[warp - 2],
                                      p.tma_out ? &tmC : nullptr, p.tma_out2 ? &tmC2 : nullptr, &pre);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_acc_empty(buf));
        }
        if (lane == 0) bulk_wait_group0();   // this warp's TMA stores have completed
        __syncwarp();
    }

    // Every role has left its loop: the next kernel of the call may be scheduled
    // (not earlier, so that its blocks do not sit beside this kernel's CTAs).
    pdl_launch_dependents();
    tc_fence_before();
    cluster_sync_all();        // no MMA, load or remote arrival of either CTA is still pending
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

// ===================================================================== single CTA
template <int EPI, bool A_MN, bool B_MN, bool GROUP_K>
__global__ void __launch_bounds__(GROUP_K ? kThreadsK : kThreads, 1)
    gemm_1cta_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2,
                     const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem1& s = *reinterpret_cast<Smem1*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &s.abort;

    const bool gather = !GROUP_K && p.gather_tok != nullptr;
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES1; ++i) {
            mbar_init(&s.full[i], gather ? 33 : 1);   // gather: the B load's arrival and one per copying lane
            mbar_init(&s.empty[i], 1);
            mbar_init(&s.ready[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.acc_full[i], 1);
            mbar_init(&s.acc_empty[i], 32 * kEpiWarps);
        }
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(&s.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    pdl_wait();                // the previous kernel's outputs (A, B, offsets) are complete
    build_schedule<GROUP_K>(s, p, BM1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s.tmem_base;
    const int total = s.total_tiles;

    if (warp == 0 && gather) {
        // ------------------------------------------------- gathering producer
        // Lane 0 loads the B tile with TMA; all 32 lanes copy the A tile's rows
        // from gather_x with 16-byte cp.async (eight lanes per row, four rows per
        // instruction) into the same 128-byte-swizzled
        // K-major layout a TMA tile has (row r at r * 128, its 16-byte chunk c
        // at c ^ (r % 8)). Each lane's arrival on the stage's full barrier fires
        // when its copies have landed; the MMA thread fences the async proxy
        // after its wait, before the tensor cores read the stage.
        int stage = 0;
        uint32_t phase = 0;
        uint32_t loads = 0;   // stage loads issued; load j used stage j % STAGES1
        bool ok = true;
        for (int id = blockIdx.x; id < total && ok; id += gridDim.x) {
            const Tile t = decode_tile<false>(s, p, id, BM1);
            // this lane's rows lane + 32 i: their source rows (NULL: zeros)
            const bf16* src[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = lane + 32 * i;
                int64_t tok = -1;
                if (r < t.rows) {
                    tok = __ldg(p.gather_tok + t.row0 + r);
                    if (tok >= p.gather_T) {
                        raise_error(p.err, kErrDeviceCheck);
                        tok = -1;
                    }
                }
                src[i] = tok >= 0 ? p.gather_x + tok * p.K : nullptr;
            }
            for (int kb = 0; kb < t.num_kb; ++kb) {
                bool got = true;
                if (lane == 0) got = mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag, p.err);
                got = __shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0) != 0;
                if (!got) {
                    ok = false;
                    break;
                }
                uint8_t* a_s = s.stage[stage];
                uint8_t* b_s = s.stage[stage] + kStageA1;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&s.full[stage], kStageB1);
                    if (B_MN) {
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            tma_load_3d(&tmB, &s.full[stage], b_s + c * kChunkBytes, b_col_1cta<EPI>(t, p, c),
                                        kb * BK, t.g);
                    } else {
                        tma_load_3d(&tmB, &s.full[stage], b_s, kb * BK, t.n_blk * BN, t.g);
                    }
                    ++loads;
                }
                // copy j: lane -> 16-byte chunk lane % 8 of row 4 j + lane / 8, so one
                // warp instruction reads four whole 128-byte row segments; the
                // row's source comes from the lane that looked it up
                const uint32_t a_base = smem_u32(a_s);
                const int k0 = kb * BK;
                const int c = lane & 7;
                const bool col_ok = k0 + 8 * c < p.K;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int r = 4 * j + (lane >> 3);
                    const bf16* row_src = reinterpret_cast<const bf16*>(
                        __shfl_sync(0xFFFFFFFFu, reinterpret_cast<uintptr_t>(src[j >> 3]), r & 31));
                    const bool have = row_src != nullptr && col_ok;
                    cp_async_16(a_base + r * 128 + ((c ^ (r & 7)) << 4), have ? row_src + k0 + 8 * c : p.gather_x,
                                have ? 16 : 0);
                }
                cp_async_arrive_noinc(&s.full[stage]);
                if (++stage == STAGES1) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // every copy and every B load lands before the CTA may exit
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
            for (int i = 0; i < STAGES1; ++i)
                if (loads > (uint32_t)i)   // the stage's last load is its ((loads - 1 - i) / S)-th use
                    mbar_wait(&s.full[i], ((loads - 1 - (uint32_t)i) / STAGES1) & 1u, abort_flag, p.err);
        }
        __syncwarp();
    } else if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t keep = l2_policy_evict_last();   // activation panels are read again
            int stage = 0;
            uint32_t phase = 0;
            uint32_t loads = 0;   // stage loads issued; load j used stage j % STAGES1
            bool ok = true;
            for (int id = blockIdx.x; id < total && ok; id += gridDim.x) {
                const Tile t = decode_tile<GROUP_K>(s, p, id, BM1);
                for (int kb = 0; kb < t.num_kb; ++kb) {
                    if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* a_s = s.stage[stage];
                    uint8_t* b_s = s.stage[stage] + kStageA1;
                    uint64_t* bar = &s.full[stage];
                    mbar_arrive_expect_tx(bar, kStage1);
                    if (GROUP_K) {
                        const int krow = t.row0 + kb * BK;
                        const int m0 = t.m_blk * BM1, n0 = t.n_blk * BN;
                        tma_load_2d_hint(&tmA, bar, a_s, m0, krow, keep);
                        tma_load_2d_hint(&tmA, bar, a_s + kChunkBytes, m0 + 64, krow, keep);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            tma_load_2d_hint(&tmB, bar, b_s + c * kChunkBytes, n0 + 64 * c, krow, keep);
                    } else {
                        tma_load_2d_hint(&tmA, bar, a_s, kb * BK, t.row0, keep);
                        if (B_MN) {
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                tma_load_3d(&tmB, bar, b_s + c * kChunkBytes, b_col_1cta<EPI>(t, p, c), kb * BK,
                                            t.g);
                        } else {
                            tma_load_3d(&tmB, bar, b_s, kb * BK, t.n_blk * BN, t.g);
                        }
                    }
                    ++loads;
                    if (++stage == STAGES1) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // let every load still in flight land before the CTA may exit
            for (int i = 0; i < STAGES1; ++i)
                if (loads > (uint32_t)i)   // the stage's last load is its ((loads - 1 - i) / S)-th use
                    mbar_wait(&s.full[i], ((loads - 1 - (uint32_t)i) / STAGES1) & 1u, abort_flag, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = instr_desc<BM1, BN, A_MN, B_MN>();
        int stage = 0;
        uint32_t phase = 0;
        int local_tile = 0;
        bool ok = true;
        bool any_mma = false;
        for (int id = blockIdx.x; id < total && ok; id += gridDim.x, ++local_tile) {
            const Tile t = decode_tile<GROUP_K>(s, p, id, BM1);
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
                // group-K waits for the fixup warp, which has zeroed the rows of a
                // ragged last slice; group-M waits for the loads themselves
                if (!mbar_wait(GROUP_K ? &s.ready[stage] : &s.full[stage], phase, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (gather) fence_proxy_async_smem();   // the A copies were written by cp.async
                const uint32_t a_addr = smem_u32(s.stage[stage]);
                const uint32_t b_addr = a_addr + kStageA1;
                int ksteps = BK / 16;
                if (GROUP_K) {
                    // Rows [valid, 64) of the last slice belong to the next expert:
                    // only the 16-row K steps that hold valid rows are issued
                    const int valid = t.rows - kb * BK;
                    if (valid < BK) ksteps = (valid + 15) / 16;
                }
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        if (kk >= ksteps) break;
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
                if (++stage == STAGES1) {
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
    } else if (warp < 2 + kEpiWarps) {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
        const int col_half = (warp - 2) / 4;
        const int warp_r0 = quarter * 32;           // first tile row of this warp
        const EpiMap em = full_map<EPI>(warp_r0, col_half);
        int local_tile = 0;
        for (int id = blockIdx.x; id < total; id += gridDim.x, ++local_tile) {
            const Tile t = decode_tile<GROUP_K>(s, p, id, BM1);
            const int buf = local_tile & 1;
            const uint32_t use = (uint32_t)(local_tile >> 1);
            Aux32 pre;
            if (EPI == kEpiSwigluBwd) {
                const int col = t.n_blk * BN + em.c_lo;
                load_aux32(p, (int64_t)t.row0 + warp_r0 + lane, col, warp_r0 + lane < t.rows && col < p.N, pre);
            }
            if (!mbar_wait(&s.acc_full[buf], use & 1u, abort_flag, p.err)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
            epilogue_tile<EPI, GROUP_K>(p, t, t_row, em, lane, BN, s.epi[warp - 2],
                                        p.tma_out ? &tmC : nullptr, p.tma_out2 ? &tmC2 : nullptr, &pre);
            tc_fence_before();
            mbar_arrive(&s.acc_empty[buf]);
        }
        if (lane == 0) bulk_wait_group0();   // this warp's TMA stores have completed
        __syncwarp();
    } else if (GROUP_K) {
        // ------------------------------------------------------ fixup (group-K)
        // Passes every landed stage on to the MMA warp. In the last slice of an
        // expert, the rows past the expert's end that share a 16-row K step with
        // its last rows are zeroed first in both operands, so no other expert's
        // data reaches this expert's gradient. The proxy fence that publishes the
        // zeros runs here, away from the MMA warp's queue.
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int id = blockIdx.x; id < total && ok; id += gridDim.x) {
            const Tile t = decode_tile<GROUP_K>(s, p, id, BM1);
            for (int kb = 0; kb < t.num_kb; ++kb) {
                bool got = true;
                if (lane == 0) got = mbar_wait(&s.full[stage], phase, abort_flag, p.err);
                got = __shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0) != 0;
                __syncwarp();
                if (!got) {
                    ok = false;
                    break;
                }
                const int valid = t.rows - kb * BK;
                if (valid < BK) {
                    const int nrows = ((valid + 15) / 16) * 16 - valid;
                    // lane: 16-byte column (lane & 7) of rows valid + (lane >> 3), +4, ...
                    // of each of the 6 chunks (A: 2, B: 4), 128 bytes per row
                    const int q = lane & 7;
#pragma unroll
                    for (int chunk = 0; chunk < 6; ++chunk)
                        for (int rr = valid + (lane >> 3); rr < valid + nrows; rr += 4)
                            *(reinterpret_cast<uint4*>(s.stage[stage] + chunk * kChunkBytes + rr * 128) + q) =
                                make_uint4(0, 0, 0, 0);
                    if (nrows > 0) fence_proxy_async_smem();
                    __syncwarp();
                }
                if (lane == 0) mbar_arrive(&s.ready[stage]);
                if (++stage == STAGES1) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }

    pdl_launch_dependents();   // every role has left its loop (see gemm_pair_kernel)
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ===================================================================== swap-AB
// gemm_swap_kernel: the forward GEMMs for expert blocks of a few rows (small
// batches). The roles of the operands are swapped: the weights are the
// 128-row A operand, read MN-major straight from their [K][N] layout (128
// output columns per tile), and the expert's token rows are the B operand
// (N = NR rows per tile, K-major; NR = 64, or 16 when no expert can have more
// than 16 rows). D = W^T X^T sits in TMEM with one output column per lane and
// one token row per TMEM column. A tile is (expert, 128-column block, NR-row
// block); a block of up to NR rows therefore reads each weight byte once, and
// a one-token expert costs no padded MMA rows. Tiles of one expert run in
// column-block order, its row blocks side by side. With NR = 16 a stage holds
// 2 KB of token rows instead of 8 KB, so the ring keeps 176 KB of weights in
// flight instead of 96 KB.
//
// SwiGLU forward: a tile's 128 columns are 64 gate columns and the matching
// 64 up columns, so lanes 0..63 hold g and lanes 64..127 hold u of the same
// h columns. The epilogue warps of the upper lane quarters pass u to those of
// the lower quarters through shared memory (an mbarrier, bounded wait), which
// compute h = silu(g) u (times the row scale) and store h (and [g | u]).
// Store epilogue (down): each lane writes its output column of every valid row.
// Warp roles as in gemm_1cta_kernel: warp 0 TMA producer, warp 1 TMEM owner
// and MMA issuer, warps 2-9 epilogue (two per lane quarter, each on half of
// the NR token columns). Every wait is bounded.
constexpr int kStageAS = 128 * BK * 2;           // 128 weight columns x 64 K: two 64-column chunks

constexpr int kTileQ = 4;   // tile ids the fused kernel's producer may run ahead by

template <int NR>
struct SwapCfg {
    static constexpr int kStages = NR == 16 ? 11 : 6;
    static constexpr int kStageB = NR * BK * 2;                 // NR token rows x 64 K
    static constexpr int kStage = kStageAS + kStageB;           // 18 or 24 KB
    static constexpr uint32_t kTmemCols = NR == 16 ? 32 : 128;  // two 128-lane x NR-column accumulators
    static constexpr int kWarpCols = NR / 2;                    // token columns of one epilogue warp
};

template <int NR>
struct __align__(1024) SmemS {
    uint8_t stage[SwapCfg<NR>::kStages][SwapCfg<NR>::kStage];
    float ubuf[2][64][NR + 1];    // SwiGLU: the up values of a tile's 64 columns, per accumulator
    uint64_t full[SwapCfg<NR>::kStages];
    uint64_t empty[SwapCfg<NR>::kStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t xchg[2];             // SwiGLU: the up values of the accumulator's tile are in ubuf
    uint64_t drain;
    // gemm_swap_mlp_kernel: the producer's tile ids for the other roles
    uint64_t tq_full[kTileQ];
    uint64_t tq_empty[kTileQ];
    int tile_q[kTileQ];
    uint32_t tmem_base;
    int abort;
    int total_tiles;
    int tile_start[kMaxGroups + 1];
    int off[kMaxGroups + 1];
};
static_assert(SwapCfg<16>::kStage % 1024 == 0 && SwapCfg<64>::kStage % 1024 == 0 && kStageAS % 1024 == 0,
              "swizzled stages stay 1024-byte aligned");
template <int NR>
constexpr size_t swap_smem_bytes() { return sizeof(SmemS<NR>) + 1024; }
static_assert(sizeof(SmemS<16>) + 1024 <= 227 * 1024 && sizeof(SmemS<64>) + 1024 <= 227 * 1024, "swap smem");

// First weight column of chunk c (0, 1) of the tile's 128 columns.
template <int EPI>
__device__ __forceinline__ int w_col_swap(const Tile& t, const Params& p, int c) {
    if (EPI == kEpiSwiglu) return (c == 0 ? 0 : p.I) + t.n_blk * 64;
    return t.n_blk * 128 + 64 * c;
}

// Epilogue of a swap-AB SwiGLU tile for one warp: v holds the warp's kWC token
// columns (j0 ..) of its lane's weight column. The warps of the upper lane
// quarters (u) hand their values to those of the lower quarters (g) through
// ubuf, which store h = silu(g) u (times the row scale) and [g | u]. Returns
// false if the hand-over wait gave up.
template <int NR>
__device__ __forceinline__ bool swap_epi_swiglu(SmemS<NR>& s, const Params& p, const Tile& t, int buf,
                                                uint32_t use, int quarter, int j0, int lane,
                                                const float (&v)[SwapCfg<NR>::kWarpCols], volatile int* abort_flag) {
    constexpr int kWC = SwapCfg<NR>::kWarpCols;
    const int nvalid = min(max(t.rows - j0, 0), kWC);
    if (quarter >= 2) {
        // up values of columns 32 (quarter - 2) + lane
        float* row = s.ubuf[buf][32 * (quarter - 2) + lane] + j0;
#pragma unroll
        for (int i = 0; i < kWC; ++i) row[i] = v[i];
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.xchg[buf]);
        return true;
    }
    if (!mbar_wait(&s.xchg[buf], use & 1u, abort_flag, p.err)) return false;
    const int hc = t.n_blk * 64 + 32 * quarter + lane;   // column of h
    const float* urow = s.ubuf[buf][32 * quarter + lane] + j0;
    const int64_t r0 = (int64_t)t.row0 + j0;
#pragma unroll
    for (int i = 0; i < kWC; ++i) {
        if (i >= nvalid || hc >= p.N) break;
        const float g = v[i], u = urow[i];
        const float rs = p.row_scale ? __ldg(p.row_scale + r0 + i) : 1.0f;
        if (p.out2) {
            p.out2[(r0 + i) * p.ldo2 + hc] = __float2bfloat16_rn(g);
            p.out2[(r0 + i) * p.ldo2 + p.I + hc] = __float2bfloat16_rn(u);
        }
        p.out[(r0 + i) * p.ldo + hc] = __float2bfloat16_rn(silu_f(g) * u * rs);
    }
    return true;
}

// Store epilogue of a swap-AB tile for one warp: its lane's output column of
// every valid token row, into out [rows][ld] (columns < n).
template <int NR>
__device__ __forceinline__ void swap_epi_store(bf16* out, int64_t ld, int n, const Tile& t, int quarter, int j0,
                                               int lane, const float (&v)[SwapCfg<NR>::kWarpCols]) {
    constexpr int kWC = SwapCfg<NR>::kWarpCols;
    const int nvalid = min(max(t.rows - j0, 0), kWC);
    const int col = t.n_blk * 128 + 32 * quarter + lane;
    const int64_t r0 = (int64_t)t.row0 + j0;
    if (col < n) {
#pragma unroll
        for (int i = 0; i < kWC; ++i) {
            if (i >= nvalid) break;
            out[(r0 + i) * ld + col] = __float2bfloat16_rn(v[i]);
        }
    }
}

template <int EPI, int NR>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_swap_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const Params p) {
    static_assert(EPI == kEpiSwiglu || EPI == kEpiStore, "forward GEMMs only");
    extern __shared__ uint8_t smem_raw[];
    using Cfg = SwapCfg<NR>;
    SmemS<NR>& s = *reinterpret_cast<SmemS<NR>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &s.abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::kStages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.acc_full[i], 1);
            mbar_init(&s.acc_empty[i], kEpiWarps);   // one arrival per epilogue warp
            mbar_init(&s.xchg[i], kEpiWarps / 2);    // one per upper-quarter warp
        }
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(&s.tmem_base, Cfg::kTmemCols);
        tmem_relinquish();
    }
    pdl_wait();                // the previous kernel's outputs (token rows, offsets) are complete
    build_schedule<false>(s, p, NR);
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
            uint32_t loads = 0;   // stage loads issued; load j used stage j % kStages
            bool ok = true;
            for (int id = blockIdx.x; id < total && ok; id += gridDim.x) {
                const Tile t = decode_tile<false>(s, p, id, NR);
                for (int kb = 0; kb < t.num_kb; ++kb) {
                    if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* a_s = s.stage[stage];
                    uint8_t* b_s = s.stage[stage] + kStageAS;
                    uint64_t* bar = &s.full[stage];
                    mbar_arrive_expect_tx(bar, Cfg::kStage);
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(&tmW, bar, a_s + c * kChunkBytes, w_col_swap<EPI>(t, p, c), kb * BK, t.g);
                    tma_load_2d(&tmX, bar, b_s, kb * BK, t.row0);
                    ++loads;
                    if (++stage == Cfg::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // let every load still in flight land before the CTA may exit
            for (int i = 0; i < Cfg::kStages; ++i)
                if (loads > (uint32_t)i)   // the stage's last load is its ((loads - 1 - i) / S)-th use
                    mbar_wait(&s.full[i], ((loads - 1 - (uint32_t)i) / Cfg::kStages) & 1u, abort_flag, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = instr_desc<128, NR, true, false>();
        int stage = 0;
        uint32_t phase = 0;
        int local_tile = 0;
        bool ok = true;
        bool any_mma = false;
        for (int id = blockIdx.x; id < total && ok; id += gridDim.x, ++local_tile) {
            const Tile t = decode_tile<false>(s, p, id, NR);
            const int buf = local_tile & 1;
            const uint32_t use = (uint32_t)(local_tile >> 1);
            if (!mbar_wait(&s.acc_empty[buf], (use & 1u) ^ 1u, abort_flag, p.err)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(buf * NR);
            for (int kb = 0; kb < t.num_kb; ++kb) {
                if (!mbar_wait(&s.full[stage], phase, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(s.stage[stage]);
                const uint32_t b_addr = a_addr + kStageAS;
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t adesc = smem_desc(a_addr + kk * 2048, kChunkBytes, 1024);
                        const uint64_t bdesc = smem_desc(b_addr + kk * 32, 16, 1024);
                        umma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(&s.empty[stage]);
                    any_mma = true;
                }
                __syncwarp();
                if (++stage == Cfg::kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(&s.acc_full[buf]);
            __syncwarp();
        }
        if (lane == 0 && any_mma) {
            umma_commit(&s.drain);
            mbar_wait(&s.drain, 0, abort_flag, p.err);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
        const int half = (warp - 2) / 4;            // token columns kWarpCols*half ..
        int local_tile = 0;
        for (int id = blockIdx.x; id < total; id += gridDim.x, ++local_tile) {
            const Tile t = decode_tile<false>(s, p, id, NR);
            const int buf = local_tile & 1;
            const uint32_t use = (uint32_t)(local_tile >> 1);
            if (!mbar_wait(&s.acc_full[buf], use & 1u, abort_flag, p.err)) break;
            tc_fence_after();
            constexpr int kWC = Cfg::kWarpCols;
            float v[kWC];
            const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * NR + kWC * half);
            if constexpr (kWC == 32) tmem_load_32(taddr, v);
            else tmem_load_8(taddr, v);
            const int j0 = kWC * half;                       // first token column of this warp
            bool ok = true;
            if (EPI == kEpiSwiglu) ok = swap_epi_swiglu<NR>(s, p, t, buf, use, quarter, j0, lane, v, abort_flag);
            else swap_epi_store<NR>(p.out, p.ldo, p.N, t, quarter, j0, lane, v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.acc_empty[buf]);
            if (!ok) break;
        }
    }

    pdl_launch_dependents();   // every role has left its loop (see gemm_pair_kernel)
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

// ================================================================ fused MLP
// gemm_swap_mlp_kernel: the expert MLP of a small batch in one launch, on the
// swap-AB tiles of gemm_swap_kernel: first the gate_up + SwiGLU tiles of every
// expert (h, and [g | u] when saved), then the down tiles (y = h W_down).
// The producer takes each tile id from one device-wide counter (sched[0]) and
// hands it to the MMA and epilogue warps through a small queue in shared
// memory. Ids are taken in increasing order across the grid, so every gate_up
// tile has been taken by a running CTA before any down tile is: a down tile
// waits only on work already in progress, whichever CTAs are resident.
// A down tile's producer first issues the weight loads of up to a ring's worth
// of its K slices (the weights do not depend on h), then waits (bounded) until
// the epilogue warps of all gate_up tiles of its expert have stored their
// part of h and counted themselves in sched[1 + g], and then issues the loads
// of h. Each expert must hold at most NR rows (one row block); otherwise the
// launch records a device-check error and computes nothing.
template <int NR>
__device__ __forceinline__ Tile decode_mlp_tile(const SmemS<NR>& s, const Params& p, int id, int total1,
                                                bool& down) {
    down = id >= total1;
    if (!down) return decode_tile<false>(s, p, id, NR);
    const int local = id - total1;
    const int q = local / p.n_blocks2;                      // q-th expert with rows
    Tile t = decode_tile<false>(s, p, q * p.n_blocks, NR);  // its (only) row block
    t.n_blk = local - q * p.n_blocks2;
    t.num_kb = (p.I + BK - 1) / BK;
    return t;
}

template <int NR>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_swap_mlp_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWgu,
                         const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmWd,
                         const Params p) {
    extern __shared__ uint8_t smem_raw[];
    using Cfg = SwapCfg<NR>;
    SmemS<NR>& s = *reinterpret_cast<SmemS<NR>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &s.abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::kStages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.acc_full[i], 1);
            mbar_init(&s.acc_empty[i], kEpiWarps);
            mbar_init(&s.xchg[i], kEpiWarps / 2);
        }
        for (int i = 0; i < kTileQ; ++i) {
            mbar_init(&s.tq_full[i], 1);
            mbar_init(&s.tq_empty[i], 1 + kEpiWarps);   // the MMA warp and each epilogue warp
        }
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmWgu);
        prefetch_tensormap(&tmH);
        prefetch_tensormap(&tmWd);
    }
    if (warp == 1) {
        tmem_alloc(&s.tmem_base, Cfg::kTmemCols);
        tmem_relinquish();
    }
    pdl_wait();                // the previous kernels' outputs (token rows, offsets, zeroed counters) are complete
    build_schedule<false>(s, p, NR);
    bool bad = false;
    for (int g = threadIdx.x; g < p.groups; g += blockDim.x) bad = bad || s.off[g + 1] - s.off[g] > NR;
    bad = __syncthreads_or(bad) != 0;
    if (bad && blockIdx.x == 0 && threadIdx.x == 0) raise_error(p.err, kErrDeviceCheck);
    const int total1 = bad ? 0 : s.total_tiles;                              // gate_up tiles
    const int total = total1 + (total1 / max(p.n_blocks, 1)) * p.n_blocks2;  // and the down tiles
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t loads = 0;   // stage loads issued; load j used stage j % kStages
            bool ok = true;
            for (int j = 0;; ++j) {
                const int slot = j % kTileQ;
                if (!mbar_wait(&s.tq_empty[slot], ((uint32_t)(j / kTileQ) & 1u) ^ 1u, abort_flag, p.err)) break;
                int id = atomicAdd(p.sched, 1);
                if (id >= total) id = -1;
                s.tile_q[slot] = id;
                mbar_arrive(&s.tq_full[slot]);
                if (id < 0) break;
                bool down;
                const Tile t = decode_mlp_tile(s, p, id, total1, down);
                const CUtensorMap* mw = down ? &tmWd : &tmWgu;
                const CUtensorMap* mx = down ? &tmH : &tmX;
                // down tiles: the weight loads of the first `pre` K slices go out before h is ready
                const int pre = down ? min(t.num_kb, Cfg::kStages) : 0;
                const int stage0 = stage;
                int early = 0;   // early stages issued whose h loads are still to be issued
                // h of expert g is complete once every gate_up tile's 4 writer warps have
                // counted; then the early stages get their h loads (issued after a failed
                // wait too, so that every issued stage completes; the error is recorded)
                auto load_h_early = [&](bool wait) {
                    if (early == 0) return;
                    if (wait) ok = wait_count(p.sched + 1 + t.g, 4 * p.n_blocks, abort_flag, p.err);
                    fence_proxy_async_global();
                    int st2 = stage0;
                    for (int k2 = 0; k2 < early; ++k2) {
                        tma_load_2d(mx, &s.full[st2], s.stage[st2] + kStageAS, k2 * BK, t.row0);
                        if (++st2 == Cfg::kStages) st2 = 0;
                    }
                    early = 0;
                };
                for (int kb = 0; kb < t.num_kb; ++kb) {
                    if (kb == pre) load_h_early(true);
                    if (!ok) break;
                    if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* a_s = s.stage[stage];
                    uint64_t* bar = &s.full[stage];
                    mbar_arrive_expect_tx(bar, Cfg::kStage);   // weights and token rows
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(mw, bar, a_s + c * kChunkBytes,
                                    down ? w_col_swap<kEpiStore>(t, p, c) : w_col_swap<kEpiSwiglu>(t, p, c),
                                    kb * BK, t.g);
                    if (kb >= pre) tma_load_2d(mx, bar, a_s + kStageAS, kb * BK, t.row0);
                    else ++early;
                    ++loads;
                    if (++stage == Cfg::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                load_h_early(ok);   // every K slice was an early one, or a wait gave up
                if (!ok) break;
            }
            // every issued stage completes (its h load was issued too): wait for each
            // stage's last load, whatever the abort flag says, before the CTA may exit
            for (int i = 0; i < Cfg::kStages; ++i)
                if (loads > (uint32_t)i)
                    mbar_wait_bounded(&s.full[i], ((loads - 1 - (uint32_t)i) / Cfg::kStages) & 1u, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = instr_desc<128, NR, true, false>();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        bool any_mma = false;
        for (int j = 0; ok; ++j) {
            const int slot = j % kTileQ;
            if (!mbar_wait(&s.tq_full[slot], (uint32_t)(j / kTileQ) & 1u, abort_flag, p.err)) break;
            const int id = s.tile_q[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.tq_empty[slot]);
            if (id < 0) break;
            bool down;
            const Tile t = decode_mlp_tile(s, p, id, total1, down);
            const int buf = j & 1;
            const uint32_t use = (uint32_t)(j >> 1);
            if (!mbar_wait(&s.acc_empty[buf], (use & 1u) ^ 1u, abort_flag, p.err)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(buf * NR);
            for (int kb = 0; kb < t.num_kb; ++kb) {
                if (!mbar_wait(&s.full[stage], phase, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(s.stage[stage]);
                const uint32_t b_addr = a_addr + kStageAS;
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t adesc = smem_desc(a_addr + kk * 2048, kChunkBytes, 1024);
                        const uint64_t bdesc = smem_desc(b_addr + kk * 32, 16, 1024);
                        umma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(&s.empty[stage]);
                    any_mma = true;
                }
                __syncwarp();
                if (++stage == Cfg::kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(&s.acc_full[buf]);
            __syncwarp();
        }
        if (lane == 0 && any_mma) {
            umma_commit(&s.drain);
            mbar_wait_bounded(&s.drain, 0, p.err);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
        const int half = (warp - 2) / 4;            // token columns kWarpCols*half ..
        constexpr int kWC = Cfg::kWarpCols;
        // A CTA's ids increase, so its gate_up tiles come before its down tiles:
        // the hand-over barrier xchg[buf] is used by tiles j = buf, buf + 2, ...
        // of the gate_up run only, and its parity follows j >> 1.
        for (int j = 0;; ++j) {
            const int slot = j % kTileQ;
            if (!mbar_wait(&s.tq_full[slot], (uint32_t)(j / kTileQ) & 1u, abort_flag, p.err)) break;
            const int id = s.tile_q[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.tq_empty[slot]);
            if (id < 0) break;
            bool down;
            const Tile t = decode_mlp_tile(s, p, id, total1, down);
            const int buf = j & 1;
            const uint32_t use = (uint32_t)(j >> 1);
            if (!mbar_wait(&s.acc_full[buf], use & 1u, abort_flag, p.err)) break;
            tc_fence_after();
            float v[kWC];
            const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * NR + kWC * half);
            if constexpr (kWC == 32) tmem_load_32(taddr, v);
            else tmem_load_8(taddr, v);
            const int j0 = kWC * half;
            bool ok = true;
            if (!down) {
                ok = swap_epi_swiglu<NR>(s, p, t, buf, use, quarter, j0, lane, v, abort_flag);
                if (ok && quarter < 2) {
                    // this warp's part of expert g's h is stored: make it visible to
                    // other CTAs' TMA loads, then count it
                    __threadfence();
                    fence_proxy_async_global();
                    __syncwarp();
                    if (lane == 0) atomicAdd(p.sched + 1 + t.g, 1);
                }
            } else {
                swap_epi_store<NR>(p.y, p.ldy, p.N2, t, quarter, j0, lane, v);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.acc_empty[buf]);
            if (!ok) break;
        }
    }

    pdl_launch_dependents();   // every role has left its loop (see gemm_pair_kernel)
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
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
                 uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 tensor [d2][d1][d0], densely packed.
bool make_map_3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint32_t box0, uint32_t box1,
                 CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class K>
cudaError_t set_smem_once(K kern, size_t bytes, std::once_flag& once, cudaError_t& status) {
    std::call_once(once, [&] {
        status = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    });
    return status;
}

template <int EPI, bool B_MN>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& a64, const CUtensorMap& b, const Params& p,
                        int64_t max_tiles, cudaStream_t st, const CUtensorMap* c = nullptr,
                        const CUtensorMap* c2 = nullptr) {
    auto kern = gemm_pair_kernel<EPI, B_MN>;
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    if (set_smem_once(kern, kSmemPBytes, once, attr) != cudaSuccess) return attr;
    if (max_tiles <= 0) return cudaSuccess;
    int64_t clusters = sm_count() / 2;
    if (clusters > max_tiles) clusters = max_tiles;
    if (clusters < 1) clusters = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * clusters));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemPBytes;
    cfg.stream = st;
    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = 2;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see launch_chained
    attrs[1].val.programmaticStreamSerializationAllowed = chained_launches() ? 1 : 0;
    cfg.attrs = attrs;
    cfg.numAttrs = 2;
    CUtensorMap unused{};   // read only when q.tma_out / q.tma_out2 say so
    Params q = p;
    q.tma_out = c != nullptr;
    q.tma_out2 = c2 != nullptr;
    return cudaLaunchKernelEx(&cfg, kern, a, a64, b, c ? *c : unused, c2 ? *c2 : unused, q);
}

template <int EPI, bool A_MN, bool B_MN, bool GROUP_K>
cudaError_t launch_1cta(const CUtensorMap& a, const CUtensorMap& b, const Params& p,
                        int64_t max_tiles, cudaStream_t st, const CUtensorMap* c = nullptr,
                        const CUtensorMap* c2 = nullptr) {
    auto kern = gemm_1cta_kernel<EPI, A_MN, B_MN, GROUP_K>;
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    if (set_smem_once(kern, kSmem1Bytes, once, attr) != cudaSuccess) return attr;
    if (max_tiles <= 0) return cudaSuccess;
    int64_t grid = sm_count();
    if (grid > max_tiles) grid = max_tiles;
    CUtensorMap unused{};   // read only when p.tma_out / p.tma_out2 say so
    Params q = p;
    q.tma_out = c != nullptr;
    q.tma_out2 = c2 != nullptr;
    return launch_chained(kern, dim3((unsigned)grid), dim3(GROUP_K ? kThreadsK : kThreads), kSmem1Bytes, st, a, b,
                          c ? *c : unused, c2 ? *c2 : unused, q);
}

Params base_params(int groups, int64_t rows, const int32_t* offsets, unsigned* err) {
    Params p{};
    p.groups = groups;
    p.rows = (int)rows;
    p.offsets = offsets;
    p.err = err;
    return p;
}

// Upper bound of group-M pair tiles without reading the device counts.
int64_t pair_tile_bound(int64_t rows, int groups, int n_blocks) {
    return ((rows + BMP - 1) / BMP + groups) * (int64_t)n_blocks;
}

int64_t single_tile_bound(int64_t rows, int groups, int n_blocks) {
    return ((rows + BM1 - 1) / BM1 + groups) * (int64_t)n_blocks;
}

// Pair tiles (256 rows) halve each CTA's weight traffic; an expert block's
// last <= 128 rows run as a 128-row pair tile, so both kinds round a block up
// to a multiple of 128 rows. Measured on B200 with the two kinds interleaved
// call by call: pair tiles are faster at 1024 rows per expert (Mixtral-8x7B
// shape) and for one dense group (the Llama-4 shared expert: 1595 against
// 1727 us), equal at 512 (Llama-4-17Bx16E routed gate_up: 1339 against
// 1326 us), and slower at 256 (Qwen3-30B-A3B shape: 321 against 286 us).
// moe_testing_set_kernels can force either kind (the tests run both kernels
// on the same shapes).
bool use_pair_tiles(int64_t rows, int groups) {
    const int forced = kernel_override().gemm_tiles;
    if (forced == MOE_TESTING_GEMM_PAIR) return true;
    if (forced != MOE_TESTING_AUTO) return false;
    return groups == 1 || rows >= (int64_t)groups * 1024;
}

// The forward GEMMs take swap-AB tiles (weights as the 128-row operand, 64
// token rows per tile) when the expert blocks average at most 16 rows: a
// small batch, where 128-row token tiles would be mostly padding and too few
// to spread the weight reads over the SMs.
bool use_swap_tiles(int64_t rows, int groups) {
    const int forced = kernel_override().gemm_tiles;
    if (forced != MOE_TESTING_AUTO) return forced == MOE_TESTING_GEMM_SWAP || forced == MOE_TESTING_GEMM_SWAP_UNFUSED;
    return rows <= (int64_t)groups * 16;
}

template <int NR>
cudaError_t launch_mlp(const CUtensorMap& x_rows, const CUtensorMap& w_gate_up, const CUtensorMap& h_rows,
                       const CUtensorMap& w_down, const Params& p, int64_t grid, cudaStream_t st) {
    auto kern = gemm_swap_mlp_kernel<NR>;
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    if (set_smem_once(kern, swap_smem_bytes<NR>(), once, attr) != cudaSuccess) return attr;
    return launch_chained(kern, dim3((unsigned)grid), dim3(kThreads), swap_smem_bytes<NR>(), st, x_rows, w_gate_up,
                          h_rows, w_down, p);
}

template <int EPI, int NR>
cudaError_t launch_swap(const CUtensorMap& x_rows, const CUtensorMap& w, const Params& p, cudaStream_t st) {
    auto kern = gemm_swap_kernel<EPI, NR>;
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    if (set_smem_once(kern, swap_smem_bytes<NR>(), once, attr) != cudaSuccess) return attr;
    // upper bound of the tiles without reading the device counts
    const int64_t bound = ((int64_t)p.rows / NR + p.groups) * (int64_t)p.n_blocks;
    if (bound <= 0) return cudaSuccess;
    int64_t grid = sm_count();
    if (grid > bound) grid = bound;
    return launch_chained(kern, dim3((unsigned)grid), dim3(kThreads), swap_smem_bytes<NR>(), st, x_rows, w, p);
}

// Swap-AB launch with 16 token rows per tile when no group can hold more than
// 16 rows (max_group_rows), else 64. x is the token-row matrix [rows][K].
template <int EPI>
cudaError_t launch_swap_rows(const bf16* x, int64_t rows, int K, int64_t max_group_rows, const CUtensorMap& w,
                             const Params& p, cudaStream_t st) {
    CUtensorMap xm;
    if (max_group_rows <= 16) {
        if (!make_map_2d(&xm, x, K, rows, K, BK, 16)) return cudaErrorInvalidValue;
        return launch_swap<EPI, 16>(xm, w, p, st);
    }
    if (!make_map_2d(&xm, x, K, rows, K, BK, 64)) return cudaErrorInvalidValue;
    return launch_swap<EPI, 64>(xm, w, p, st);
}

// Group-M GEMM on pair or single tiles. `ta` and `ta64` are A maps with
// 128- and 64-row boxes (pair tiles of 256 and of 128 rows); `tb_pair` and
// `tb_single` are the B maps for each kernel (their K-major boxes differ: 128
// or 256 rows of N).
template <int EPI, bool B_MN>
cudaError_t launch_group_m(const CUtensorMap& ta, const CUtensorMap& ta64, const CUtensorMap& tb_pair,
                           const CUtensorMap& tb_single, const Params& p, cudaStream_t st,
                           const CUtensorMap* out_map, const CUtensorMap* out2_map = nullptr) {
    if (use_pair_tiles(p.rows, p.groups))
        return launch_pair<EPI, B_MN>(ta, ta64, tb_pair, p, pair_tile_bound(p.rows, p.groups, p.n_blocks), st,
                                      out_map, out2_map);
    return launch_1cta<EPI, false, B_MN, false>(ta, tb_single, p,
                                                single_tile_bound(p.rows, p.groups, p.n_blocks), st,
                                                out_map, out2_map);
}

// TMA store map of a row-major bf16 output [rows][cols]: 32 x 32 blocks, no swizzle.
bool make_out_map(CUtensorMap* m, const bf16* out, int64_t rows, uint64_t cols) {
    return make_map_2d(m, out, cols, (uint64_t)rows, cols, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

}  // namespace

cudaError_t gemm_gate_up_swiglu(const bf16* x, int64_t rows, const int32_t* offsets, int E, int H,
                                int I, const bf16* w_gate_up, bf16* h, bf16* gu_save,
                                cudaStream_t st, unsigned* err, const float* row_scale, int64_t max_group_rows) {
    if (max_group_rows <= 0 || max_group_rows > rows) max_group_rows = rows;
    if (rows == 0) return cudaSuccess;
    CUtensorMap ta, ta64, tb;
    if (!make_map_2d(&ta, x, H, rows, H, BK, 128)) return cudaErrorInvalidValue;
    if (!make_map_2d(&ta64, x, H, rows, H, BK, 64)) return cudaErrorInvalidValue;
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
    p.row_scale = row_scale;
    if (use_swap_tiles(rows, groups)) {
        p.n_blocks = (I + 63) / 64;   // 64 gate and the matching 64 up columns per tile
        return launch_swap_rows<kEpiSwiglu>(x, rows, H, max_group_rows, tb, p, st);
    }
    CUtensorMap tc, tc2;
    if (!make_out_map(&tc, h, rows, I)) return cudaErrorInvalidValue;
    if (gu_save && !make_out_map(&tc2, gu_save, rows, 2 * (uint64_t)I)) return cudaErrorInvalidValue;
    return launch_group_m<kEpiSwiglu, true>(ta, ta64, tb, tb, p, st, &tc, gu_save ? &tc2 : nullptr);
}

cudaError_t gemm_gate_up_swiglu_gather(const bf16* x, int64_t T, const int32_t* sorted_token, int64_t rows,
                                       const int32_t* offsets, int E, int H, int I, const bf16* w_gate_up, bf16* h,
                                       bf16* gu_save, cudaStream_t st, unsigned* err, const float* row_scale) {
    if (rows == 0) return cudaSuccess;
    if (H % 8 != 0 || (reinterpret_cast<uintptr_t>(x) & 15u) != 0 || !sorted_token || !offsets)
        return cudaErrorInvalidValue;
    CUtensorMap ta, tb;
    // a valid map for the kernel's signature; the A rows are gathered, not loaded through it
    if (!make_map_2d(&ta, x, H, T, H, BK, 128)) return cudaErrorInvalidValue;
    if (!make_map_3d(&tb, w_gate_up, 2 * (uint64_t)I, H, E, 64, BK)) return cudaErrorInvalidValue;
    Params p = base_params(E, rows, offsets, err);
    p.N = I;
    p.K = H;
    p.I = I;
    p.n_blocks = (I + BN / 2 - 1) / (BN / 2);
    p.out = h;
    p.ldo = I;
    p.out2 = gu_save;
    p.ldo2 = 2 * (int64_t)I;
    p.row_scale = row_scale;
    p.gather_x = x;
    p.gather_tok = sorted_token;
    p.gather_T = T;
    CUtensorMap tc, tc2;
    if (!make_out_map(&tc, h, rows, I)) return cudaErrorInvalidValue;
    if (gu_save && !make_out_map(&tc2, gu_save, rows, 2 * (uint64_t)I)) return cudaErrorInvalidValue;
    return launch_1cta<kEpiSwiglu, false, true, false>(ta, tb, p, single_tile_bound(rows, E, p.n_blocks), st, &tc,
                                                       gu_save ? &tc2 : nullptr);
}

bool use_fused_mlp(int64_t rows, int groups, int64_t max_group_rows, int I) {
    if (kernel_override().gemm_tiles == MOE_TESTING_GEMM_SWAP_UNFUSED) return false;
    if (!use_swap_tiles(rows, groups) || max_group_rows <= 0 || max_group_rows > 64 || groups > kMaxGroups)
        return false;
    if (kernel_override().gemm_tiles == MOE_TESTING_GEMM_SWAP) return true;
    // With fewer gate_up tiles than SMs, the SMs without one can stage only a
    // ring's worth of down weights before h is ready, and the rest of the down
    // tiles queue behind the gate_up tiles on the busy SMs: two launches, the
    // second on every SM, measured faster there (T = 1, Qwen3-30B-A3B shape:
    // 34.9 against 35.8 us a step).
    const int64_t experts = rows < groups ? rows : groups;   // at most this many hold rows
    return experts * ((I + 63) / 64) >= sm_count();
}

cudaError_t gemm_expert_mlp_fused(const bf16* x, int64_t rows, const int32_t* offsets, int E, int H, int I,
                                  const bf16* w_gate_up, const bf16* w_down, bf16* h, bf16* gu_save, bf16* y,
                                  int32_t* sched, int64_t max_group_rows, cudaStream_t st, unsigned* err) {
    if (rows == 0) return cudaSuccess;
    if (!offsets || !sched || max_group_rows <= 0 || max_group_rows > 64 || E > kMaxGroups)
        return cudaErrorInvalidValue;
    const int nr = max_group_rows <= 16 ? 16 : 64;
    CUtensorMap tx, th, twgu, twd;
    if (!make_map_2d(&tx, x, H, rows, H, BK, nr)) return cudaErrorInvalidValue;
    if (!make_map_2d(&th, h, I, rows, I, BK, nr)) return cudaErrorInvalidValue;
    if (!make_map_3d(&twgu, w_gate_up, 2 * (uint64_t)I, H, E, 64, BK)) return cudaErrorInvalidValue;
    if (!make_map_3d(&twd, w_down, H, I, E, 64, BK)) return cudaErrorInvalidValue;
    Params p = base_params(E, rows, offsets, err);
    p.N = I;
    p.K = H;
    p.I = I;
    p.n_blocks = (I + 63) / 64;   // gate_up: 64 gate and the matching 64 up columns per tile
    p.out = h;
    p.ldo = I;
    p.out2 = gu_save;
    p.ldo2 = 2 * (int64_t)I;
    p.y = y;
    p.ldy = H;
    p.N2 = H;
    p.n_blocks2 = (H + 127) / 128;   // down: 128 output columns per tile
    p.sched = sched;
    // at most min(E, rows) experts hold rows, each one row block
    const int64_t experts = rows < E ? rows : E;
    int64_t grid = experts * (p.n_blocks + p.n_blocks2);
    if (grid > sm_count()) grid = sm_count();
    return nr == 16 ? launch_mlp<16>(tx, twgu, th, twd, p, grid, st) : launch_mlp<64>(tx, twgu, th, twd, p, grid, st);
}

bool grouped_gemm_single_tiles(int64_t rows, int groups) {
    return !use_pair_tiles(rows, groups) && !use_swap_tiles(rows, groups);
}

cudaError_t gemm_down(const bf16* h, int64_t rows, const int32_t* offsets, int E, int H, int I,
                      const bf16* w_down, bf16* y, cudaStream_t st, unsigned* err, int64_t max_group_rows) {
    if (max_group_rows <= 0 || max_group_rows > rows) max_group_rows = rows;
    if (rows == 0) return cudaSuccess;
    CUtensorMap ta, ta64, tb;
    if (!make_map_2d(&ta, h, I, rows, I, BK, 128)) return cudaErrorInvalidValue;
    if (!make_map_2d(&ta64, h, I, rows, I, BK, 64)) return cudaErrorInvalidValue;
    if (!make_map_3d(&tb, w_down, H, I, offsets ? E : 1, 64, BK)) return cudaErrorInvalidValue;
    const int groups = offsets ? E : 1;
    Params p = base_params(groups, rows, offsets, err);
    p.N = H;
    p.K = I;
    p.n_blocks = (H + BN - 1) / BN;
    p.out = y;
    p.ldo = H;
    if (use_swap_tiles(rows, groups)) {
        p.n_blocks = (H + 127) / 128;   // 128 output columns per tile
        return launch_swap_rows<kEpiStore>(h, rows, I, max_group_rows, tb, p, st);
    }
    CUtensorMap tc;
    if (!make_out_map(&tc, y, rows, H)) return cudaErrorInvalidValue;
    return launch_group_m<kEpiStore, true>(ta, ta64, tb, tb, p, st, &tc);
}

bool grouped_gemm_pair_tiles(int64_t rows, int groups) {
    return use_pair_tiles(rows, groups) && !use_swap_tiles(rows, groups);
}

cudaError_t gemm_down_combine(const bf16* h, int64_t T, int H, int I, const bf16* w_down, const bf16* y_perm,
                              int64_t y_rows, const int32_t* row_of, const float* probs, int k, bf16* out,
                              cudaStream_t st, unsigned* err) {
    if (T == 0) return cudaSuccess;
    if (!grouped_gemm_pair_tiles(T, 1)) return cudaErrorNotSupported;
    CUtensorMap ta, ta64, tb;
    if (!make_map_2d(&ta, h, I, T, I, BK, 128)) return cudaErrorInvalidValue;
    if (!make_map_2d(&ta64, h, I, T, I, BK, 64)) return cudaErrorInvalidValue;
    if (!make_map_3d(&tb, w_down, H, I, 1, 64, BK)) return cudaErrorInvalidValue;
    Params p = base_params(1, T, nullptr, err);
    p.N = H;
    p.K = I;
    p.n_blocks = (H + BN - 1) / BN;
    p.out = out;
    p.ldo = H;
    p.add_rows = y_perm;
    p.add_row_of = row_of;
    p.add_prob = probs;
    p.add_k = k;
    p.add_nrows = y_rows;
    CUtensorMap tc;
    if (!make_out_map(&tc, out, T, H)) return cudaErrorInvalidValue;
    return launch_pair<kEpiStoreAdd, true>(ta, ta64, tb, p, pair_tile_bound(T, 1, p.n_blocks), st, &tc);
}

cudaError_t gemm_down_dgrad_swiglu(const bf16* dy, int64_t rows, const int32_t* offsets, int E,
                                   int H, int I, const bf16* w_down, const bf16* gu, bf16* dgu,
                                   cudaStream_t st, unsigned* err, const float* row_scale, float* row_dot) {
    if (rows == 0) return cudaSuccess;
    CUtensorMap ta, ta64, tb;
    if (!make_map_2d(&ta, dy, H, rows, H, BK, 128)) return cudaErrorInvalidValue;
    if (!make_map_2d(&ta64, dy, H, rows, H, BK, 64)) return cudaErrorInvalidValue;
    // B[n = i][k = h] = w_down[e][i][h]: K-major, box 64 (h) x 128 (i) per CTA of a
    // pair, 64 x 256 for a single CTA
    CUtensorMap tb1;
    if (!make_map_3d(&tb, w_down, H, I, E, BK, BN / 2)) return cudaErrorInvalidValue;
    if (!make_map_3d(&tb1, w_down, H, I, E, BK, BN)) return cudaErrorInvalidValue;
    Params p = base_params(E, rows, offsets, err);
    p.N = I;
    p.K = H;
    p.I = I;
    p.n_blocks = (I + BN - 1) / BN;
    p.out = dgu;
    p.ldo = 2 * (int64_t)I;
    p.aux = gu;
    p.ld_aux = 2 * (int64_t)I;
    if (row_dot) {
        p.row_scale = row_scale;
        p.row_dot = row_dot;
        p.ld_row_dot = (I + 63) / 64;
    }
    CUtensorMap tc;
    if (!make_out_map(&tc, dgu, rows, 2 * (uint64_t)I)) return cudaErrorInvalidValue;
    return launch_group_m<kEpiSwigluBwd, false>(ta, ta64, tb, tb1, p, st, &tc);
}

cudaError_t gemm_gate_up_dgrad(const bf16* dgu, int64_t rows, const int32_t* offsets, int E, int H,
                               int I, const bf16* w_gate_up, bf16* dx_perm, cudaStream_t st,
                               unsigned* err) {
    if (rows == 0) return cudaSuccess;
    CUtensorMap ta, ta64, tb;
    if (!make_map_2d(&ta, dgu, 2 * (uint64_t)I, rows, 2 * (uint64_t)I, BK, 128))
        return cudaErrorInvalidValue;
    if (!make_map_2d(&ta64, dgu, 2 * (uint64_t)I, rows, 2 * (uint64_t)I, BK, 64))
        return cudaErrorInvalidValue;
    // B[n = h][k = c] = w_gate_up[e][h][c]: K-major, box 64 (c) x 128 (h) per CTA of a
    // pair, 64 x 256 for a single CTA
    CUtensorMap tb1;
    if (!make_map_3d(&tb, w_gate_up, 2 * (uint64_t)I, H, E, BK, BN / 2)) return cudaErrorInvalidValue;
    if (!make_map_3d(&tb1, w_gate_up, 2 * (uint64_t)I, H, E, BK, BN)) return cudaErrorInvalidValue;
    Params p = base_params(E, rows, offsets, err);
    p.N = H;
    p.K = 2 * I;
    p.n_blocks = (H + BN - 1) / BN;
    p.out = dx_perm;
    p.ldo = H;
    CUtensorMap tc;
    if (!make_out_map(&tc, dx_perm, rows, H)) return cudaErrorInvalidValue;
    return launch_group_m<kEpiStore, false>(ta, ta64, tb, tb1, p, st, &tc);
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
    p.m_blocks = (M + BM1 - 1) / BM1;
    p.n_blocks = (N + BN - 1) / BN;
    p.out = dW;
    p.ldo = N;
    p.out_group_stride = (int64_t)M * N;
    CUtensorMap tc;   // dW [E][M][N], stored in 32 x 32 blocks without swizzle
    if (!make_map_3d(&tc, dW, N, M, E > 0 ? E : 1, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    // One 128 x 256 tile per CTA at a time. A kernel that kept each expert's
    // B rows in shared memory across M blocks measured slower at the
    // Qwen3-30B-A3B shape (313 against 288 us for the gate_up gradient): its
    // A ring had 3 stages and each item waited for its whole panel.
    return launch_1cta<kEpiStore, true, true, true>(ta, tb, p, (int64_t)E * p.m_blocks * p.n_blocks, st,
                                                   &tc);
}

}  // namespace moe
