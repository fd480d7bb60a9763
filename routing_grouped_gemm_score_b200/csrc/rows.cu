// rows.cu -- the row-moving kernels on bulk asynchronous copies: token
// dispatch (permute), and the weighted combine (also the token sum of the
// backward's dx rows, with weight 1).
//
// Transformer Engine "Mixture of Experts", sections Token dispatch, Token
// combine and Token probabilities:
//   permute:      x_perm[row(t,j)] = x[t]
//   combine:      out[t] = shared[t] + sum_j p[t,j] * y_perm[row_of[t,j]]
//
// Both move whole rows whose addresses come from a chain of index loads.
// Each block has one producer warp and four consumer warps (permute: one).
// The producer reads the routing of its tokens a chunk ahead and brings each
// unit's rows into a ring of shared-memory stages with cp.async.bulk, which
// completes on the stage's mbarrier. Combine's consumers compute from shared
// memory and store 16-byte vectors to global memory; permute writes its k
// copies of a row with bulk stores straight from shared memory. A unit is a
// column piece of one token, sized so that a stage holds about 16 KB; a block
// takes a contiguous range of tokens and each token's pieces in order. Each
// output element has a single writer and a fixed order of operations: shared
// first, then j ascending, in fp32.
//
// Every wait is bounded (kWaitLimitNs). A timeout records MOE_ERR_TIMEOUT and
// stops both roles. The producer then waits, again bounded, for the copies it
// has issued before the block exits.
#include <mutex>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kConsumerWarps = 4;
constexpr int kRowsThreads = 32 * (1 + kConsumerWarps);
constexpr int kConsumerThreads = 32 * kConsumerWarps;
constexpr int kMaxStages = 8;
constexpr uint32_t kStageBudget = 16u * 1024;    // one stage: the row pieces of a unit
constexpr uint32_t kBlockBudget = 48u * 1024;    // all stages of a block: four blocks per SM
constexpr int kMaxBlocksPerSm = 4;
constexpr int kRouteEntries = 128;              // assignments per routing chunk

enum RowsMode { kPermute = 0, kCombine = 1 };

struct RowsJob {
    int64_t T;
    int k, H;
    int64_t A;
    const bf16* src;        // rows gathered by index (combine): y_perm [A,H]
    const bf16* tok;        // the token-order row: shared (combine, may be null) or x (permute)
    const int32_t* row_of;  // [T,k] (combine)
    const float* probs;     // [T,k]; null: weight 1 (combine)
    bf16* out;              // combine: out [T,H]; permute: x_perm [A,H]
    // permute: where each assignment goes
    const int32_t* topk_idx;
    const int32_t* offsets;
    int E;
    const int32_t* block_base;
    int nb, tpb;
    const int32_t* local_rank;
    int32_t* sorted_token;
    int32_t* row_of_out;
    unsigned* err;
    // geometry, set by the launcher
    int cols, pieces, stages;
    uint32_t slot_bytes, stage_bytes;
};

struct StageMeta {
    float p[16];
    int32_t row[16];
    uint32_t valid;     // bit j: assignment j has a row
    uint32_t pad[31];
};
static_assert(sizeof(StageMeta) == 256, "stage metadata is 256 bytes");

// Shared memory: barriers and flags | per-stage metadata | routing tables
// (2 x rows, 2 x weights) | expert offsets | data stages.
constexpr uint32_t kMetaOffset = 256;
constexpr uint32_t kRouteOffset = kMetaOffset + kMaxStages * sizeof(StageMeta);
constexpr uint32_t kOffsOffset = kRouteOffset + 4 * kRouteEntries * 4;
constexpr uint32_t kDataOffset = (kOffsOffset + 260 * 4 + 127) & ~127u;

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Bounded wait used at exit: ignores the abort flag, only the time limit.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, unsigned* err) {
    if (mbar_try_wait(bar, parity)) return;
    const unsigned long long start = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - start > kWaitLimitNs) {
            raise_error(err, kErrTimeout);
            return;
        }
    }
}

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about `ns` nanoseconds pass, instead of polling.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Bounded wait that sleeps between checks (see mbar_wait for the bounds).
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                unsigned* err) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    const unsigned long long start = global_timer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (*abort) return false;
        if (global_timer_ns() - start > kWaitLimitNs) {
            raise_error(err, kErrTimeout);
            *abort = 1;
            return false;
        }
    }
}

// One lane waits (bounded), the warp follows its verdict.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          unsigned* err, int lane) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait_sleep(bar, parity, abort, err);
    ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

__device__ __forceinline__ void add_scaled(float (&acc)[8], const uint4& v, float p) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = unpack_bf16x2(w[i]);
        acc[2 * i] += p * f.x;
        acc[2 * i + 1] += p * f.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float (&acc)[8]) {
    return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                      pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
}

// The producer reads the routing of its tokens in chunks of up to
// kRouteEntries assignments (4 per lane, coalesced), one chunk ahead of use,
// into a double-buffered table in shared memory: rt_a holds the source row
// (gather modes) or the destination row (permute) of each assignment of the
// chunk, rt_p its weight.
struct RouteRegs {
    int32_t a[4];
    int32_t b[4];
};

__device__ __forceinline__ int chunk_tokens(int k) { return kRouteEntries / k; }

// Gather modes: row_of and probs of the chunk's assignments.
__device__ __forceinline__ RouteRegs load_gather(const RowsJob& j, int64_t t0, int n, int lane) {
    RouteRegs r;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = lane + 32 * q;
        r.a[q] = -1;
        r.b[q] = __float_as_int(1.0f);
        if (e < n) {
            r.a[q] = __ldg(j.row_of + t0 * j.k + e);
            if (j.probs) r.b[q] = __float_as_int(__ldg(j.probs + t0 * j.k + e));
        }
    }
    return r;
}

__device__ __forceinline__ void store_gather(const RouteRegs& r, int32_t* rt_a, float* rt_p, int n, int lane) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = lane + 32 * q;
        if (e < n) {
            rt_a[e] = r.a[q];
            rt_p[e] = __int_as_float(r.b[q]);
        }
    }
}

// Permute, level 1: expert and rank of each assignment.
__device__ __forceinline__ RouteRegs load_perm1(const RowsJob& j, int64_t t0, int n, int lane) {
    RouteRegs r;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = lane + 32 * q;
        r.a[q] = -1;
        r.b[q] = -1;
        if (e < n) {
            r.a[q] = __ldg(j.topk_idx + t0 * j.k + e);
            r.b[q] = __ldg(j.local_rank + t0 * j.k + e);
        }
    }
    return r;
}

// Permute, level 2: the prefix of the assignment's token block inside its expert.
__device__ __forceinline__ void load_perm2(const RowsJob& j, int64_t t0, int n, const RouteRegs& l1, int lane,
                                           int32_t (&base)[4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = lane + 32 * q;
        base[q] = 0;
        if (e < n && l1.a[q] >= 0 && l1.a[q] < j.E) {
            const int64_t t = t0 + e / j.k;
            base[q] = __ldg(j.block_base + (int64_t)l1.a[q] * j.nb + t / j.tpb);
        }
    }
}

// Permute: destination rows offsets[e] + base + rank, checked against the
// expert's block; also written out as row_of and sorted_token.
__device__ __forceinline__ void store_perm(const RowsJob& j, int64_t t0, int n, const RouteRegs& l1,
                                           const int32_t (&base)[4], const int32_t* s_off, int32_t* rt_a,
                                           int lane) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = lane + 32 * q;
        if (e >= n) continue;
        const int ex = l1.a[q], rank = l1.b[q];
        int32_t row = -1;
        if (ex >= 0 && ex < j.E && rank >= 0) {
            const int64_t r = (int64_t)s_off[ex] + base[q] + rank;
            if (r >= s_off[ex] && r < s_off[ex + 1] && r < j.A) row = (int32_t)r;
        }
        if (row < 0) raise_error(j.err, kErrDeviceCheck);
        rt_a[e] = row;
        j.row_of_out[t0 * j.k + e] = row;
        if (row >= 0) j.sorted_token[row] = (int32_t)(t0 + e / j.k);
    }
}

__device__ __forceinline__ void block_tokens(const RowsJob& j, int64_t& t_begin, int64_t& t_end) {
    const int64_t per = (j.T + gridDim.x - 1) / gridDim.x;
    t_begin = (int64_t)blockIdx.x * per;
    t_end = t_begin + per < j.T ? t_begin + per : j.T;
}

template <int MODE>
__device__ void rows_producer(const RowsJob& j, uint64_t* full, uint64_t* empty, volatile int* abort,
                              StageMeta* meta, uint8_t* data, int32_t* rt_a, float* rt_p, int32_t* s_off,
                              int lane) {
    const int S = j.stages;
    const int k = j.k;
    int64_t t_begin, t_end;
    block_tokens(j, t_begin, t_end);
    const int C = chunk_tokens(k);
    auto chunk_n = [&](int64_t t0) -> int {   // assignments in the chunk starting at t0
        if (t0 >= t_end) return 0;
        const int64_t nt = t_end - t0 < C ? t_end - t0 : C;
        return (int)nt * k;
    };
    const bool tok_row = MODE != kCombine || j.tok != nullptr;
    const int tok_slots = tok_row ? 1 : 0;

    // routing pipeline: the table for chunk c is complete when chunk c starts
    RouteRegs P, R;       // permute: level 1 of chunks c+1 and c+2; gather: R = chunk c+1
    int32_t Q[4];         // permute: level 2 of chunk c+1
    if (t_begin < t_end) {
        if (MODE == kPermute) {
            for (int e = lane; e <= j.E; e += 32) s_off[e] = __ldg(j.offsets + e);
            __syncwarp();
            RouteRegs l1 = load_perm1(j, t_begin, chunk_n(t_begin), lane);
            int32_t b0[4];
            load_perm2(j, t_begin, chunk_n(t_begin), l1, lane, b0);
            store_perm(j, t_begin, chunk_n(t_begin), l1, b0, s_off, rt_a, lane);
            P = load_perm1(j, t_begin + C, chunk_n(t_begin + C), lane);
            load_perm2(j, t_begin + C, chunk_n(t_begin + C), P, lane, Q);
            R = load_perm1(j, t_begin + 2 * C, chunk_n(t_begin + 2 * C), lane);
        } else {
            store_gather(load_gather(j, t_begin, chunk_n(t_begin), lane), rt_a, rt_p, chunk_n(t_begin), lane);
            R = load_gather(j, t_begin + C, chunk_n(t_begin + C), lane);
        }
        __syncwarp();
    }
    int i = 0;   // units issued by this block
    bool stop = false;
    int buf = 0;
    for (int64_t c0 = t_begin; c0 < t_end && !stop; c0 += C, buf ^= 1) {
        const int ntok = chunk_n(c0) / k;
        const int32_t* ta = rt_a + buf * kRouteEntries;
        const float* tp = rt_p + buf * kRouteEntries;
        for (int tt = 0; tt < ntok && !stop; ++tt) {
            const int64_t t = c0 + tt;
            int32_t row = -1;
            float p = 1.0f;
            if (lane < k) {
                row = ta[tt * k + lane];
                if (MODE != kPermute) {
                    p = tp[tt * k + lane];
                    if (row < 0 || row >= j.A) row = -1;
                }
            }
            const bool has = lane < k && row >= 0;
            if (MODE != kPermute && lane < k && !has) raise_error(j.err, kErrDeviceCheck);
            const uint32_t valid = __ballot_sync(kFull, has);
            const uint32_t nrows = (MODE == kPermute ? 0u : (uint32_t)__popc(valid)) + (uint32_t)tok_slots;
            for (int piece = 0; piece < j.pieces; ++piece, ++i) {
                const int col0 = piece * j.cols;
                const int w = min(j.cols, j.H - col0);
                const int s = i % S;
                const uint32_t ph = (uint32_t)(i / S) & 1u;
                if (i >= S && !warp_wait(&empty[s], ph ^ 1u, abort, j.err, lane)) {
                    stop = true;
                    break;
                }
                StageMeta& m = meta[s];
                if (lane < k) {
                    m.p[lane] = p;
                    m.row[lane] = row;
                }
                if (lane == 0) m.valid = valid;
                const uint32_t piece_bytes = (uint32_t)w * 2u;
                if (lane == 0) mbar_expect_tx(&full[s], nrows * piece_bytes);
                __syncwarp();
                uint8_t* st = data + (size_t)s * j.stage_bytes;
                if (MODE != kPermute && has)
                    bulk_load(st + (size_t)(tok_slots + lane) * j.slot_bytes, j.src + (int64_t)row * j.H + col0,
                              piece_bytes, &full[s]);
                if (lane == 31 && tok_row) bulk_load(st, j.tok + t * j.H + col0, piece_bytes, &full[s]);
                mbar_arrive(&full[s]);   // 32 arrivals: the metadata stores of every lane are released
            }
        }
        // the next chunk's table (its loads were issued a chunk ago), then the
        // loads for the chunk after it
        const int64_t c1 = c0 + C, c2 = c0 + 2 * C, c3 = c0 + 3 * C;
        int32_t* na = rt_a + (buf ^ 1) * kRouteEntries;
        if (MODE == kPermute) {
            store_perm(j, c1, chunk_n(c1), P, Q, s_off, na, lane);
            P = R;
            load_perm2(j, c2, chunk_n(c2), P, lane, Q);
            R = load_perm1(j, c3, chunk_n(c3), lane);
        } else {
            store_gather(R, na, rt_p + (buf ^ 1) * kRouteEntries, chunk_n(c1), lane);
            R = load_gather(j, c2, chunk_n(c2), lane);
        }
        __syncwarp();
    }
    // wait for the copies of the stages still in flight (bounded), so none
    // lands after the block has left
    if (lane == 0)
        for (int q = i - S < 0 ? 0 : i - S; q < i; ++q)
            mbar_wait_drain(&full[q % S], (uint32_t)(q / S) & 1u, j.err);
    __syncwarp();
}

__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Permute's consumer: one warp; lane j writes the stage's row to destination
// j with a bulk store. A stage is released once the stores of the stage after
// it are issued and its own have been read out of shared memory.
__device__ void permute_storer(const RowsJob& j, uint64_t* full, uint64_t* empty, volatile int* abort,
                               const StageMeta* meta, const uint8_t* data, int lane) {
    const int S = j.stages;
    int i = 0;
    int prev_s = -1;
    int64_t t_begin, t_end;
    block_tokens(j, t_begin, t_end);
    for (int64_t t = t_begin; t < t_end; ++t) {
        bool ok = true;
        for (int piece = 0; piece < j.pieces; ++piece, ++i) {
            const int col0 = piece * j.cols;
            const int w = min(j.cols, j.H - col0);
            const int s = i % S;
            if (!warp_wait(&full[s], (uint32_t)(i / S) & 1u, abort, j.err, lane)) {
                ok = false;
                break;
            }
            const StageMeta& m = meta[s];
            if (lane < j.k && ((m.valid >> lane) & 1u))
                bulk_store(j.out + (int64_t)m.row[lane] * j.H + col0, data + (size_t)s * j.stage_bytes,
                           (uint32_t)w * 2u);
            bulk_commit();
            bulk_wait_read<1>();     // the previous stage's stores have read their data
            __syncwarp();
            if (prev_s >= 0 && lane == 0) mbar_arrive(&empty[prev_s]);
            prev_s = s;
        }
        if (!ok) break;
    }
    bulk_wait_all();   // every store issued by this lane has completed
    __syncwarp();
    if (prev_s >= 0 && lane == 0) mbar_arrive(&empty[prev_s]);
}

// Combine's consumer warps: shared + sum_j p_j y_j for each column chunk of
// the stage, in fp32, j in order, then one 16-byte store.
__device__ void rows_consumer(const RowsJob& j, uint64_t* full, uint64_t* empty, volatile int* abort,
                              const StageMeta* meta, const uint8_t* data, int cw, int lane) {
    const int S = j.stages;
    const int ct = cw * 32 + lane;                 // 0 .. kConsumerThreads-1
    const int H8 = j.H / 8;
    const int k = j.k;
    const int slot16 = (int)(j.slot_bytes / 16);
    uint4* out = reinterpret_cast<uint4*>(j.out);
    const bool tok_row = j.tok != nullptr;
    const int ts = tok_row ? 1 : 0;                // slot of the first gathered row
    int64_t t_begin, t_end;
    block_tokens(j, t_begin, t_end);
    int i = 0;
    for (int64_t t = t_begin; t < t_end; ++t) {
        for (int piece = 0; piece < j.pieces; ++piece, ++i) {
            const int col0 = piece * j.cols;
            const int w8 = min(j.cols, j.H - col0) / 8;
            const int s = i % S;
            if (!warp_wait(&full[s], (uint32_t)(i / S) & 1u, abort, j.err, lane)) return;
            const StageMeta& m = meta[s];
            const uint32_t valid = m.valid;
            const uint4* st = reinterpret_cast<const uint4*>(data + (size_t)s * j.stage_bytes);
            for (int c = ct; c < w8; c += kConsumerThreads) {
                float acc[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
                if (tok_row) add_scaled(acc, st[c], 1.0f);
                for (int jj = 0; jj < k; ++jj)
                    if ((valid >> jj) & 1u) add_scaled(acc, st[(ts + jj) * slot16 + c], m.p[jj]);
                out[t * H8 + col0 / 8 + c] = pack8(acc);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
}

template <int MODE>
__global__ void __launch_bounds__(kRowsThreads) rows_kernel(const RowsJob j) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    volatile int* abort = reinterpret_cast<volatile int*>(empty + kMaxStages);
    StageMeta* meta = reinterpret_cast<StageMeta*>(smem + kMetaOffset);
    int32_t* rt_a = reinterpret_cast<int32_t*>(smem + kRouteOffset);
    float* rt_p = reinterpret_cast<float*>(smem + kRouteOffset + 2 * kRouteEntries * 4);
    int32_t* s_off = reinterpret_cast<int32_t*>(smem + kOffsOffset);
    uint8_t* data = smem + kDataOffset;
    if (threadIdx.x == 0) {
        for (int s = 0; s < j.stages; ++s) {
            mbar_init(&full[s], 32);
            mbar_init(&empty[s], MODE == kPermute ? 1 : kConsumerWarps);
        }
        *abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        rows_producer<MODE>(j, full, empty, abort, meta, data, rt_a, rt_p, s_off, lane);
    } else {
        if constexpr (MODE == kPermute)
            permute_storer(j, full, empty, abort, meta, data, lane);   // launched with two warps
        else
            rows_consumer(j, full, empty, abort, meta, data, warp - 1, lane);
    }
}

// Column pieces and stages for rows of H bf16 with `slots` rows per unit.
void rows_geometry(RowsJob& j, int slots) {
    const uint32_t row_bytes = (uint32_t)j.H * 2u;
    int pieces = (int)(((uint64_t)slots * row_bytes + kStageBudget - 1) / kStageBudget);
    const int h64 = j.H / 64;
    if (pieces > h64) pieces = h64;
    const int cols = ((h64 + pieces - 1) / pieces) * 64;
    pieces = (j.H + cols - 1) / cols;
    j.cols = cols;
    j.pieces = pieces;
    j.slot_bytes = (uint32_t)cols * 2u;
    j.stage_bytes = (uint32_t)slots * j.slot_bytes;
    int stages = (int)(kBlockBudget / j.stage_bytes);
    stages = stages < 2 ? 2 : (stages > kMaxStages ? kMaxStages : stages);
    j.stages = stages;
}

template <int MODE>
cudaError_t rows_launch(RowsJob& j, cudaStream_t st) {
    const size_t smem = kDataOffset + (size_t)j.stages * j.stage_bytes + 128;
    // the shared-memory limit is a per-device attribute of the kernel
    constexpr int kMaxDev = 64;
    static std::once_flag once[kMaxDev];
    static cudaError_t status[kMaxDev];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [dev] {
        status[dev] = cudaFuncSetAttribute(rows_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           227 * 1024);
    });
    if (status[dev] != cudaSuccess) return status[dev];
    // blocks per SM by shared memory (228 KB per SM, 1 KB reserved per block)
    int per_sm = (int)((228u * 1024u) / (smem + 1024u));
    per_sm = per_sm < 1 ? 1 : (per_sm > kMaxBlocksPerSm ? kMaxBlocksPerSm : per_sm);
    int64_t grid = (int64_t)sm_count() * per_sm;
    if (grid > j.T) grid = j.T;
    if (grid < 1) return cudaSuccess;
    rows_kernel<MODE><<<(unsigned)grid, MODE == kPermute ? 64 : kRowsThreads, smem, st>>>(j);
    return cudaGetLastError();
}

RowsJob base_job(int64_t T, int k, int H, int64_t A, unsigned* err) {
    RowsJob j{};
    j.T = T;
    j.k = k;
    j.H = H;
    j.A = A;
    j.err = err;
    return j;
}

}  // namespace

bool rows_combine(const bf16* y_perm, const int32_t* row_of, const float* probs, int64_t T, int k, int H,
                  int64_t A, const bf16* shared, bf16* out, cudaStream_t st, unsigned* err, cudaError_t* res) {
    RowsJob j = base_job(T, k, H, A, err);
    rows_geometry(j, k + (shared ? 1 : 0));
    j.src = y_perm;
    j.tok = shared;
    j.row_of = row_of;
    j.probs = probs;
    j.out = out;
    *res = rows_launch<kCombine>(j, st);
    return true;
}

bool rows_permute(const bf16* x, int64_t T, int H, const int32_t* topk_idx, int k, const int32_t* offsets, int E,
                  const int32_t* block_base, int nb, int tpb, const int32_t* local_rank, bf16* x_perm,
                  int32_t* sorted_token, int32_t* row_of, int64_t A, cudaStream_t st, unsigned* err,
                  cudaError_t* res) {
    RowsJob j = base_job(T, k, H, A, err);
    rows_geometry(j, 1);
    j.tok = x;
    j.out = x_perm;
    j.topk_idx = topk_idx;
    j.offsets = offsets;
    j.E = E;
    j.block_base = block_base;
    j.nb = nb;
    j.tpb = tpb;
    j.local_rank = local_rank;
    j.sorted_token = sorted_token;
    j.row_of_out = row_of;
    *res = rows_launch<kPermute>(j, st);
    return true;
}

}  // namespace moe
