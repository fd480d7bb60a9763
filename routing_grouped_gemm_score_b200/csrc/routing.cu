// routing.cu -- router (score function + top-k + routing weights), rank and
// expert-offset scan, the router's backward, the expert-bias update, and the
// permute (token dispatch) kernels, padded dispatch included.
//
// Transformer Engine "Mixture of Experts", sections Router, Token dispatch
// and Padding and alignment; te_mixtral.py TEMixtralSparseMoeBlock.forward.
//
// Design: one warp per token. A lane holds the scores of experts lane,
// lane+32, ... in registers. The k experts are picked in k rounds; each round
// is two single-instruction warp reductions: the largest order key (the score
// mapped to an unsigned integer that sorts like the float), then the lowest
// expert index among the lanes holding it, which breaks ties toward the lower
// index. The choice is made on the logit itself: softmax and sigmoid are
// increasing, so the ranking is the same and no rounding of the score
// function can create a tie. For large T a lane-per-token kernel makes the
// same choice with sorting networks (router_lane_kernel). Ranks inside each
// expert are counted per block of 8 to 64 tokens (route_tokens_per_block) in
// shared memory, in token order, and an exclusive scan over the token blocks
// turns them into global rows. Positions never come from atomics, so the
// permutation is the same on every run.
#include <cstdlib>
#include <mutex>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kRouteThreads = 256;  // 8 warps; a token block has 8..64 tokens
constexpr unsigned kFull = 0xFFFFFFFFu;

// Order-preserving map of a float to uint32: a larger float gives a larger
// key. NaN maps below -inf, and -0 maps like +0.
__device__ __forceinline__ uint32_t float_order_key(float s) {
    uint32_t b = __float_as_uint(s);
    if ((b & 0x7FFFFFFFu) > 0x7F800000u) return 0u;  // NaN
    if ((b & 0x7FFFFFFFu) == 0u) b = 0u;             // -0 -> +0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct RouterArgs {
    const float* logits;
    int64_t T;
    int E, k;
    int score_fn, renormalize;
    float scaling;
    const float* bias;
    int32_t* topk_idx;
    float* topk_prob;
    uint8_t* routing_map;
    int32_t* block_base;  // [E][nb]
    int32_t* local_rank;  // [T][k]
    unsigned* ticket;
    int nb;
    int tpb;   // tokens per block
    // a single token block (nb == 1) may also write the experts' counts and
    // offsets, so that no scan kernel follows (NULL: the scan kernel does)
    int32_t* counts;
    int32_t* offsets;
    int32_t* zero;   // with counts: zero[0 .. n_zero) is set to 0 as well
    int n_zero;
    // with counts and x_perm: the permute as well (rows of H8 16-byte chunks)
    const uint4* x;
    int H8;
    uint4* x_perm;
    int32_t* sorted_token;
    int32_t* row_of;
};

// After the token loop: thread e counts, in token order, the assignments of
// the block's tokens to expert e. sel[tt][e] holds j+1 if token tt chose e as
// its j-th expert, else 0.
__device__ __forceinline__ void rank_block(const uint8_t (*sel)[256], int64_t t0, int tpb,
                                           int E, int k, int32_t* local_rank,
                                           int32_t* block_base, int nb) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int cnt = 0;
        for (int tt = 0; tt < tpb; ++tt) {
            int v = sel[tt][e];
            if (v) {
                local_rank[(t0 + tt) * k + (v - 1)] = cnt;
                ++cnt;
            }
        }
        block_base[(int64_t)e * nb + blockIdx.x] = cnt;
    }
}

// Inverse of float_order_key for a key that came from a logit: key 0 (NaN)
// gives NaN, and -0 comes back as +0, which changes no routing weight.
__device__ __forceinline__ float order_key_to_float(uint32_t key) {
    if (key == 0u) return __uint_as_float(0x7FC00000u);
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Put slot j behind slot i unless j ranks strictly better (larger key, or the
// same key and a lower expert index).
__device__ __forceinline__ void order_pair(uint32_t& ki, uint32_t& ei, uint32_t& kj, uint32_t& ej) {
    const bool swap = kj > ki || (kj == ki && ej < ei);
    const uint32_t k0 = ki, e0 = ei;
    ki = swap ? kj : ki;
    ei = swap ? ej : ei;
    kj = swap ? k0 : kj;
    ej = swap ? e0 : ej;
}

// Sort a lane's slots best first. Networks: 1 pair for 2, 5 pairs for 4,
// Batcher's odd-even merge (19 pairs) for 8.
template <int SLOTS>
__device__ __forceinline__ void sort_slots(uint32_t (&so)[SLOTS], uint32_t (&se)[SLOTS]) {
    if constexpr (SLOTS == 2) {
        order_pair(so[0], se[0], so[1], se[1]);
    } else if constexpr (SLOTS == 4) {
        constexpr int net[5][2] = {{0, 1}, {2, 3}, {0, 2}, {1, 3}, {1, 2}};
#pragma unroll
        for (int c = 0; c < 5; ++c) order_pair(so[net[c][0]], se[net[c][0]], so[net[c][1]], se[net[c][1]]);
    } else if constexpr (SLOTS == 8) {
        constexpr int net[19][2] = {{0, 1}, {2, 3}, {4, 5}, {6, 7}, {0, 2}, {1, 3}, {4, 6},
                                    {5, 7}, {1, 2}, {5, 6}, {0, 4}, {1, 5}, {2, 6}, {3, 7},
                                    {2, 4}, {3, 5}, {1, 2}, {3, 4}, {5, 6}};
#pragma unroll
        for (int c = 0; c < 19; ++c) order_pair(so[net[c][0]], se[net[c][0]], so[net[c][1]], se[net[c][1]]);
    }
}

// Inclusive scan over the block (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ int block_inclusive_scan(int v, int* warp_tot, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(kFull, v, off);
        if (lane >= off) v += o;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(kFull, w, off);
            if (lane >= off) w += o;
        }
        if (lane < nw) warp_tot[lane] = w;
    }
    __syncthreads();
    if (warp > 0) v += warp_tot[warp - 1];
    total = warp_tot[nw - 1];
    __syncthreads();
    return v;
}

// Router, one warp per token. SLOTS = experts per lane (E <= 32*SLOTS). KC is
// the number of picks when fixed at compile time, or 0 for any k <= 16 given
// at run time.
template <int SLOTS, int KC>
__global__ void __launch_bounds__(kRouteThreads) router_topk_kernel(const RouterArgs a) {
    __shared__ uint8_t sel[kMaxTokensPerRouteBlock][256];
    __shared__ __align__(16) float wbuf[kRouteThreads / 32][32 * SLOTS];   // per warp: values to sum in order
    constexpr int KMAX = KC ? KC : 16;
    constexpr uint32_t kNone = 0xFFFFFFFFu;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = a.E, k = KC ? KC : a.k, tpb = a.tpb;
    for (int i = threadIdx.x; i < tpb * 256 / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(&sel[0][0])[i] = make_uint4(0, 0, 0, 0);
    pdl_wait();
    pdl_launch_dependents();
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.ticket = 0u;
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * tpb;
    float* wrow = wbuf[warp];

    for (int tt = warp; tt < tpb; tt += kRouteThreads / 32) {
        const int64_t t = t0 + tt;
        if (t >= a.T) break;
        const float* lrow = a.logits + t * E;
        float lv[SLOTS];
#pragma unroll
        for (int s = 0; s < SLOTS; ++s) {
            const int e = lane + 32 * s;
            lv[s] = e < E ? __ldg(lrow + e) : 0.0f;
        }
        // Selection keys; a slot beyond E has key 0 and index kNone, so it
        // ranks below every expert, a NaN one (key 0, real index) included.
        uint32_t so[SLOTS], se[SLOTS];
#pragma unroll
        for (int s = 0; s < SLOTS; ++s) {
            const int e = lane + 32 * s;
            float score = lv[s];
            if (a.bias) score = 1.0f / (1.0f + expf(-lv[s])) + __ldg(a.bias + (e < E ? e : 0));
            so[s] = e < E ? float_order_key(score) : 0u;
            se[s] = e < E ? (uint32_t)e : kNone;
        }
        sort_slots<SLOTS>(so, se);   // best first in each lane
        // k rounds: the largest head key, then the lowest expert index holding
        // it; the lane that owns the pick drops its head.
        int my_e = 0;
        uint32_t my_key = 0u, top0 = 0u;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (KC == 0 && j >= k) break;
            const uint32_t top = __reduce_max_sync(kFull, so[0]);
            const uint32_t e = __reduce_min_sync(kFull, so[0] == top ? se[0] : kNone);
            if (j == 0) top0 = top;
            my_e = lane == j ? (int)e : my_e;
            my_key = lane == j ? top : my_key;
            const bool win = lane == (int)(e & 31u);
#pragma unroll
            for (int s = 0; s + 1 < SLOTS; ++s) {
                so[s] = win ? so[s + 1] : so[s];
                se[s] = win ? se[s + 1] : se[s];
            }
            so[SLOTS - 1] = win ? 0u : so[SLOTS - 1];
            se[SLOTS - 1] = win ? kNone : se[SLOTS - 1];
        }
        const bool picks = lane < k;                 // lane j holds the j-th pick
        if (picks) sel[tt][my_e] = (uint8_t)(lane + 1);
        // logit of the pick: the key inverted, or reread when a bias shaped the key
        float my_l = 0.0f;
        if (picks) my_l = a.bias ? __ldg(lrow + my_e) : order_key_to_float(my_key);

        // routing weights (fp32), in the oracle's order of operations; sums
        // run in order over a per-warp row of shared memory
        __syncwarp();
        float p = 0.0f;
        if (a.score_fn == MOE_SCORE_SOFTMAX) {
            if (a.renormalize) {
                // the first pick holds the largest logit of the picks (or NaN)
                const float m = __shfl_sync(kFull, my_l, 0);
                const float ex = picks ? expf(my_l - m) : 0.0f;
                if (lane < KMAX) wrow[lane] = ex;
                __syncwarp();
                float sum = 0.0f;
#pragma unroll
                for (int j = 0; j < KMAX; ++j) sum += (KC || j < k) ? wrow[j] : 0.0f;
                p = ex / sum;
            } else {
                // softmax over all experts: row maximum (NaN if expert 0 is
                // NaN, as a scan from expert 0 gives), then the sum in expert order
                const bool nan0 = isnan(__shfl_sync(kFull, lv[0], 0));
                const float m = nan0 ? __uint_as_float(0x7FC00000u) : order_key_to_float(top0);
#pragma unroll
                for (int s = 0; s < SLOTS; ++s) {
                    const int e = lane + 32 * s;
                    wrow[e] = e < E ? expf(lv[s] - m) : 0.0f;
                }
                __syncwarp();
                float sum = 0.0f;
                const float4* w4 = reinterpret_cast<const float4*>(wrow);
                for (int q = 0; q < (E + 3) / 4; ++q) {
                    const float4 v = w4[q];
                    sum += v.x;
                    sum += v.y;
                    sum += v.z;
                    sum += v.w;
                }
                p = picks ? expf(my_l - m) / sum : 0.0f;
            }
        } else {
            const float sg = picks ? 1.0f / (1.0f + expf(-my_l)) : 0.0f;
            if (a.renormalize) {
                if (lane < KMAX) wrow[lane] = sg;
                __syncwarp();
                float sum = 0.0f;
#pragma unroll
                for (int j = 0; j < KMAX; ++j) sum += (KC || j < k) ? wrow[j] : 0.0f;
                p = sg / sum;
            } else {
                p = sg;
            }
        }
        p = p * a.scaling;
        if (picks) {
            a.topk_idx[t * k + lane] = my_e;
            a.topk_prob[t * k + lane] = p;
        }
        if (a.routing_map) {
            uint8_t* mrow = a.routing_map + t * E;
#pragma unroll
            for (int s = 0; s < SLOTS; ++s) {
                const int e = lane + 32 * s;
                if (e < E) mrow[e] = sel[tt][e] != 0 ? 1 : 0;
            }
        }
        __syncwarp();   // wrow and this token's sel row are settled before the next token
    }
    __syncthreads();
    rank_block(sel, t0, tpb, E, k, a.local_rank, a.block_base, a.nb);
    if (a.counts != nullptr) {
        // the only token block: its counts are the experts' counts (thread e
        // wrote expert e's in rank_block; E <= blockDim), the block's base rank
        // in each expert is 0, and the offsets are the counts' exclusive scan
        __shared__ int warp_tot[kRouteThreads / 32];
        const int e = threadIdx.x;
        const int cnt = e < E ? a.block_base[e] : 0;
        if (e < E) {
            a.counts[e] = cnt;
            a.block_base[e] = 0;
        }
        int total;
        const int incl = block_inclusive_scan(cnt, warp_tot, total);
        if (e < E) a.offsets[e + 1] = incl;
        if (e == 0) a.offsets[0] = 0;
        for (int i = threadIdx.x; i < a.n_zero; i += blockDim.x) a.zero[i] = 0;
        if (a.x_perm != nullptr) {
            // and the permute (TE Token dispatch): assignment (t, j) of expert e
            // goes to row offsets[e] + its rank among e's assignments; each x row
            // is read once and stored to its k rows
            __shared__ int s_off[kRouteThreads];
            __shared__ int s_row[kMaxTokensPerRouteBlock * 16];
            if (e < E) s_off[e] = incl - cnt;
            __syncthreads();
            const int nt = (int)min((int64_t)tpb, a.T - t0);
            for (int i = threadIdx.x; i < nt * k; i += blockDim.x) {
                const int64_t tj = t0 * k + i;
                const int r = s_off[a.topk_idx[tj]] + a.local_rank[tj];
                a.row_of[tj] = r;
                a.sorted_token[r] = (int32_t)(t0 + i / k);
                s_row[i] = r;
            }
            __syncthreads();
            const int H8 = a.H8;
            for (int idx = threadIdx.x; idx < nt * H8; idx += blockDim.x) {
                const int tt = idx / H8, c = idx - tt * H8;
                const uint4 v = __ldg(a.x + (t0 + tt) * H8 + c);
                for (int j = 0; j < k; ++j) a.x_perm[(int64_t)s_row[tt * k + j] * H8 + c] = v;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Router for large T, one lane per token. A block holds 256 tokens, a warp 32.
// The warp stages its tokens' logits in shared memory 32 experts at a time
// (one coalesced 16-byte load per lane per 4 rows; the next chunk's loads are
// in flight while the current chunk is sorted); each lane then reads its own
// token's row and keeps that token's best 8 experts in registers: every 8
// experts are sorted with Batcher's network (19 compare-exchanges) and merged
// into the running 8 with one bitonic step (8 pairs) and a bitonic clean
// (12 pairs).
//
// The sorting runs on 32-bit entries: the top bits of the score's signed
// order key, with the complement of the expert index in the low 7 bits (E <=
// 128) or 8 bits, so a compare-exchange is one integer max and one min.
// Between entries whose prefixes differ this is the exact selection order
// (larger score, then the lower index); entries that share a prefix are
// ordered by index alone, which is exact only when their scores are equal.
// The kernel therefore also keeps the entry just after the picks (for k = 8
// the best entry any merge dropped; for k < 8 the (k+1)-th of the running 8)
// and checks the neighbours (+0 and -0 count as one prefix):
//  - the last pick and that entry share a prefix, the best entry is +inf or
//    above (a NaN with the sign bit clear), or that entry is -inf or below (a
//    NaN with the sign bit set): the set of picks may be wrong, and the token
//    is selected again on 64-bit entries (full key, index) over its row in
//    global memory;
//  - otherwise, two picks share a prefix: the set is right, and the picks are
//    sorted again on full keys.
// Either way the picks are those of the warp kernel above, and the weights
// are computed from the picked logits in the same order of operations. The
// block's counts come from one bit per (expert, token) in shared memory: a
// token's rank inside its rank block (tpb tokens, as in the warp kernel) is a
// population count of the bits below it.
// Restrictions: E a multiple of 32 (up to 256), k <= 8, softmax weights
// renormalised over the picks or sigmoid weights, 16-byte aligned logits;
// other cases use the warp kernel.
constexpr int kLaneTokens = 256;                 // tokens (threads) per block
constexpr int64_t kLaneMinTokens = 32768;        // below this, the warp kernel (more blocks, lower latency)
constexpr int kLaneChunk = 32;                   // experts staged per step
constexpr int kLanePitch = kLaneChunk + 4;       // floats per staged row (conflict-free 16-byte reads)

// An exact selection entry as one 64-bit value: the order key above, the
// complement of the expert index below, so that a larger value ranks strictly
// better in the selection order (larger key, then the lower index). 0 ranks
// below every expert (key 0 with the largest index).
__device__ __forceinline__ uint64_t lane_entry(uint32_t key, uint32_t e) {
    return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - e);
}
__device__ __forceinline__ uint32_t lane_expert(uint64_t v) { return 0xFFFFFFFFu - (uint32_t)v; }

// Signed order key: a larger float gives a larger int. -0 sits one below +0,
// NaNs with the sign bit clear lie above +inf and the others below -inf.
__device__ __forceinline__ int32_t lane_skey(float s) {
    const int32_t b = __float_as_int(s);
    return b ^ ((b >> 31) & 0x7FFFFFFF);
}
// The 32-bit entry: the key's top 32 - ib bits, then the complement of the
// expert index in the low ib bits (ib = 7 for E <= 128, else 8).
struct LaneFmt {
    int ib;            // index bits
    int32_t hi_mask;   // ~((1 << ib) - 1)
    int32_t cmax;      // (1 << ib) - 1
};
__device__ __forceinline__ int32_t lane_entry32(float s, int e, const LaneFmt& f) {
    return (lane_skey(s) & f.hi_mask) | (f.cmax - e);
}
__device__ __forceinline__ int lane_expert32(int32_t v, const LaneFmt& f) { return f.cmax - (v & f.cmax); }
constexpr int32_t kLaneNone = INT32_MIN;                          // below every entry of a score
constexpr int32_t kLaneKeyPosInf = 0x7F800000;                    // signed order keys of +inf and -inf
constexpr int32_t kLaneKeyNegInf = (int32_t)0x807FFFFFu;
// Neighbours (a before b in the 32-bit order) whose exact order may differ:
// the same prefix, or the prefixes of -0 and +0.
__device__ __forceinline__ bool lane_close(int32_t a, int32_t b, int ib) {
    const int32_t pa = a >> ib, pb = b >> ib;
    return pa == pb || (pa == 0 && pb == -1);
}

// Larger / smaller of two entries: one integer max or min for 32-bit entries.
__device__ __forceinline__ int32_t lane_hi(int32_t a, int32_t b) { return max(a, b); }
__device__ __forceinline__ int32_t lane_lo(int32_t a, int32_t b) { return min(a, b); }
__device__ __forceinline__ uint64_t lane_hi(uint64_t a, uint64_t b) { return a > b ? a : b; }
__device__ __forceinline__ uint64_t lane_lo(uint64_t a, uint64_t b) { return a > b ? b : a; }

template <typename V>
__device__ __forceinline__ void lane_cx(V& a, V& b) {   // a := better, b := worse
    const V hi = lane_hi(a, b), lo = lane_lo(a, b);
    a = hi;
    b = lo;
}

template <typename V>
__device__ __forceinline__ void lane_sort8(V (&v)[8]) {
    constexpr int net[19][2] = {{0, 1}, {2, 3}, {4, 5}, {6, 7}, {0, 2}, {1, 3}, {4, 6},
                                {5, 7}, {1, 2}, {5, 6}, {0, 4}, {1, 5}, {2, 6}, {3, 7},
                                {2, 4}, {3, 5}, {1, 2}, {3, 4}, {5, 6}};
#pragma unroll
    for (int c = 0; c < 19; ++c) lane_cx(v[net[c][0]], v[net[c][1]]);
}

// Sorts a bitonic 8 best first (12 pairs).
template <typename V>
__device__ __forceinline__ void lane_clean8(V (&t)[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) lane_cx(t[i], t[i + 4]);
#pragma unroll
    for (int i = 0; i < 8; i += 4) {
        lane_cx(t[i], t[i + 2]);
        lane_cx(t[i + 1], t[i + 3]);
    }
#pragma unroll
    for (int i = 0; i < 8; i += 2) lane_cx(t[i], t[i + 1]);
}

// t (best first) := the best 8 of t and g (both best first). With DROP, drop
// also takes the best of the 8 entries left out.
template <bool DROP, typename V>
__device__ __forceinline__ void lane_merge8(V (&t)[8], const V (&g)[8], V& drop) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const V x = t[i], y = g[7 - i];
        t[i] = lane_hi(x, y);     // bitonic, holds the best 8
        if (DROP) drop = lane_hi(drop, lane_lo(x, y));
    }
    lane_clean8(t);
}

// The score that is ranked: the logit, or with an expert bias sigmoid(logit) + bias.
template <bool BIAS>
__device__ __forceinline__ float lane_score(float l, const float* bias, int e) {
    return BIAS ? 1.0f / (1.0f + expf(-l)) + __ldg(bias + e) : l;
}

// The exact picks of one token, best first: 64-bit entries over its row in
// global memory, 32 experts (eight 16-byte loads) in flight at a time. Out of
// line, so that the main loop's registers are not spent on this rare path.
template <bool BIAS>
__device__ __noinline__ void lane_exact_row(const float* __restrict__ row, int E, const float* __restrict__ bias,
                                            int* te) {
    uint64_t x[8], none = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = 0u;
    for (int c0 = 0; c0 < E; c0 += 32) {
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __ldg(reinterpret_cast<const float4*>(row + c0) + i);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const float l[8] = {v[2 * g].x, v[2 * g].y, v[2 * g].z, v[2 * g].w,
                                v[2 * g + 1].x, v[2 * g + 1].y, v[2 * g + 1].z, v[2 * g + 1].w};
            uint64_t gv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int e = c0 + 8 * g + q;
                gv[q] = lane_entry(float_order_key(lane_score<BIAS>(l[q], bias, e)), (uint32_t)e);
            }
            lane_sort8(gv);
            lane_merge8<false>(x, gv, none);
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) te[j] = (int)lane_expert(x[j]);
}

// A tie at the edge of the picks: the experts whose 32-bit prefix equals pb,
// the prefix of the last pick, compete for picks n_sure..k-1 (the picks
// before them have larger prefixes and stay). They are found in one pass over
// the row and ranked on 64-bit entries; te[n_sure..k) receives the best.
template <bool BIAS>
__device__ __noinline__ void lane_edge_picks(const float* __restrict__ row, int E, int k, int n_sure,
                                             const float* __restrict__ bias, LaneFmt fmt, int32_t pb, int* te) {
    uint64_t x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = 0u;
    for (int c0 = 0; c0 < E; c0 += 32) {
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __ldg(reinterpret_cast<const float4*>(row + c0) + i);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float4 w = v[i / 4];
            const float l = (i & 3) == 0 ? w.x : (i & 3) == 1 ? w.y : (i & 3) == 2 ? w.z : w.w;
            const int e = c0 + i;
            const float sc = lane_score<BIAS>(l, bias, e);
            if ((lane_entry32(sc, e, fmt) >> fmt.ib) == pb) {
                uint64_t y = lane_entry(float_order_key(sc), (uint32_t)e);
#pragma unroll
                for (int j = 0; j < 8; ++j) lane_cx(x[j], y);   // insert, keeping the best 8
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (j >= n_sure && j < k) te[j] = (int)lane_expert(x[j - n_sure]);
}

// The k picks te[0..k) sorted again on full keys (the set is right).
template <bool BIAS>
__device__ __noinline__ void lane_exact_picks(const float* __restrict__ row, int k, const float* __restrict__ bias,
                                              int* te) {
    uint64_t x[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        x[j] = j < k ? lane_entry(float_order_key(lane_score<BIAS>(__ldg(row + te[j]), bias, te[j])), (uint32_t)te[j])
                     : 0u;   // below every pick
    lane_sort8(x);
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (j < k) te[j] = (int)lane_expert(x[j]);
}

// Tokens of [lo, hi) (block-local indices, hi <= 256) whose bit is set in m[0..7].
__device__ __forceinline__ int lane_count(const uint32_t* m, int lo, int hi) {
    int c = 0;
    for (int w = lo >> 5; w <= (hi - 1) >> 5 && lo < hi; ++w) {
        uint32_t bits = m[w];
        const int b0 = w * 32;
        if (lo > b0) bits &= ~0u << (lo - b0);
        if (hi < b0 + 32) bits &= (hi - b0) > 0 ? (~0u >> (32 - (hi - b0))) : 0u;
        c += __popc(bits);
    }
    return c;
}

template <int KC, bool BIAS>
__global__ void __launch_bounds__(kLaneTokens, 3)
    router_lane_kernel(const RouterArgs a) {
    __shared__ __align__(16) float stage[kLaneTokens / 32][32][kLanePitch];   // 36 KB
    __shared__ uint32_t mask[256][kLaneTokens / 32];                          // 8 KB
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = a.E;
    const int64_t t0 = (int64_t)blockIdx.x * kLaneTokens;
    const int64_t t = t0 + threadIdx.x;
    const bool live = t < a.T;
    pdl_wait();
    pdl_launch_dependents();
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.ticket = 0u;
    for (int i = threadIdx.x; i < E * (kLaneTokens / 32); i += blockDim.x) (&mask[0][0])[i] = 0u;

    LaneFmt fmt;
    fmt.ib = E <= 128 ? 7 : 8;
    fmt.cmax = (1 << fmt.ib) - 1;
    fmt.hi_mask = ~fmt.cmax;
    int32_t top[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) top[i] = kLaneNone;
    int32_t drop = kLaneNone;
    float(*st)[kLanePitch] = stage[warp];
    const int64_t wrow0 = t0 + warp * 32;
    // lane -> rows 4i + lane/8 of the warp's 32, 16-byte column lane % 8 of the chunk
    float4 pf[8];
    auto load_chunk = [&](int c0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = 4 * i + (lane >> 3);
            pf[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (wrow0 + r < a.T)
                pf[i] = __ldg(reinterpret_cast<const float4*>(a.logits + (wrow0 + r) * E + c0) + (lane & 7));
        }
    };
    load_chunk(0);
    for (int c0 = 0; c0 < E; c0 += kLaneChunk) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            *reinterpret_cast<float4*>(&st[4 * i + (lane >> 3)][4 * (lane & 7)]) = pf[i];
        __syncwarp();
        if (c0 + kLaneChunk < E) load_chunk(c0 + kLaneChunk);   // in flight while this chunk is sorted
#pragma unroll
        for (int g = 0; g < kLaneChunk; g += 8) {
            const float4 v0 = *reinterpret_cast<const float4*>(&st[lane][g]);
            const float4 v1 = *reinterpret_cast<const float4*>(&st[lane][g + 4]);
            const float l[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            int32_t gv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) gv[q] = lane_entry32(lane_score<BIAS>(l[q], a.bias, c0 + g + q), c0 + g + q, fmt);
            lane_sort8(gv);
            if (c0 == 0 && g == 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) top[i] = gv[i];
            } else {
                lane_merge8<KC == 8>(top, gv, drop);
            }
        }
        __syncwarp();   // the stage is read before the next chunk overwrites it
    }

    // Where the 32-bit order may differ from the exact one. At the edge (the
    // last pick and the entry after it share a prefix, or an infinity or NaN
    // sits at either end) the set of picks itself may differ: the row is
    // selected again. Otherwise the picks are right and only neighbours that
    // share a prefix may be out of order: the picks are sorted again on full keys.
    const int k = KC;
    const int32_t next = KC == 8 ? drop : top[KC < 8 ? KC : 7];
    const bool edge = top[0] >= (kLaneKeyPosInf & fmt.hi_mask) || next <= (kLaneKeyNegInf | fmt.cmax) ||
                      lane_close(top[k - 1], next, fmt.ib);
    bool inner = false;
#pragma unroll
    for (int j = 0; j + 1 < KC; ++j) inner |= lane_close(top[j], top[j + 1], fmt.ib);
    int te[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) te[j] = lane_expert32(top[j], fmt);
    if ((edge || inner) && live) {
        int fix[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) fix[j] = te[j];
        const float* row = a.logits + t * E;
        const int32_t pb = top[k - 1] >> fmt.ib;
        // an infinity or NaN at either end, or the prefixes of -0 and +0 at the
        // edge: the whole row again on full keys
        const bool whole = top[0] >= (kLaneKeyPosInf & fmt.hi_mask) || next <= (kLaneKeyNegInf | fmt.cmax) ||
                           (edge && (pb == 0 || pb == -1));
        if (whole) {
            lane_exact_row<BIAS>(row, E, a.bias, fix);
        } else {
            if (edge) {
                int n_sure = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) n_sure += (j < k && (top[j] >> fmt.ib) != pb) ? 1 : 0;
                lane_edge_picks<BIAS>(row, E, k, n_sure, a.bias, fmt, pb, fix);
            }
            lane_exact_picks<BIAS>(row, k, a.bias, fix);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) te[j] = fix[j];
    }

    // routing weights from the picked logits, in the warp kernel's order of operations
    float lsel[8], p[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        lsel[j] = 0.0f;
        if (j < k && live) {
            const float l = __ldg(a.logits + t * E + te[j]);
            // without a bias the warp kernel works from the key: NaN comes back
            // as the canonical NaN and -0 as +0
            lsel[j] = BIAS ? l : order_key_to_float(float_order_key(l));
        }
    }
    if (a.score_fn == MOE_SCORE_SOFTMAX) {
        const float m = lsel[0];   // the first pick holds the largest logit of the picks (or NaN)
        float ex[8], sum = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            ex[j] = j < k ? expf(lsel[j] - m) : 0.0f;
            if (j < k) sum += ex[j];
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) p[j] = ex[j] / sum;
    } else {
        float sg[8], sum = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            sg[j] = j < k ? 1.0f / (1.0f + expf(-lsel[j])) : 0.0f;
            if (j < k) sum += sg[j];
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) p[j] = a.renormalize ? sg[j] / sum : sg[j];
    }
    const bool vec = KC == 8 &&
                     ((((uintptr_t)a.topk_idx) | ((uintptr_t)a.topk_prob) | ((uintptr_t)a.local_rank)) & 15u) == 0;
    if (live) {
        if (vec) {
            int4* ip = reinterpret_cast<int4*>(a.topk_idx + t * 8);
            float4* pp = reinterpret_cast<float4*>(a.topk_prob + t * 8);
            ip[0] = make_int4(te[0], te[1], te[2], te[3]);
            ip[1] = make_int4(te[4], te[5], te[6], te[7]);
            pp[0] = make_float4(p[0] * a.scaling, p[1] * a.scaling, p[2] * a.scaling, p[3] * a.scaling);
            pp[1] = make_float4(p[4] * a.scaling, p[5] * a.scaling, p[6] * a.scaling, p[7] * a.scaling);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j >= k) break;
                a.topk_idx[t * k + j] = te[j];
                a.topk_prob[t * k + j] = p[j] * a.scaling;
            }
        }
        if (a.routing_map) {
            uint4* mrow = reinterpret_cast<uint4*>(a.routing_map + t * E);
            for (int i = 0; i < E / 16; ++i) mrow[i] = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < k) a.routing_map[t * E + te[j]] = 1;
        }
    }

    // counts and ranks per rank block of tpb tokens
    __syncthreads();   // masks zeroed
    if (live) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < k) atomicOr(&mask[te[j]][warp], 1u << lane);
    }
    __syncthreads();
    const int tpb = a.tpb;
    if (live) {
        const int lo = (threadIdx.x / tpb) * tpb;
        int rk[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) rk[j] = j < k ? lane_count(mask[te[j]], lo, threadIdx.x) : 0;
        if (vec) {
            int4* rp = reinterpret_cast<int4*>(a.local_rank + t * 8);
            rp[0] = make_int4(rk[0], rk[1], rk[2], rk[3]);
            rp[1] = make_int4(rk[4], rk[5], rk[6], rk[7]);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < k) a.local_rank[t * k + j] = rk[j];
        }
    }
    const int nsub = kLaneTokens / tpb;
    const int64_t sb0 = t0 / tpb;
    for (int i = threadIdx.x; i < E * nsub; i += blockDim.x) {
        const int e = i / nsub, sb = i - e * nsub;
        if (sb0 + sb >= a.nb) continue;
        a.block_base[(int64_t)e * a.nb + sb0 + sb] = lane_count(mask[e], sb * tpb, (sb + 1) * tpb);
    }
}

// Router backward: dL/dlogits from dL/dtopk_prob, one warp per token, fp32.
// Lane j < k holds pick j: its expert, logit and g_j = scaling * dprob[t,j].
// The formulas per mode are those of the forward's weights differentiated
// with the selection held fixed (see moe_router_backward in the header).
template <int SLOTS>
__global__ void __launch_bounds__(kRouteThreads)
    router_backward_kernel(const float* __restrict__ logits, int64_t T, int E, int k, int score_fn,
                           int renormalize, float scaling, const int32_t* __restrict__ topk_idx,
                           const float* __restrict__ dprob, float* __restrict__ dlogits, unsigned* err) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const float* lrow = logits + t * E;
        int sel = -1;
        float g = 0.0f, lsel = 0.0f;
        if (lane < k) {
            sel = __ldg(topk_idx + t * k + lane);
            if (sel < 0 || sel >= E) {
                raise_error(err, kErrDeviceCheck);
                sel = -1;
            }
            g = scaling * __ldg(dprob + t * k + lane);
            if (sel >= 0) lsel = __ldg(lrow + sel);
        }
        const bool pick = sel >= 0;
        float dsel = 0.0f;          // gradient at this lane's pick
        float dall[SLOTS];          // softmax over all experts: gradient of every slot
#pragma unroll
        for (int s = 0; s < SLOTS; ++s) dall[s] = 0.0f;
        if (score_fn == MOE_SCORE_SOFTMAX && renormalize) {
            float m = pick ? lsel : -INFINITY;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
            const float ex = pick ? expf(lsel - m) : 0.0f;
            float sum = ex;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
            const float q = ex / sum;
            float c = q * g;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(kFull, c, off);
            dsel = q * (g - c);
        } else if (score_fn == MOE_SCORE_SOFTMAX) {
            float lv[SLOTS];
            float m = -INFINITY;
#pragma unroll
            for (int s = 0; s < SLOTS; ++s) {
                const int e = lane + 32 * s;
                lv[s] = e < E ? __ldg(lrow + e) : -INFINITY;
                m = fmaxf(m, lv[s]);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
            float sum = 0.0f;
#pragma unroll
            for (int s = 0; s < SLOTS; ++s) {
                lv[s] = lane + 32 * s < E ? expf(lv[s] - m) : 0.0f;   // exp, in place
                sum += lv[s];
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
            const float qsel = pick ? expf(lsel - m) / sum : 0.0f;
            float c = qsel * g;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(kFull, c, off);
#pragma unroll
            for (int s = 0; s < SLOTS; ++s) dall[s] = (lv[s] / sum) * (0.0f - c);
            dsel = qsel * (g - c);
        } else {
            const float sg = pick ? 1.0f / (1.0f + expf(-lsel)) : 0.0f;
            float ds = g;
            if (renormalize) {
                float S = sg;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) S += __shfl_xor_sync(kFull, S, off);
                float c = (sg / S) * g;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(kFull, c, off);
                ds = (g - c) / S;
            }
            // s (1 - s) with 1 - s = sigmoid(-l), accurate where s is near 1
            dsel = pick ? ds * sg * (1.0f / (1.0f + expf(lsel))) : 0.0f;
        }
        // the row: each slot's value, replaced by the pick's where it is a pick
        float v[SLOTS];
#pragma unroll
        for (int s = 0; s < SLOTS; ++s) v[s] = dall[s];
        for (int j = 0; j < k; ++j) {
            const int sj = __shfl_sync(kFull, sel, j);
            const float dj = __shfl_sync(kFull, dsel, j);
#pragma unroll
            for (int s = 0; s < SLOTS; ++s)
                if (lane + 32 * s == sj) v[s] = dj;
        }
        float* drow = dlogits + t * E;
#pragma unroll
        for (int s = 0; s < SLOTS; ++s) {
            const int e = lane + 32 * s;
            if (e < E) drow[e] = v[s];
        }
    }
}

// Expert-bias update (auxiliary-loss-free load balancing), one block of 256
// threads: delta_e = coeff * sign(mean(c) - c_e), decided exactly as
// sign(sum(c) - E c_e), then centred (mean of delta = coeff (n_below -
// n_above) / E) and added to the bias.
__global__ void __launch_bounds__(256)
    expert_bias_update_kernel(const int32_t* __restrict__ counts, int E, float coeff, float* __restrict__ bias) {
    __shared__ long long s_sum[8];
    __shared__ int s_net[8];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    const int c = e < E ? counts[e] : 0;
    long long sum = c;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
    if (lane == 0) s_sum[warp] = sum;
    __syncthreads();
    long long total = 0;
    for (int w = 0; w < 8; ++w) total += s_sum[w];
    const long long d = total - (long long)E * c;
    const int sgn = e < E ? (d > 0) - (d < 0) : 0;
    int net = sgn;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) net += __shfl_xor_sync(kFull, net, off);
    if (lane == 0) s_net[warp] = net;
    __syncthreads();
    int n = 0;
    for (int w = 0; w < 8; ++w) n += s_net[w];
    if (e < E) bias[e] = bias[e] + (coeff * (float)sgn - coeff * (float)n / (float)E);
}

// Rank pass for caller-supplied expert indices (moe_permute on its own).
__global__ void __launch_bounds__(kRouteThreads)
    rank_from_indices_kernel(const int32_t* __restrict__ topk_idx, int64_t T, int E, int k,
                             int32_t* local_rank, int32_t* block_base, unsigned* ticket, int nb,
                             int tpb, unsigned* err) {
    __shared__ uint8_t sel[kMaxTokensPerRouteBlock][256];
    for (int i = threadIdx.x; i < tpb * 256 / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(&sel[0][0])[i] = make_uint4(0, 0, 0, 0);
    if (blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0u;
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * tpb;
    for (int tt = threadIdx.x; tt < tpb; tt += blockDim.x) {
        const int64_t t = t0 + tt;
        if (t >= T) break;
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[t * k + j];
            local_rank[t * k + j] = -1;  // stays -1 for an invalid or repeated expert
            if (e < 0 || e >= E || sel[tt][e] != 0) {
                raise_error(err, kErrDeviceCheck);
                continue;
            }
            sel[tt][e] = (uint8_t)(j + 1);
        }
    }
    __syncthreads();
    rank_block(sel, t0, tpb, E, k, local_rank, block_base, nb);
}


constexpr int kScanPerThread = 8;   // values a scan thread holds per pass
// Shared-memory slot of value i of a pass: thread i / 8's run, one padding
// word per run, so that a warp reading its runs hits 32 different banks.
__device__ __forceinline__ int scan_slot(int i) { return (i / kScanPerThread) * (kScanPerThread + 1) + i % kScanPerThread; }

// One block per expert: exclusive scan of its per-token-block counts. The last
// block to finish also writes offsets (exclusive scan of the expert counts).
__global__ void __launch_bounds__(1024)
    expert_scan_kernel(int32_t* block_base, int nb, int E, int32_t* counts, int32_t* offsets,
                       unsigned* ticket, int32_t* zero, int n_zero) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ int warp_tot[32];
    __shared__ bool is_last;
    int carry_off = 0;
    const int e = blockIdx.x;
    int32_t* row = block_base + (int64_t)e * nb;
    __shared__ int s_v[(kScanPerThread + 1) * 1024];   // a run of 8 per thread, padded by one word
    int carry = 0;
    // kScanPerThread values per thread per pass: coalesced loads into shared
    // memory (all in flight at once), a serial scan of each thread's run, one
    // block scan of the run totals, coalesced stores
    const int span = kScanPerThread * (int)blockDim.x;
    for (int base = 0; base < nb; base += span) {
        const int n = nb - base < span ? nb - base : span;
#pragma unroll
        for (int j = 0; j < kScanPerThread; ++j) {
            const int i = j * (int)blockDim.x + threadIdx.x;
            s_v[scan_slot(i)] = i < n ? row[base + i] : 0;
        }
        __syncthreads();
        int run[kScanPerThread], sum = 0;
#pragma unroll
        for (int j = 0; j < kScanPerThread; ++j) {
            run[j] = sum;
            sum += s_v[threadIdx.x * (kScanPerThread + 1) + j];
        }
        int total;
        const int excl = carry + block_inclusive_scan(sum, warp_tot, total) - sum;
#pragma unroll
        for (int j = 0; j < kScanPerThread; ++j) s_v[threadIdx.x * (kScanPerThread + 1) + j] = excl + run[j];
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kScanPerThread; ++j) {
            const int i = j * (int)blockDim.x + threadIdx.x;
            if (i < n) row[base + i] = s_v[scan_slot(i)];
        }
        carry += total;
        __syncthreads();   // s_v is read before the next pass overwrites it
    }
    if (counts == nullptr) return;
    if (threadIdx.x == 0) {
        counts[e] = carry;
        __threadfence();
        const unsigned done = atomicAdd(ticket, 1u);
        is_last = (done == (unsigned)E - 1);
    }
    __syncthreads();
    if (!is_last) return;
    // last block: offsets = exclusive scan of all experts' counts, loaded in
    // parallel (L2, bypassing L1) and scanned across the block
    __threadfence();
    for (int base = 0; base < E; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int v = i < E ? __ldcg(counts + i) : 0;
        int total;
        const int incl = block_inclusive_scan(v, warp_tot, total);
        if (i < E) offsets[i + 1] = carry_off + incl;
        if (base == 0 && threadIdx.x == 0) offsets[0] = 0;
        carry_off += total;
    }
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero[i] = 0;
    if (threadIdx.x == 0) *ticket = 0u;
}

// The same scan for at most 32 token blocks (T <= 256 at 8 tokens a block), in
// one block and without the ticket: warp w scans the block counts of experts
// w, w + 32, ... with one value per lane, then the block scans the expert
// counts into the offsets. A small batch then pays for one block instead of E.
constexpr int kScanSmallBlocks = 32;
__global__ void __launch_bounds__(1024)
    expert_scan_small_kernel(int32_t* block_base, int nb, int E, int32_t* counts, int32_t* offsets, int32_t* zero,
                             int n_zero) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ int cnt[256];
    __shared__ int warp_tot[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int e = warp; e < E; e += nw) {
        int32_t* row = block_base + (int64_t)e * nb;
        const int v = lane < nb ? row[lane] : 0;
        int incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(kFull, incl, off);
            if (lane >= off) incl += o;
        }
        if (lane < nb) row[lane] = incl - v;
        if (lane == 31) cnt[e] = incl;
    }
    __syncthreads();
    if (counts == nullptr) return;
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = cnt[e];
    int carry = 0;
    for (int base = 0; base < E; base += blockDim.x) {   // E <= 256 < blockDim: one pass
        const int i = base + threadIdx.x;
        const int v = i < E ? cnt[i] : 0;
        int total;
        const int incl = block_inclusive_scan(v, warp_tot, total);
        if (i < E) offsets[i + 1] = carry + incl;
        if (base == 0 && threadIdx.x == 0) offsets[0] = 0;
        carry += total;
    }
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero[i] = 0;
}

// Permute over contiguous token ranges, on plain 16-byte loads and stores. A
// block owns tokens [t_begin, t_end). Its threads compute the destination rows
// of kPermStage assignments at a time (offsets[e] + block_base[e][t / tpb] +
// local_rank, checked against the expert's block; row_of and sorted_token are
// written here) into shared memory. Then each thread owns one 16-byte column
// chunk (blockDim = H/8 rounded up to a warp, H <= 4096), loads it for 4
// tokens at once and stores each to the token's k rows.
constexpr int kPermStage = 2048;

__global__ void __launch_bounds__(512)
    permute_tokens_kernel(const uint4* __restrict__ x, int64_t T, int H8, const int32_t* __restrict__ topk_idx,
                          int k, const int32_t* __restrict__ offsets, int E, const int32_t* __restrict__ block_base,
                          int nb, int tpb, const int32_t* __restrict__ local_rank, uint4* __restrict__ x_perm,
                          int32_t* __restrict__ sorted_token, int32_t* __restrict__ row_of, int64_t A,
                          int64_t per_block, unsigned* err) {
    __shared__ int32_t s_row[kPermStage];
    pdl_wait();
    pdl_launch_dependents();
    const int64_t t_begin = (int64_t)blockIdx.x * per_block;
    const int64_t t_end = t_begin + per_block < T ? t_begin + per_block : T;
    const int c = threadIdx.x;
    const bool active = c < H8;
    const int tok_per_stage = kPermStage / k;
    for (int64_t s0 = t_begin; s0 < t_end; s0 += tok_per_stage) {
        const int ntok = (int)(t_end - s0 < tok_per_stage ? t_end - s0 : tok_per_stage);
        __syncthreads();   // the previous stage's rows are no longer read
        for (int i = threadIdx.x; i < ntok * k; i += blockDim.x) {
            const int64_t t = s0 + i / k;
            const int e = __ldg(topk_idx + s0 * k + i);
            const int rank = __ldg(local_rank + s0 * k + i);
            int32_t row = -1;
            if (e >= 0 && e < E && rank >= 0) {
                const int64_t lo = __ldg(offsets + e), hi = __ldg(offsets + e + 1);
                const int64_t r = lo + __ldg(block_base + (int64_t)e * nb + t / tpb) + rank;
                if (r >= lo && r < hi && r < A) row = (int32_t)r;
            }
            if (row < 0) raise_error(err, kErrDeviceCheck);
            s_row[i] = row;
            row_of[s0 * k + i] = row;
            if (row >= 0) sorted_token[row] = (int32_t)t;
        }
        __syncthreads();
        if (!active || x_perm == nullptr) continue;   // no x_perm: the rows only
        for (int tt0 = 0; tt0 < ntok; tt0 += 4) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (tt0 + u < ntok) v[u] = __ldg(x + (s0 + tt0 + u) * H8 + c);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (tt0 + u >= ntok) break;
                for (int j = 0; j < k; ++j) {
                    const int32_t r = s_row[(tt0 + u) * k + j];
                    if (r >= 0) x_perm[(int64_t)r * H8 + c] = v[u];
                }
            }
        }
    }
}

// Dispatch, one warp per token. The destination rows of a token come three
// tokens deep in a software pipeline: its expert indices and ranks are loaded
// two tokens ahead, its block bases one token ahead, so when the token's turn
// comes the k rows are known (lane j holds row j) and the warp only copies:
// CH 16-byte chunks of the row per lane per step, each stored to the k rows.
// Expert offsets are cached in shared memory per block.
constexpr int kPermMaxExperts = 256;   // the ABI's bound on E

template <int KB, int CH>
__global__ void __launch_bounds__(256)
    permute_warp_kernel(const uint4* __restrict__ x, int64_t T, int H8, const int32_t* __restrict__ topk_idx,
                        int k, const int32_t* __restrict__ offsets, int E, const int32_t* __restrict__ block_base,
                        int nb, int tpb, const int32_t* __restrict__ local_rank, uint4* __restrict__ x_perm,
                        int32_t* __restrict__ sorted_token, int32_t* __restrict__ row_of, int64_t A,
                        unsigned* err) {
    __shared__ int32_t s_off[kPermMaxExperts + 1];
    pdl_wait();
    pdl_launch_dependents();
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = __ldg(offsets + e);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t t0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    // stage 2 (token t + 2 nw): expert and rank; stage 1 (token t + nw): block base
    auto load_er = [&](int64_t t, int& e, int& rk) {
        e = -1;
        rk = -1;
        if (t < T && lane < k) {
            e = __ldg(topk_idx + t * k + lane);
            rk = __ldg(local_rank + t * k + lane);
        }
    };
    auto load_bb = [&](int64_t t, int e) -> int {
        return (t < T && lane < k && e >= 0 && e < E) ? __ldg(block_base + (int64_t)e * nb + t / tpb) : 0;
    };
    auto make_row = [&](int64_t t, int e, int rk, int bb) -> int32_t {
        if (t >= T || lane >= k) return -1;
        int32_t row = -1;
        if (e >= 0 && e < E && rk >= 0) {
            const int64_t lo = s_off[e], hi = s_off[e + 1];
            const int64_t r = lo + bb + rk;
            if (r >= lo && r < hi && r < A) row = (int32_t)r;
        }
        if (row < 0) raise_error(err, kErrDeviceCheck);
        return row;
    };
    int e1, rk1, e2, rk2;
    load_er(t0, e1, rk1);
    const int bb1 = load_bb(t0, e1);
    int32_t row_cur = make_row(t0, e1, rk1, bb1);
    load_er(t0 + nw, e1, rk1);
    int bb_next = load_bb(t0 + nw, e1);
    load_er(t0 + 2 * nw, e2, rk2);
    for (int64_t t = t0; t < T; t += nw) {
        // routing bookkeeping of this token
        if (lane < k) {
            row_of[t * k + lane] = row_cur;
            if (row_cur >= 0) sorted_token[row_cur] = (int32_t)t;
        }
        int64_t off[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            const int32_t rj = __shfl_sync(kFull, row_cur, j);
            off[j] = (j < k && rj >= 0) ? (int64_t)rj * H8 : -1;
        }
        // advance the pipeline: the next token's row, then the loads behind it
        const int32_t row_next = make_row(t + nw, e1, rk1, bb_next);
        const int bb_next2 = load_bb(t + 2 * nw, e2);
        int e3, rk3;
        load_er(t + 3 * nw, e3, rk3);
        // copy the row
        const uint4* src = x + t * H8;
        for (int c0 = 0; c0 < H8; c0 += 32 * CH) {
            uint4 v[CH];
#pragma unroll
            for (int h = 0; h < CH; ++h) {
                const int c = c0 + 32 * h + lane;
                if (c < H8) v[h] = __ldg(src + c);
            }
#pragma unroll
            for (int h = 0; h < CH; ++h) {
                const int c = c0 + 32 * h + lane;
                if (c >= H8) continue;
#pragma unroll
                for (int j = 0; j < KB; ++j)
                    if (off[j] >= 0) x_perm[off[j] + c] = v[h];
            }
        }
        row_cur = row_next;
        e1 = e2;
        rk1 = rk2;
        bb_next = bb_next2;
        e2 = e3;
        rk2 = rk3;
    }
}

// Padded dispatch (Transformer Engine "Mixture of Experts", Token permutation,
// Padding and alignment): each expert's block is rounded up to a multiple of
// align rows, an empty block stays empty, and the permute kernels then run on
// the padded offsets, so the rows keep their unpadded order inside a block.
// pad_offsets_kernel: one block, one thread per expert, an exclusive scan of
// the rounded counts in expert order.
__global__ void __launch_bounds__(256)
    pad_offsets_kernel(const int32_t* __restrict__ offsets, int E, int align, int32_t* __restrict__ padded) {
    __shared__ int32_t warp_sum[8];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    int32_t c = 0;
    if (e < E) {
        const int32_t cnt = __ldg(offsets + e + 1) - __ldg(offsets + e);
        c = cnt > 0 ? (int32_t)(((int64_t)cnt + align - 1) / align * align) : 0;
    }
    int32_t incl = c;   // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int32_t base = 0;
    for (int w = 0; w < warp; ++w) base += warp_sum[w];
    if (e < E) padded[e + 1] = base + incl;
    if (e == 0) padded[0] = 0;
}

// Pad rows of expert e (blockIdx.x): [padded[e] + count, padded[e+1]). Their
// x_perm rows become zeros, their sorted_token -1 and their weight 0.
__global__ void __launch_bounds__(256)
    pad_fill_kernel(const int32_t* __restrict__ offsets, const int32_t* __restrict__ padded, int H8,
                    uint4* __restrict__ x_perm, int32_t* __restrict__ sorted_token, float* __restrict__ prob_perm) {
    const int e = blockIdx.x;
    const int64_t cnt = (int64_t)__ldg(offsets + e + 1) - __ldg(offsets + e);
    const int64_t r0 = (int64_t)__ldg(padded + e) + (cnt > 0 ? cnt : 0);
    const int64_t r1 = __ldg(padded + e + 1);
    if (r1 <= r0) return;
    const int64_t n = (r1 - r0) * H8;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) x_perm[r0 * H8 + i] = make_uint4(0, 0, 0, 0);
    for (int64_t r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
        sorted_token[r] = -1;
        if (prob_perm) prob_perm[r] = 0.0f;
    }
}

// prob_perm[row_of[i]] = topk_prob[i]: the routing weight of each permuted row.
__global__ void __launch_bounds__(256)
    prob_perm_kernel(const float* __restrict__ topk_prob, const int32_t* __restrict__ row_of, int64_t n,
                     float* __restrict__ prob_perm) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t r = __ldg(row_of + i);
        if (r >= 0) prob_perm[r] = __ldg(topk_prob + i);
    }
}

// Scratch for moe_router_topk_noalloc: a fixed array in device memory, so the
// call allocates nothing. Its size bounds the routing sizes that call accepts.
constexpr size_t kNoAllocScratchBytes = (3u << 20) + 4096;
static __device__ __align__(256) unsigned char g_router_noalloc_scratch[kNoAllocScratchBytes];

}  // namespace

size_t route_scratch_bytes(int64_t T, int E, int k) {
    const int64_t nb = route_blocks(T);
    size_t b = (size_t)E * nb * 4;
    b = (b + 255) & ~size_t(255);
    b += (size_t)T * k * 4;
    b = (b + 255) & ~size_t(255);
    b += 256;
    return b;
}

RouteScratch carve_route_scratch(void* base, int64_t T, int E, int k) {
    const int64_t nb = route_blocks(T);
    char* p = static_cast<char*>(base);
    RouteScratch rs;
    rs.block_base = reinterpret_cast<int32_t*>(p);
    size_t off = ((size_t)E * nb * 4 + 255) & ~size_t(255);
    rs.local_rank = reinterpret_cast<int32_t*>(p + off);
    off = (off + (size_t)T * k * 4 + 255) & ~size_t(255);
    rs.ticket = reinterpret_cast<unsigned*>(p + off);
    return rs;
}

template <int SLOTS>
cudaError_t launch_router_k(const RouterArgs& a, dim3 grid, dim3 block, cudaStream_t st) {
    switch (a.k) {
        case 1: return launch_chained(router_topk_kernel<SLOTS, 1>, grid, block, 0, st, a);
        case 2: return launch_chained(router_topk_kernel<SLOTS, 2>, grid, block, 0, st, a);
        case 4: return launch_chained(router_topk_kernel<SLOTS, 4>, grid, block, 0, st, a);
        case 6: return launch_chained(router_topk_kernel<SLOTS, 6>, grid, block, 0, st, a);
        case 8: return launch_chained(router_topk_kernel<SLOTS, 8>, grid, block, 0, st, a);
        default: return launch_chained(router_topk_kernel<SLOTS, 0>, grid, block, 0, st, a);
    }
}

cudaError_t launch_router_topk(const float* logits, int64_t T, int E, int k,
                               const moe_router_opts& opts, int32_t* topk_idx, float* topk_prob,
                               uint8_t* routing_map, const RouteScratch& rs, cudaStream_t st,
                               unsigned* err, int32_t* counts, int32_t* offsets, bool* scanned, int32_t* zero,
                               int n_zero, const bf16* x, int H, bf16* x_perm, int32_t* sorted_token,
                               int32_t* row_of, bool* permuted) {
    if (scanned) *scanned = false;
    RouterArgs a;
    a.logits = logits;
    a.T = T;
    a.E = E;
    a.k = k;
    a.score_fn = opts.score_fn;
    a.renormalize = opts.renormalize;
    a.scaling = opts.scaling;
    a.bias = opts.expert_bias;
    a.topk_idx = topk_idx;
    a.topk_prob = topk_prob;
    a.routing_map = routing_map;
    a.block_base = rs.block_base;
    a.local_rank = rs.local_rank;
    a.ticket = rs.ticket;
    a.nb = (int)route_blocks(T);
    a.tpb = route_tokens_per_block(T);
    a.counts = nullptr;
    a.offsets = nullptr;
    a.zero = nullptr;
    a.n_zero = 0;
    a.x = nullptr;
    a.H8 = 0;
    a.x_perm = nullptr;
    a.sorted_token = nullptr;
    a.row_of = nullptr;
    if (permuted) *permuted = false;
    // Large T: the lane-per-token kernel where it applies. moe_testing_set_kernels
    // can force either kernel (the tests run both on the same inputs).
    const int force = kernel_override().router;
    const bool lane_ok = E % 32 == 0 && E <= 256 && k <= 8 && kLaneTokens % a.tpb == 0 &&
                         (opts.score_fn == MOE_SCORE_SIGMOID || opts.renormalize) &&
                         ((uintptr_t)logits & 15u) == 0;
    const bool use_lane = lane_ok && (force != MOE_TESTING_AUTO ? force == MOE_TESTING_ROUTER_LANE
                                                                 : T >= kLaneMinTokens);
    if (use_lane) {
        const dim3 lgrid((unsigned)((T + kLaneTokens - 1) / kLaneTokens)), lblock(kLaneTokens);
        const bool bias = opts.expert_bias != nullptr;
        cudaError_t e = cudaSuccess;
#define MOE_LANE(KC)                                                                    \
    e = bias ? launch_chained(router_lane_kernel<KC, true>, lgrid, lblock, 0, st, a)    \
             : launch_chained(router_lane_kernel<KC, false>, lgrid, lblock, 0, st, a)
        switch (k) {
            case 1: MOE_LANE(1); break;
            case 2: MOE_LANE(2); break;
            case 3: MOE_LANE(3); break;
            case 4: MOE_LANE(4); break;
            case 5: MOE_LANE(5); break;
            case 6: MOE_LANE(6); break;
            case 7: MOE_LANE(7); break;
            default: MOE_LANE(8); break;
        }
#undef MOE_LANE
        (void)err;
        return e;
    }
    const dim3 grid((unsigned)a.nb), block(kRouteThreads);
    (void)err;
    if (a.nb == 1 && counts != nullptr && offsets != nullptr) {   // one token block: no scan kernel
        a.counts = counts;
        a.offsets = offsets;
        a.zero = zero;
        a.n_zero = zero ? n_zero : 0;
        if (scanned) *scanned = true;
        // The permute in the router's one block: it saves a launch, but one
        // CTA copies the rows. Measured on B200 (Qwen3 shape, L2 flushed): T = 1,
        // 32 KB of rows, 33.4 against 34.8 us a step; T = 8, 256 KB, 48.6
        // against 44.3 us. Hence at most 64 KB of rows.
        if (x && x_perm && sorted_token && row_of && permuted && k <= 16 && H % 8 == 0 &&
            T * (int64_t)k * H * (int64_t)sizeof(bf16) <= 65536) {
            a.x = reinterpret_cast<const uint4*>(x);
            a.H8 = H / 8;
            a.x_perm = reinterpret_cast<uint4*>(x_perm);
            a.sorted_token = sorted_token;
            a.row_of = row_of;
            *permuted = true;
        }
    }
    if (E <= 32) return launch_router_k<1>(a, grid, block, st);
    if (E <= 64) return launch_router_k<2>(a, grid, block, st);
    if (E <= 128) return launch_router_k<4>(a, grid, block, st);
    return launch_router_k<8>(a, grid, block, st);
}

cudaError_t launch_router_backward(const float* logits, int64_t T, int E, int k, const moe_router_opts& opts,
                                   const int32_t* topk_idx, const float* dprob, float* dlogits,
                                   cudaStream_t st, unsigned* err) {
    const int64_t warps_per_block = kRouteThreads / 32;
    int64_t blocks = (T + warps_per_block - 1) / warps_per_block;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) return cudaSuccess;
    const dim3 grid((unsigned)blocks), block(kRouteThreads);
#define MOE_ROUTER_BWD(S)                                                                              \
    router_backward_kernel<S><<<grid, block, 0, st>>>(logits, T, E, k, opts.score_fn, opts.renormalize, \
                                                      opts.scaling, topk_idx, dprob, dlogits, err)
    if (E <= 32) MOE_ROUTER_BWD(1);
    else if (E <= 64) MOE_ROUTER_BWD(2);
    else if (E <= 128) MOE_ROUTER_BWD(4);
    else MOE_ROUTER_BWD(8);
#undef MOE_ROUTER_BWD
    return cudaGetLastError();
}

cudaError_t launch_expert_bias_update(const int32_t* counts, int E, float coeff, float* bias, cudaStream_t st) {
    expert_bias_update_kernel<<<1, 256, 0, st>>>(counts, E, coeff, bias);
    return cudaGetLastError();
}

cudaError_t launch_rank_from_indices(const int32_t* topk_idx, int64_t T, int E, int k,
                                     const RouteScratch& rs, cudaStream_t st, unsigned* err) {
    const int nb = (int)route_blocks(T);
    rank_from_indices_kernel<<<nb, kRouteThreads, 0, st>>>(topk_idx, T, E, k, rs.local_rank,
                                                          rs.block_base, rs.ticket, nb,
                                                          route_tokens_per_block(T), err);
    return cudaGetLastError();
}

cudaError_t launch_expert_scan(int64_t T, int E, const RouteScratch& rs, int32_t* counts,
                               int32_t* offsets, cudaStream_t st, int32_t* zero, int n_zero) {
    const int nb = (int)route_blocks(T);
    if (!counts) zero = nullptr;   // the kernels return before the offsets without counts
    if (!zero) n_zero = 0;
    if (nb <= kScanSmallBlocks)
        return launch_chained(expert_scan_small_kernel, dim3(1), dim3(1024), 0, st, rs.block_base, nb, E, counts,
                              offsets, zero, n_zero);
    int threads = 32;
    while (threads * kScanPerThread < nb && threads < 1024) threads <<= 1;
    return launch_chained(expert_scan_kernel, dim3(E), dim3(threads), 0, st, rs.block_base, nb, E, counts, offsets,
                          rs.ticket, zero, n_zero);
}

cudaError_t launch_pad_offsets(const int32_t* offsets, int E, int align, int32_t* padded_offsets, cudaStream_t st) {
    pad_offsets_kernel<<<1, 256, 0, st>>>(offsets, E, align, padded_offsets);
    return cudaGetLastError();
}

cudaError_t launch_pad_fill(const int32_t* offsets, const int32_t* padded_offsets, int E, int H, bf16* x_perm,
                            int32_t* sorted_token, float* prob_perm, cudaStream_t st) {
    pad_fill_kernel<<<(unsigned)E, 256, 0, st>>>(offsets, padded_offsets, H / 8, reinterpret_cast<uint4*>(x_perm),
                                                sorted_token, prob_perm);
    return cudaGetLastError();
}

cudaError_t launch_prob_perm(const float* topk_prob, const int32_t* row_of, int64_t n, float* prob_perm,
                             cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    prob_perm_kernel<<<(unsigned)blocks, 256, 0, st>>>(topk_prob, row_of, n, prob_perm);
    return cudaGetLastError();
}

cudaError_t launch_permute(const bf16* x, int64_t T, int H, const int32_t* topk_idx, int k,
                           const int32_t* offsets, int E, const RouteScratch& rs, bf16* x_perm,
                           int32_t* sorted_token, int32_t* row_of, cudaStream_t st, unsigned* err,
                           int64_t row_bound) {
    const int64_t A = row_bound > 0 ? row_bound : T * k;   // rows of x_perm and sorted_token
    const int nb = (int)route_blocks(T);
    if (T == 0) return cudaSuccess;
    const int H8r = H / 8;
    // Token-range register kernel for rows up to 4096 wide, warp per token
    // otherwise. Measured inside the steps on B200 (fraction of HBM): k=8,
    // H=2048: 0.73 against 0.67 for the warp kernel; k=2, H=4096: 0.67
    // against 0.64; H=5120: warp 0.76. moe_testing_set_kernels can select
    // the warp kernel for any width.
    const int force = kernel_override().permute;
    const bool regs = x_perm == nullptr || (H8r <= 512 && force != MOE_TESTING_PERMUTE_WARP);
    if (regs) {
        // without x_perm only the rows are computed: 256 threads whatever H
        const int threads = x_perm == nullptr ? 256 : (H8r + 31) / 32 * 32;
        int per_sm = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, permute_tokens_kernel, threads, 0) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
        const int64_t slots = (int64_t)sm_count() * per_sm;
        const int64_t per_block = (T + slots - 1) / slots;
        const int64_t blocks = (T + per_block - 1) / per_block;
        return launch_chained(permute_tokens_kernel, dim3((unsigned)blocks), dim3(threads), 0, st,
                              reinterpret_cast<const uint4*>(x), T, H8r, topk_idx, k, offsets, E,
                              (const int32_t*)rs.block_base, nb, route_tokens_per_block(T),
                              (const int32_t*)rs.local_rank, reinterpret_cast<uint4*>(x_perm), sorted_token, row_of,
                              A, per_block, err);
    }
    if (E > kPermMaxExperts) return cudaErrorInvalidValue;
    constexpr int kThreadsW = 256;
    auto kern = k <= 2 ? permute_warp_kernel<2, 4>
              : k <= 4 ? permute_warp_kernel<4, 4>
              : k <= 8 ? permute_warp_kernel<8, 4> : permute_warp_kernel<16, 4>;
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreadsW, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int64_t cap = (int64_t)sm_count() * per_sm * (kThreadsW / 32);
    const int64_t warps = T < cap ? T : cap;
    const int64_t blocks = (warps + kThreadsW / 32 - 1) / (kThreadsW / 32);
    return launch_chained(kern, dim3((unsigned)blocks), dim3(kThreadsW), 0, st, reinterpret_cast<const uint4*>(x), T,
                          H8r, topk_idx, k, offsets, E, (const int32_t*)rs.block_base, nb, route_tokens_per_block(T),
                          (const int32_t*)rs.local_rank, reinterpret_cast<uint4*>(x_perm), sorted_token, row_of, A,
                          err);
}

// Device address of g_router_noalloc_scratch on the current device. In host
// code the array's name is only a host-side stand-in, so the address is taken
// with cudaGetSymbolAddress while that device is current. A successful lookup
// is kept for the device; a failed one (for example a first call made while
// the stream is being captured) is not, and the next call tries again.
size_t router_noalloc_capacity() { return kNoAllocScratchBytes; }

cudaError_t router_noalloc_scratch(void** ptr) {
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static void* addr[kMaxDev];
    *ptr = nullptr;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_router_noalloc_scratch);
        if (e != cudaSuccess) {
            cudaGetLastError();   // the failed lookup's error is returned here, not left for a later call
            return e;
        }
        addr[dev] = p;
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

}  // namespace moe
