// ep_layout.cu -- layout kernels.
//
// Token choice ("get_dispatch_layout", DeepEP-Ascend README, API Overview):
// one thread-block cluster of up to 16 CTAs.  Each CTA owns a contiguous
// token range; each of its 32 warps walks a contiguous run of (t,k) pairs
// 32 at a time, ranks equal expert ids inside the step with __match_any_sync
// and keeps a private per-expert counter row in shared memory, so the rank
// of a pair inside its expert is
//     (pairs of that expert in earlier CTAs)          -- read over DSMEM
//   + (pairs in earlier warps of this CTA)            -- scan down the rows
//   + (pairs earlier in this warp's run)              -- the warp's counter
// which is the stable (token-major) order with integer arithmetic only.
// The cluster barrier is the hardware one; there is no spin loop.
//
// Expert choice (DeepEP issue #595, Solution 1): token_indices[E, C] is
// inverted into a per-token CSR of slot ids.  Degrees and rank masks by
// global atomics (order-free integer sums), one-CTA scan, an unordered fill,
// then each token's slot list is put in ascending order by a warp that ranks
// every entry against the others (slot ids are distinct).
#include <algorithm>
#include <atomic>

#include <cooperative_groups.h>

#include "ep_device.cuh"
#include "ep_internal.h"

namespace cg = cooperative_groups;

namespace ep {

namespace {

#ifndef EP_LAYOUT_THREADS
#define EP_LAYOUT_THREADS 512
#endif
#ifndef EP_LAYOUT_PAIRS_PER_CTA
#define EP_LAYOUT_PAIRS_PER_CTA 2048
#endif
#ifndef EP_LAYOUT_MAX_CLUSTER
#define EP_LAYOUT_MAX_CLUSTER 16
#endif
// one-CTA layouts launched without the cluster attribute: every launch is an
// implicit cluster of one CTA, and the plain launch measured ~1 us faster
// (decode and tiny batches: 14.3 -> 13.2 us, 12.3 -> 11.3 us event-timed)
#ifndef EP_LAYOUT_SINGLE_PLAIN
#define EP_LAYOUT_SINGLE_PLAIN 1
#endif
// from this many (token, k) pairs on, the grid-wide kernel is used: up to a
// full 16-CTA cluster's 16 x 2048 pairs the cluster kernel makes the layout +
// dispatch step faster (4096 x 8 pairs: 177.2 -> 173.1 us per step, it
// leaves more SMs to the dispatch that runs under it); beyond, the grid kernel
// (16384 x 8 pairs: cluster 611 us, grid 602 us per step)
#ifndef EP_LAYOUT_GRID_MIN_PAIRS
#define EP_LAYOUT_GRID_MIN_PAIRS 32769
#endif
constexpr int kLayoutThreads = EP_LAYOUT_THREADS;
constexpr int kLayoutWarps = kLayoutThreads / 32;
// 32-pair steps a warp keeps in registers: a full 16-CTA cluster holds 8192
// pairs per CTA (131072 pairs) on the register path
constexpr int kPrefetch = 8192 / kLayoutThreads;
constexpr int kLoadBatch = 8;                       // ids loaded together
constexpr int64_t kPairsPerCta = EP_LAYOUT_PAIRS_PER_CTA;
constexpr int kMaxCluster = 16;
constexpr int64_t kSmemIds = 8192; // pairs per CTA whose ids are staged in shared memory

struct TcArgs {
    const int64_t* topk_idx;
    int32_t T, K, E, R, per_rank;
    int32_t* counts;
    int32_t* offsets;
    int32_t* rank_counts;
    uint8_t* in_rank;
    int32_t* slot;
    uint32_t* err;
    int32_t in_rank_words; // 1: write is_token_in_rank as 32-bit words
    int32_t trigger;       // let the dispatch launched next start at once
};

__device__ __forceinline__ void write_rank_row(const TcArgs& a, int64_t t, uint32_t mask)
{
    uint8_t* row = a.in_rank + t * a.R;
    if (a.in_rank_words) {
        for (int r = 0; r < a.R; r += 4) {
            const uint32_t w = ((mask >> r) & 1u) | (((mask >> (r + 1)) & 1u) << 8) |
                               (((mask >> (r + 2)) & 1u) << 16) | (((mask >> (r + 3)) & 1u) << 24);
            *reinterpret_cast<uint32_t*>(row + r) = w;
        }
    } else {
        for (int r = 0; r < a.R; ++r)
            row[r] = static_cast<uint8_t>((mask >> r) & 1u);
    }
}

__device__ __forceinline__ void cluster_arrive_relaxed()
{
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait()
{
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// Exclusive scan of one int per thread over the block; returns the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int& total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int o = __shfl_up_sync(kFullMask, incl, d);
        if (lane >= d)
            incl += o;
    }
    if (lane == 31)
        warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int nw = blockDim.x >> 5;
        int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            int o = __shfl_up_sync(kFullMask, s, d);
            if (lane >= d)
                s += o;
        }
        warp_sums[lane] = s; // inclusive
    }
    __syncthreads();
    total = warp_sums[(blockDim.x >> 5) - 1];
    int excl = incl - v + (warp > 0 ? warp_sums[warp - 1] : 0);
    __syncthreads();
    return excl;
}

__global__ void __launch_bounds__(kLayoutThreads, 1) tc_layout_cluster_kernel(TcArgs a)
{
    if (a.trigger)
        pdl_launch_dependents(); // the dispatch of the same call may load its rows now
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = static_cast<int>(cluster.num_blocks());
    const int b = static_cast<int>(cluster.block_rank());
    extern __shared__ __align__(16) int32_t smem[];
    int32_t* wtab = smem;                      // [warps][E] per-warp counters, later prefixes
    int32_t* tot = wtab + kLayoutWarps * a.E;  // [E] this CTA's pairs per expert
    int32_t* base = tot + a.E;                 // [E] pairs of each expert in earlier CTAs
    int32_t* all = base + a.E;                 // [E] pairs of each expert in the cluster
    int32_t* srank = all + a.E;                // [32] this CTA's tokens per rank
    int32_t* sscan = srank + 32;               // [32] scan scratch
    int* sid = sscan + 32;                     // [<= kSmemIds] expert id of each pair (or -1)
    uint32_t* smask = reinterpret_cast<uint32_t*>(sid + kSmemIds); // [<= kSmemIds] rank bits per token
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    for (int i = tid; i < kLayoutWarps * a.E; i += kLayoutThreads)
        wtab[i] = 0;
    if (tid < 32)
        srank[tid] = 0;
    __syncthreads();

    const int64_t tpc = (static_cast<int64_t>(a.T) + cs - 1) / cs;
    const int64_t t0 = min(static_cast<int64_t>(a.T), static_cast<int64_t>(b) * tpc);
    const int64_t t1 = min(static_cast<int64_t>(a.T), t0 + tpc);
    const int64_t p0 = t0 * a.K, p1 = t1 * a.K;
    const int64_t ppw = ((p1 - p0 + kLayoutWarps - 1) / kLayoutWarps + 31) / 32 * 32;
    const int64_t wb = min(p1, p0 + warp * ppw);
    const int64_t we = min(p1, wb + ppw);
    int32_t* mine = wtab + warp * a.E;
    const uint32_t lanes_below = (1u << lane) - 1u;
    bool bad = false;

    // phase 1: per-warp stable ranks and counters.  When the warp's run fits
    // kPrefetch steps the ids and ranks stay in registers; longer runs park
    // the rank in slot[] and re-read it in phase 3.
    const bool in_regs = (we - wb) <= 32 * kPrefetch;
    // with the whole CTA on the register path its ids are also staged in
    // shared memory for the rank-membership pass
    const bool ids_in_smem = (p1 - p0) <= kSmemIds;
    int ev[kPrefetch]; // expert id, or -1 for a pair that is not routed
    int loc[kPrefetch];
    for (int64_t start = wb; start < we; start += 32 * kPrefetch) {
#pragma unroll
        for (int j0 = 0; j0 < kPrefetch; j0 += kLoadBatch) {
            int64_t raw[kLoadBatch];
#pragma unroll
            for (int j = 0; j < kLoadBatch; ++j) {
                const int64_t p = start + (j0 + j) * 32 + lane;
                raw[j] = p < we ? __ldg(a.topk_idx + p) : -1;
            }
#pragma unroll
            for (int j = 0; j < kLoadBatch; ++j) {
                const bool ok = raw[j] >= 0 && raw[j] < a.E;
                bad |= !ok && raw[j] != -1;
                ev[j0 + j] = ok ? static_cast<int>(raw[j]) : -1;
                const int64_t p = start + (j0 + j) * 32 + lane;
                if (ids_in_smem && p < we)
                    sid[p - p0] = ev[j0 + j];
            }
        }
        // the steps' equal-id lane sets are independent: issue them together,
        // then run the dependent counter updates step after step
        uint32_t peers[kPrefetch];
#pragma unroll
        for (int j = 0; j < kPrefetch; ++j)
            peers[j] = start + j * 32 < we ? __match_any_sync(kFullMask, ev[j]) : 0u;
#pragma unroll
        for (int j = 0; j < kPrefetch; ++j) {
            loc[j] = -1;
            const int64_t step = start + j * 32;
            if (step >= we)
                break; // warp-uniform
            const int64_t p = step + lane;
            const int e = ev[j];
            int prior = 0;
            if (e >= 0)
                prior = mine[e];
            __syncwarp();
            if (e >= 0) {
                const int r = __popc(peers[j] & lanes_below);
                loc[j] = prior + r;
                if (r == 0)
                    mine[e] = prior + __popc(peers[j]);
            }
            if (!in_regs && p < we)
                a.slot[p] = loc[j];
            __syncwarp();
        }
    }

    // phase 1b: rank membership of this CTA's tokens, from the staged ids in
    // shared memory, else re-read from L1/L2 (a token's loads issued together)
    __syncthreads();
    for (int64_t tb = t0 + static_cast<int64_t>(warp) * 32; tb < t1; tb += kLayoutThreads) {
        const int64_t t = tb + lane;
        uint32_t mask = 0;
        if (t < t1 && ids_in_smem) {
            const int* ids = sid + (t - t0) * a.K;
            for (int k = 0; k < a.K; ++k)
                if (ids[k] >= 0)
                    mask |= 1u << static_cast<uint32_t>(ids[k] / a.per_rank);
            smask[t - t0] = mask; // written out after the cluster barriers
        } else if (t < t1) {
            for (int k0 = 0; k0 < a.K; k0 += kLoadBatch) {
                int64_t ids[kLoadBatch];
#pragma unroll
                for (int k = 0; k < kLoadBatch; ++k)
                    ids[k] = k0 + k < a.K ? __ldg(a.topk_idx + t * a.K + k0 + k) : -1;
#pragma unroll
                for (int k = 0; k < kLoadBatch; ++k)
                    if (ids[k] >= 0 && ids[k] < a.E)
                        mask |= 1u << static_cast<uint32_t>(ids[k] / a.per_rank);
            }
            write_rank_row(a, t, mask);
        }
        for (int r = 0; r < a.R; ++r) {
            const int c = __popc(__ballot_sync(kFullMask, (mask >> r) & 1u));
            if (lane == 0 && c)
                atomicAdd(&srank[r], c);
        }
    }
    if (__any_sync(kFullMask, bad) && lane == 0)
        flag_error(a.err, EP_DEVERR_BAD_INDEX);
    __syncthreads();

    // phase 2: counters -> exclusive prefix down the warps; CTA totals
    for (int e = tid; e < a.E; e += kLayoutThreads) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kLayoutWarps; ++w) {
            const int c = wtab[w * a.E + e];
            wtab[w * a.E + e] = run;
            run += c;
        }
        tot[e] = run;
    }
    cluster.sync();

    // totals of every CTA of the cluster, all loads in flight together
    for (int e = tid; e < a.E; e += kLayoutThreads) {
        int v[kMaxCluster];
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j)
            v[j] = j < cs ? cluster.map_shared_rank(tot, j)[e] : 0;
        int bs = 0, al = 0;
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j) {
            bs += j < b ? v[j] : 0;
            al += v[j];
        }
        base[e] = bs;
        all[e] = al;
    }
    int rank_total = 0;
    if (b == 0 && tid < a.R) {
        int v[kMaxCluster];
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j)
            v[j] = j < cs ? cluster.map_shared_rank(srank, j)[tid] : 0;
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j)
            rank_total += v[j];
    }
    // every remote read above has completed (its value is in registers or
    // shared memory); the matching wait sits at the end of the kernel so that
    // no CTA exits while another may still read its shared memory
    cluster_arrive_relaxed();

    if (b == 0) {
        // expert offsets: exclusive scan of the cluster totals, one block-wide
        // pass per kLayoutThreads experts
        int carry = 0;
        for (int e0 = 0; e0 < a.E; e0 += kLayoutThreads) {
            const int e = e0 + tid;
            const int v = e < a.E ? all[e] : 0;
            int total = 0;
            const int excl = block_exclusive_scan(v, sscan, total);
            if (e < a.E) {
                a.counts[e] = v;
                a.offsets[e] = carry + excl;
            }
            carry += total;
        }
        if (tid == 0)
            a.offsets[a.E] = carry;
        if (tid < a.R)
            a.rank_counts[tid] = rank_total;
    }
    for (int e = tid; e < a.E; e += kLayoutThreads) {
        const int bs = base[e];
#pragma unroll
        for (int w = 0; w < kLayoutWarps; ++w)
            wtab[w * a.E + e] += bs;
    }
    __syncthreads();

    // phase 3: slot = rank inside the warp's run + (earlier warps + earlier
    // CTAs); the same lane owns the same pair as in phase 1
    if (in_regs) {
#pragma unroll
        for (int j = 0; j < kPrefetch; ++j) {
            const int64_t p = wb + j * 32 + lane;
            if (p < we)
                a.slot[p] = loc[j] >= 0 ? loc[j] + mine[ev[j]] : -1;
        }
    } else {
        for (int64_t step = wb; step < we; step += 32) {
            const int64_t p = step + lane;
            if (p < we) {
                const int32_t l = a.slot[p];
                if (l >= 0)
                    a.slot[p] = l + mine[__ldg(a.topk_idx + p)];
            }
        }
    }
    if (ids_in_smem) {
        for (int64_t t = t0 + tid; t < t1; t += kLayoutThreads)
            write_rank_row(a, t, smask[t - t0]);
    }
    cluster_wait();
}

// ---------------------------------------------------------------------------
// Token choice over the whole device: one CTA per SM (cooperative launch),
// each with a contiguous token range.  Phase 1 is the cluster kernel's
// (per-warp runs ranked with match.any, per-warp counters in shared memory);
// each CTA then publishes its per-expert totals and per-rank token counts in
// the workspace, all CTAs meet at a grid barrier (bounded wait), and every
// CTA sums the totals of the CTAs before it to get its base per expert.  The
// bookkeeping is spread over every SM instead of 16.
constexpr int kGridThreads = 256;
constexpr int kGridWarps = kGridThreads / 32;
constexpr int kGridPrefetch = 8;                          // 32-pair steps per warp in registers
constexpr int64_t kGridIds = kGridWarps * kGridPrefetch * 32; // pairs per CTA staged in shared memory
constexpr int kGridMaxBlocks = 64;                      // workspace holds this many CTAs' totals
#ifndef EP_LAYOUT_GRID_PAIRS_PER_CTA
#define EP_LAYOUT_GRID_PAIRS_PER_CTA 1024
#endif
constexpr int64_t kGridPairsPerCta = EP_LAYOUT_GRID_PAIRS_PER_CTA;

struct GridBar {
    uint32_t* arrive;
    uint32_t* generation;
};

// All CTAs of a cooperative launch meet here; false if the wait ran out.
__device__ __forceinline__ bool grid_sync(GridBar bar, uint32_t nblocks, uint32_t* err, int* ok_smem)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        volatile uint32_t* gen = bar.generation;
        const uint32_t g = *gen;
        __threadfence();
        bool ok = true;
        if (atomicAdd(bar.arrive, 1u) == nblocks - 1) {
            atomicExch(bar.arrive, 0u);
            __threadfence();
            atomicAdd(bar.generation, 1u);
        } else {
            const uint64_t t0 = global_timer_ns();
            for (uint32_t i = 1; *gen == g; ++i) {
                if ((i & 63u) == 0u && global_timer_ns() - t0 > kWaitLimitNs) {
                    flag_error(err, EP_DEVERR_TIMEOUT);
                    ok = false;
                    break;
                }
            }
        }
        __threadfence();
        *ok_smem = ok ? 1 : 0;
    }
    __syncthreads();
    return *ok_smem != 0;
}

__global__ void __launch_bounds__(kGridThreads) tc_layout_grid_kernel(TcArgs a, int32_t* tile_counts,
                                                                      int32_t* tile_ranks, GridBar bar)
{
    if (a.trigger)
        pdl_launch_dependents(); // the dispatch of the same call may load its rows now
    const int G = static_cast<int>(gridDim.x);
    const int b = static_cast<int>(blockIdx.x);
    extern __shared__ __align__(16) int32_t smem[];
    int32_t* wtab = smem;                      // [warps][E] per-warp counters, later prefixes
    int32_t* srank = wtab + kGridWarps * a.E;  // [32] this CTA's tokens per rank
    int32_t* sscan = srank + 32;               // [32] scan scratch
    int* sid = sscan + 32;                     // [kGridIds] expert id of each pair (or -1)
    uint32_t* smask = reinterpret_cast<uint32_t*>(sid + kGridIds); // [kGridIds] rank bits per token
    int* ok_smem = reinterpret_cast<int*>(smask + kGridIds);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    for (int i = tid; i < kGridWarps * a.E; i += kGridThreads)
        wtab[i] = 0;
    if (tid < 32)
        srank[tid] = 0;
    __syncthreads();

    const int64_t tpc = (static_cast<int64_t>(a.T) + G - 1) / G;
    const int64_t t0 = min(static_cast<int64_t>(a.T), static_cast<int64_t>(b) * tpc);
    const int64_t t1 = min(static_cast<int64_t>(a.T), t0 + tpc);
    const int64_t p0 = t0 * a.K, p1 = t1 * a.K;
    const int64_t ppw = ((p1 - p0 + kGridWarps - 1) / kGridWarps + 31) / 32 * 32;
    const int64_t wb = min(p1, p0 + warp * ppw);
    const int64_t we = min(p1, wb + ppw);
    int32_t* mine = wtab + warp * a.E;
    const uint32_t lanes_below = (1u << lane) - 1u;
    bool bad = false;
    const bool in_regs = (we - wb) <= 32 * kGridPrefetch;
    const bool ids_in_smem = (p1 - p0) <= kGridIds;

    // phase 1: per-warp stable ranks and counters (as in the cluster kernel)
    int ev[kGridPrefetch];
    int loc[kGridPrefetch];
    for (int64_t start = wb; start < we; start += 32 * kGridPrefetch) {
        int64_t raw[kGridPrefetch];
#pragma unroll
        for (int j = 0; j < kGridPrefetch; ++j) {
            const int64_t p = start + j * 32 + lane;
            raw[j] = p < we ? __ldg(a.topk_idx + p) : -1;
        }
#pragma unroll
        for (int j = 0; j < kGridPrefetch; ++j) {
            const bool ok = raw[j] >= 0 && raw[j] < a.E;
            bad |= !ok && raw[j] != -1;
            ev[j] = ok ? static_cast<int>(raw[j]) : -1;
            const int64_t p = start + j * 32 + lane;
            if (ids_in_smem && p < we)
                sid[p - p0] = ev[j];
        }
        uint32_t peers[kGridPrefetch];
#pragma unroll
        for (int j = 0; j < kGridPrefetch; ++j)
            peers[j] = start + j * 32 < we ? __match_any_sync(kFullMask, ev[j]) : 0u;
#pragma unroll
        for (int j = 0; j < kGridPrefetch; ++j) {
            loc[j] = -1;
            const int64_t step = start + j * 32;
            if (step >= we)
                break; // warp-uniform
            const int64_t p = step + lane;
            const int e = ev[j];
            int prior = 0;
            if (e >= 0)
                prior = mine[e];
            __syncwarp();
            if (e >= 0) {
                const int r = __popc(peers[j] & lanes_below);
                loc[j] = prior + r;
                if (r == 0)
                    mine[e] = prior + __popc(peers[j]);
            }
            if (!in_regs && p < we)
                a.slot[p] = loc[j];
            __syncwarp();
        }
    }
    __syncthreads();

    // phase 1b: rank membership of this CTA's tokens
    for (int64_t tb = t0 + static_cast<int64_t>(warp) * 32; tb < t1; tb += kGridThreads) {
        const int64_t t = tb + lane;
        uint32_t mask = 0;
        if (t < t1) {
            if (ids_in_smem) {
                const int* ids = sid + (t - t0) * a.K;
                for (int k = 0; k < a.K; ++k)
                    if (ids[k] >= 0)
                        mask |= 1u << static_cast<uint32_t>(ids[k] / a.per_rank);
                smask[t - t0] = mask;
            } else {
                for (int k = 0; k < a.K; ++k) {
                    const int64_t e = __ldg(a.topk_idx + t * a.K + k);
                    if (e >= 0 && e < a.E)
                        mask |= 1u << static_cast<uint32_t>(e / a.per_rank);
                }
                write_rank_row(a, t, mask);
            }
        }
        for (int r = 0; r < a.R; ++r) {
            const int c = __popc(__ballot_sync(kFullMask, (mask >> r) & 1u));
            if (lane == 0 && c)
                atomicAdd(&srank[r], c);
        }
    }
    if (__any_sync(kFullMask, bad) && lane == 0)
        flag_error(a.err, EP_DEVERR_BAD_INDEX);
    __syncthreads();

    // phase 2: exclusive prefix down the warps; publish this CTA's totals
    for (int e = tid; e < a.E; e += kGridThreads) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kGridWarps; ++w) {
            const int c = wtab[w * a.E + e];
            wtab[w * a.E + e] = run;
            run += c;
        }
        tile_counts[static_cast<int64_t>(b) * a.E + e] = run;
    }
    if (tid < a.R)
        tile_ranks[b * 32 + tid] = srank[tid];
    if (!grid_sync(bar, static_cast<uint32_t>(G), a.err, ok_smem))
        return;

    // phase 3: base per expert = totals of the CTAs before this one; CTA 0
    // also forms the counts, offsets and rank totals
    constexpr int kUnroll = kGridMaxBlocks; // every CTA's total in flight at once
    int carry = 0;
    for (int e0 = 0; e0 < a.E; e0 += kGridThreads) {
        const int e = e0 + tid;
        int bs = 0, all = 0;
        if (e < a.E) {
            for (int j0 = 0; j0 < G; j0 += kUnroll) {
                int v[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u)
                    v[u] = j0 + u < G ? __ldcg(tile_counts + static_cast<int64_t>(j0 + u) * a.E + e) : 0;
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    bs += j0 + u < b ? v[u] : 0;
                    all += v[u];
                }
            }
#pragma unroll
            for (int w = 0; w < kGridWarps; ++w)
                wtab[w * a.E + e] += bs;
        }
        if (b == 0) {
            int total = 0;
            const int excl = block_exclusive_scan(e < a.E ? all : 0, sscan, total);
            if (e < a.E) {
                a.counts[e] = all;
                a.offsets[e] = carry + excl;
            }
            carry += total;
        }
    }
    if (b == 0) {
        if (tid == 0)
            a.offsets[a.E] = carry;
        if (tid < a.R) {
            int v[kGridMaxBlocks];
#pragma unroll
            for (int j = 0; j < kGridMaxBlocks; ++j)
                v[j] = j < G ? __ldcg(tile_ranks + j * 32 + tid) : 0;
            int n = 0;
#pragma unroll
            for (int j = 0; j < kGridMaxBlocks; ++j)
                n += v[j];
            a.rank_counts[tid] = n;
        }
    }
    __syncthreads();

    // phase 4: slots and rank rows
    if (in_regs) {
#pragma unroll
        for (int j = 0; j < kGridPrefetch; ++j) {
            const int64_t p = wb + j * 32 + lane;
            if (p < we)
                a.slot[p] = loc[j] >= 0 ? loc[j] + mine[ev[j]] : -1;
        }
    } else {
        for (int64_t step = wb; step < we; step += 32) {
            const int64_t p = step + lane;
            if (p < we) {
                const int32_t l = a.slot[p];
                if (l >= 0)
                    a.slot[p] = l + mine[__ldg(a.topk_idx + p)];
            }
        }
    }
    if (ids_in_smem) {
        for (int64_t t = t0 + tid; t < t1; t += kGridThreads)
            write_rank_row(a, t, smask[t - t0]);
    }
}

// ---------------------------------------------------------------- expert choice
struct EcArgs {
    const int32_t* ti;
    int32_t T, E, C, R, per_rank;
    int32_t* counts;
    int32_t* rank_counts;
    uint8_t* in_rank;
    int32_t* token_offsets;
    int32_t* token_slots;
    uint32_t* tmask;
    int32_t* fill;
    int32_t* scratch;
    uint32_t* err;
};

constexpr int kEcThreads = 256;

// grid: E * ceil(C / kEcThreads) blocks; block b covers expert b / cblocks.
__global__ void __launch_bounds__(kEcThreads) ec_count_kernel(EcArgs a, int32_t cblocks)
{
    const int e = static_cast<int>(blockIdx.x / cblocks);
    const int64_t c = static_cast<int64_t>(blockIdx.x % cblocks) * kEcThreads + threadIdx.x;
    int valid = 0;
    if (c < a.C) {
        const int t = __ldg(a.ti + static_cast<int64_t>(e) * a.C + c);
        if (t >= 0 && t < a.T) {
            valid = 1;
            atomicAdd(a.token_offsets + 1 + t, 1);
            atomicOr(a.tmask + t, 1u << static_cast<uint32_t>(e / a.per_rank));
        } else if (t != -1) {
            flag_error(a.err, EP_DEVERR_BAD_INDEX);
        }
    }
    const int n = __syncthreads_count(valid);
    if (threadIdx.x == 0 && n)
        atomicAdd(a.counts + e, n);
}

constexpr int kScanThreads = 1024;
constexpr int kScanPerThread = 8;

// In-place inclusive scan of token_offsets[1..T] (degrees) -> offsets, and
// the rank membership of every token.  One CTA.
__global__ void __launch_bounds__(kScanThreads, 1) ec_scan_kernel(EcArgs a)
{
    __shared__ int warp_sums[32];
    __shared__ int srank[32];
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid < 32)
        srank[tid] = 0;
    int carry = 0;
    int32_t* deg = a.token_offsets + 1;
    for (int64_t base = 0; base < a.T; base += static_cast<int64_t>(kScanThreads) * kScanPerThread) {
        int v[kScanPerThread];
        int run = 0;
#pragma unroll
        for (int j = 0; j < kScanPerThread; ++j) {
            const int64_t i = base + static_cast<int64_t>(tid) * kScanPerThread + j;
            v[j] = i < a.T ? deg[i] : 0;
            run += v[j];
            v[j] = run;
        }
        int total = 0;
        const int excl = block_exclusive_scan(run, warp_sums, total);
#pragma unroll
        for (int j = 0; j < kScanPerThread; ++j) {
            const int64_t i = base + static_cast<int64_t>(tid) * kScanPerThread + j;
            if (i < a.T)
                deg[i] = carry + excl + v[j];
        }
        carry += total;
    }
    __syncthreads();
    for (int64_t tb = static_cast<int64_t>(tid & ~31); tb < a.T; tb += kScanThreads) {
        const int64_t t = tb + lane;
        uint32_t mask = 0;
        if (t < a.T) {
            mask = a.tmask[t];
            for (int r = 0; r < a.R; ++r)
                a.in_rank[t * a.R + r] = static_cast<uint8_t>((mask >> r) & 1u);
        }
        for (int r = 0; r < a.R; ++r) {
            const int c = __popc(__ballot_sync(kFullMask, (mask >> r) & 1u));
            if (lane == 0 && c)
                atomicAdd(&srank[r], c);
        }
    }
    __syncthreads();
    if (tid < a.R)
        a.rank_counts[tid] = srank[tid];
}

__global__ void __launch_bounds__(kEcThreads) ec_fill_kernel(EcArgs a)
{
    const int64_t s = static_cast<int64_t>(blockIdx.x) * kEcThreads + threadIdx.x;
    if (s >= static_cast<int64_t>(a.E) * a.C)
        return;
    const int t = __ldg(a.ti + s);
    if (t < 0 || t >= a.T)
        return;
    const int pos = atomicAdd(a.fill + t, 1);
    a.scratch[a.token_offsets[t] + pos] = static_cast<int32_t>(s);
}

// One warp per token: entry i of the unordered list goes to position
// (number of entries smaller than it).  Values are processed 32 at a time
// against all entries, broadcast by shuffles.
__global__ void __launch_bounds__(kEcThreads) ec_sort_kernel(EcArgs a)
{
    const int64_t t = (static_cast<int64_t>(blockIdx.x) * kEcThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= a.T)
        return;
    const int beg = a.token_offsets[t];
    const int n = a.token_offsets[t + 1] - beg;
    const int32_t* src = a.scratch + beg;
    int32_t* dst = a.token_slots + beg;
    if (n == 1) {
        if (lane == 0)
            dst[0] = src[0];
        return;
    }
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const int32_t v = i < n ? src[i] : 0x7fffffff;
        int rank = 0;
        for (int j0 = 0; j0 < n; j0 += 32) {
            const int32_t u = j0 + lane < n ? src[j0 + lane] : 0x7fffffff;
            const int m = min(32, n - j0);
            for (int j = 0; j < m; ++j)
                rank += __shfl_sync(kFullMask, u, j) < v ? 1 : 0;
        }
        if (i < n)
            dst[rank] = v;
    }
}

// Expert choice in one launch: a cluster of up to 16 CTAs, CTA j holding a
// contiguous range of slots and owning a contiguous range of tokens.
//   1. one warp walks the CTA's slots in order (32 at a time, equal token ids
//      ranked by __match_any_sync) keeping a per-token counter in shared
//      memory: the rank of a slot among the CTA's slots of its token;
//      the other warps OR rank bits per token and count each expert's row;
//   2. cluster barrier; each owner reads every CTA's counters of its tokens
//      over DSMEM: degree, rank mask, and the CTA's total; the degrees are
//      scanned over the owner's range;
//   3. cluster barrier; owners add the totals of earlier owners, write
//      token_offsets, and store into every CTA i's shared memory the start of
//      CTA i's run inside each owned token's list (offset + counts of CTAs
//      before i);
//   4. cluster barrier; every slot is written at start + its rank.
// Slot lists come out in ascending slot order with integer arithmetic only.
constexpr int kEcClusterThreads = 256;
constexpr int64_t kEcClusterMaxT = 16384;
constexpr int64_t kEcClusterSlotsPerCta = 2048;
constexpr int kEcClusterPrefetch = 16; // ranking steps whose lane sets are formed together
constexpr int64_t kEcClusterOwnMax = 4 * kEcClusterThreads; // tokens owned per CTA, 4 per thread
constexpr int64_t kEcClusterMaxE = 2048;

struct EcClusterArgs {
    const int32_t* ti;
    int32_t T, E, C, R, per_rank;
    int32_t* counts;
    int32_t* rank_counts;
    uint8_t* in_rank;
    int32_t* token_offsets;
    int32_t* token_slots;
    uint32_t* err;
    int32_t trigger; // let the dispatch launched next start at once
};

// per-token arrays are padded to a multiple of 4 tokens for 16-byte DSMEM access
__host__ __device__ inline int64_t ec_padded_tokens(int64_t T)
{
    return (T + 3) / 4 * 4;
}

size_t ec_cluster_smem_bytes(int64_t T, int64_t spc, int64_t E)
{
    return sizeof(int32_t) * static_cast<size_t>(3 * ec_padded_tokens(T) + 2 * spc + E + 32 + 32 + 8);
}

__global__ void __launch_bounds__(kEcClusterThreads, 1) ec_layout_cluster_kernel(EcClusterArgs a, int32_t spc)
{
    if (a.trigger)
        pdl_launch_dependents(); // the dispatch of the same call may load its rows now
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = static_cast<int>(cluster.num_blocks());
    const int b = static_cast<int>(cluster.block_rank());
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t S = static_cast<int64_t>(a.E) * a.C;
    const int64_t Tp = ec_padded_tokens(a.T);
    // owned token ranges are multiples of 4 tokens
    const int64_t own = ((Tp / 4 + cs - 1) / cs) * 4;
    extern __shared__ __align__(16) int32_t smem[];
    int32_t* hist = smem;                                      // [Tp] this CTA's slots per token
    uint32_t* tmask = reinterpret_cast<uint32_t*>(hist + Tp);  // [Tp] rank bits of this CTA's slots
    int32_t* start = reinterpret_cast<int32_t*>(tmask + Tp);   // [Tp] where this CTA's run of a token starts
    int32_t* sid = start + Tp;                                 // [spc] token of each slot (-1: none)
    int32_t* lrank = sid + spc;                                // [spc] rank of each slot in its token's run
    int32_t* pcount = lrank + spc;                             // [E] this CTA's filled slots per expert
    int32_t* srank = pcount + a.E;                             // [32] owner: tokens per rank
    int32_t* sscan = srank + 32;                               // [32] scan scratch
    int32_t* rtot = sscan + 32;                                // [1] owner: total picks of its tokens

    for (int64_t i = tid; i < Tp; i += kEcClusterThreads) {
        hist[i] = 0;
        tmask[i] = 0u;
    }
    for (int e = tid; e < a.E; e += kEcClusterThreads)
        pcount[e] = 0;
    if (tid < 32)
        srank[tid] = 0;
    __syncthreads();

    // 1. the CTA's slots: ids into shared memory (all warps, one pass),
    // rank bits per token and filled slots per expert
    const int64_t s0 = min(S, static_cast<int64_t>(b) * spc);
    const int64_t s1 = min(S, s0 + spc);
    bool bad = false;
    // every id of this thread in flight at once (spc <= kEcClusterSlotsPerCta)
    constexpr int kIdsPerThread = static_cast<int>(kEcClusterSlotsPerCta / kEcClusterThreads);
    int tids[kIdsPerThread];
#pragma unroll
    for (int i = 0; i < kIdsPerThread; ++i) {
        const int64_t s = s0 + (tid & ~31) + static_cast<int64_t>(i) * kEcClusterThreads + lane;
        tids[i] = s < s1 ? __ldg(a.ti + s) : -1;
    }
#pragma unroll
    for (int i = 0; i < kIdsPerThread; ++i) {
        const int64_t sb = s0 + (tid & ~31) + static_cast<int64_t>(i) * kEcClusterThreads;
        if (sb >= s1)
            break; // warp-uniform
        const int64_t s = sb + lane;
        const bool in = s < s1;
        const int t = tids[i];
        const bool good = in && t >= 0 && t < a.T;
        bad |= in && !good && t != -1;
        const int e = in ? static_cast<int>(s / a.C) : -1;
        if (in)
            sid[s - s0] = good ? t : -1;
        if (good)
            atomicOr(&tmask[t], 1u << static_cast<uint32_t>(e / a.per_rank));
        // lanes of one expert add their filled slots once
        const uint32_t peers = __match_any_sync(kFullMask, e);
        const int n = __popc(__ballot_sync(kFullMask, good) & peers);
        if (in && (__ffs(peers) - 1) == lane && n)
            atomicAdd(&pcount[e], n);
    }
    __syncthreads();
    if (warp == 0) {
        // ranking walk over the staged ids, 32 slots per step
        const uint32_t lanes_below = (1u << lane) - 1u;
        for (int64_t base = s0; base < s1; base += 32 * kEcClusterPrefetch) {
            // equal-token lane sets of kEcClusterPrefetch steps issued together,
            // then the dependent counter updates step after step
            int key[kEcClusterPrefetch];
            uint32_t peers[kEcClusterPrefetch];
#pragma unroll
            for (int j = 0; j < kEcClusterPrefetch; ++j) {
                const int64_t s = base + j * 32 + lane;
                key[j] = s < s1 ? sid[s - s0] : -1;
            }
#pragma unroll
            for (int j = 0; j < kEcClusterPrefetch; ++j)
                peers[j] = base + j * 32 < s1 ? __match_any_sync(kFullMask, key[j]) : 0u;
#pragma unroll
            for (int j = 0; j < kEcClusterPrefetch; ++j) {
                if (base + j * 32 >= s1)
                    break; // warp-uniform
                const int64_t s = base + j * 32 + lane;
                int prior = 0;
                if (key[j] >= 0)
                    prior = hist[key[j]];
                __syncwarp();
                if (key[j] >= 0) {
                    const int r = __popc(peers[j] & lanes_below);
                    lrank[s - s0] = prior + r;
                    if (r == 0)
                        hist[key[j]] = prior + __popc(peers[j]);
                }
                __syncwarp();
            }
        }
    }
    if (__any_sync(kFullMask, bad) && lane == 0)
        flag_error(a.err, EP_DEVERR_BAD_INDEX);
    __syncthreads();
    cluster.sync();

    // 2. owner of tokens [u0, u1), four per thread: every CTA's counters of
    // the four tokens in one 16-byte DSMEM load each, kept in registers
    const int64_t u0 = min(Tp, static_cast<int64_t>(b) * own);
    const int64_t u1 = min(static_cast<int64_t>(a.T), u0 + own);
    const int64_t t4 = u0 + 4 * static_cast<int64_t>(tid);
    const bool owns = t4 < u1;
    int4 h[kMaxCluster];
    int deg[4] = {0, 0, 0, 0};
    uint32_t mask[4] = {0u, 0u, 0u, 0u};
    if (owns) {
        uint4 m[kMaxCluster];
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j) {
            h[j] = j < cs ? *reinterpret_cast<const int4*>(cluster.map_shared_rank(hist, j) + t4) : make_int4(0, 0, 0, 0);
            m[j] = j < cs ? *reinterpret_cast<const uint4*>(cluster.map_shared_rank(tmask, j) + t4)
                          : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j) {
            deg[0] += h[j].x;
            deg[1] += h[j].y;
            deg[2] += h[j].z;
            deg[3] += h[j].w;
            mask[0] |= m[j].x;
            mask[1] |= m[j].y;
            mask[2] |= m[j].z;
            mask[3] |= m[j].w;
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        for (int r = 0; r < a.R; ++r) {
            const int c = __popc(__ballot_sync(kFullMask, (mask[i] >> r) & 1u));
            if (lane == 0 && c)
                atomicAdd(&srank[r], c);
        }
    }
    // CTA 0: filled slots per expert, summed over the cluster
    int ecount = 0;
    const int e_own = tid;
    if (b == 0) {
        for (int e = tid; e < a.E; e += kEcClusterThreads) {
            int v[kMaxCluster];
#pragma unroll
            for (int j = 0; j < kMaxCluster; ++j)
                v[j] = j < cs ? cluster.map_shared_rank(pcount, j)[e] : 0;
            int n = 0;
#pragma unroll
            for (int j = 0; j < kMaxCluster; ++j)
                n += v[j];
            if (e == e_own)
                ecount = n;
            else
                a.counts[e] = n; // E > threads: rare, written directly
        }
    }
    int range_total = 0;
    const int excl = block_exclusive_scan(deg[0] + deg[1] + deg[2] + deg[3], sscan, range_total);
    if (tid == 0)
        rtot[0] = range_total;
    __syncthreads();
    cluster.sync();

    // 3. owners: global offsets, and the start of every CTA's run in each token
    int carry = 0;
    {
        int v[kMaxCluster];
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j)
            v[j] = j < b ? cluster.map_shared_rank(rtot, j)[0] : 0;
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j)
            carry += v[j];
    }
    int off[4];
    off[0] = carry + excl;
    off[1] = off[0] + deg[0];
    off[2] = off[1] + deg[1];
    off[3] = off[2] + deg[2];
    if (owns) {
        int4 pre = make_int4(off[0], off[1], off[2], off[3]);
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j) {
            if (j < cs) {
                *reinterpret_cast<int4*>(cluster.map_shared_rank(start, j) + t4) = pre;
                pre.x += h[j].x;
                pre.y += h[j].y;
                pre.z += h[j].z;
                pre.w += h[j].w;
            }
        }
    }
    int rank_total = 0;
    if (b == 0 && tid < a.R) {
        int v[kMaxCluster];
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j)
            v[j] = j < cs ? cluster.map_shared_rank(srank, j)[tid] : 0;
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j)
            rank_total += v[j];
    }
    cluster.sync();

    // 4. global outputs, after the last cluster barrier (so no barrier waits
    // for them): every filled slot at its run's start + its rank, then the
    // owners' offsets and rank rows, CTA 0's counts
    for (int64_t s = s0 + tid; s < s1; s += kEcClusterThreads) {
        const int t = sid[s - s0];
        if (t >= 0)
            a.token_slots[start[t] + lrank[s - s0]] = static_cast<int32_t>(s);
    }
    if (owns) {
        for (int i = 0; i < 4; ++i) {
            if (t4 + i >= u1)
                break;
            a.token_offsets[t4 + i] = off[i];
            uint8_t* row = a.in_rank + (t4 + i) * a.R;
            for (int r = 0; r < a.R; ++r)
                row[r] = static_cast<uint8_t>((mask[i] >> r) & 1u);
        }
    }
    if (b == cs - 1 && tid == 0)
        a.token_offsets[a.T] = carry + rtot[0];
    if (b == 0) {
        if (e_own < a.E)
            a.counts[e_own] = ecount;
        if (tid < a.R)
            a.rank_counts[tid] = rank_total;
    }
}

// per-device caches of driver queries (host threads may race to fill an
// entry; they store the same value)
std::atomic<int> cluster_limit_cache[64];
std::atomic<size_t> smem_attr_cache[64];

// Kernel attributes (dynamic shared memory limit, 16-CTA clusters) are set
// once per device and shared-memory size; later calls skip the driver calls.
cudaError_t prepare_layout_kernel(size_t smem)
{
    int dev = 0;
    cudaError_t st = cudaGetDevice(&dev);
    if (st != cudaSuccess)
        return st;
    if (dev >= 0 && dev < 64 && smem_attr_cache[dev].load(std::memory_order_relaxed) >= smem)
        return cudaSuccess;
    const size_t want = std::max<size_t>(smem, sizeof(int32_t) * (kLayoutWarps * 256 + 3 * 256 + 64 + 2 * kSmemIds));
    st = cudaFuncSetAttribute(tc_layout_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(want));
    if (st != cudaSuccess)
        return st;
    st = cudaFuncSetAttribute(tc_layout_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (st != cudaSuccess)
        return st;
    if (dev >= 0 && dev < 64)
        smem_attr_cache[dev].store(want, std::memory_order_relaxed);
    return cudaSuccess;
}

int max_layout_cluster(size_t smem_bytes)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 8;
    int cached = cluster_limit_cache[dev].load(std::memory_order_relaxed);
    if (cached > 0)
        return cached;
    int best = 8;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(16);
    cfg.blockDim = dim3(kLayoutThreads);
    cfg.dynamicSmemBytes = smem_bytes;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 16;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, tc_layout_cluster_kernel, &cfg) == cudaSuccess && n >= 1)
        best = 16;
    cudaGetLastError();
    cluster_limit_cache[dev].store(best, std::memory_order_relaxed);
    return best;
}

std::atomic<int> ec_cluster_limit_cache[64];

// 16-CTA clusters of the expert-choice kernel fit on this device (else 8).
int max_ec_cluster()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 8;
    const int cached_ec = ec_cluster_limit_cache[dev].load(std::memory_order_relaxed);
    if (cached_ec > 0)
        return cached_ec;
    int best = 8;
    const size_t smem = ec_cluster_smem_bytes(kEcClusterMaxT, kEcClusterSlotsPerCta, kEcClusterMaxE);
    if (cudaFuncSetAttribute(ec_layout_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) == cudaSuccess &&
        cudaFuncSetAttribute(ec_layout_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        cfg.gridDim = dim3(16);
        cfg.blockDim = dim3(kEcClusterThreads);
        cfg.dynamicSmemBytes = smem;
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 16;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, ec_layout_cluster_kernel, &cfg) == cudaSuccess && n >= 1)
            best = 16;
    }
    cudaGetLastError();
    ec_cluster_limit_cache[dev].store(best, std::memory_order_relaxed);
    return best;
}

} // namespace

size_t tc_layout_workspace_bytes(int64_t E)
{
    return kWorkspaceHeaderBytes + sizeof(int32_t) * static_cast<size_t>(kGridMaxBlocks) * (E + 32);
}

std::atomic<int> grid_blocks_cache[64];

cudaError_t launch_tc_layout_grid(const TcArgs& k, void* workspace, cudaStream_t stream)
{
    int dev = 0;
    cudaError_t st = cudaGetDevice(&dev);
    if (st != cudaSuccess)
        return st;
    const size_t smem = sizeof(int32_t) * (static_cast<size_t>(kGridWarps) * k.E + 64 + 2 * kGridIds + 4);
    int resident = dev >= 0 && dev < 64 ? grid_blocks_cache[dev].load(std::memory_order_relaxed) : 0;
    if (resident == 0) {
        const size_t max_smem = sizeof(int32_t) * (static_cast<size_t>(kGridWarps) * kMaxTopkLayoutExperts + 64 +
                                                   2 * kGridIds + 4);
        st = cudaFuncSetAttribute(tc_layout_grid_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(max_smem));
        if (st != cudaSuccess)
            return st;
        int sms = 0, per_sm = 0;
        st = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (st == cudaSuccess)
            st = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tc_layout_grid_kernel, kGridThreads, max_smem);
        if (st != cudaSuccess)
            return st;
        resident = std::max(1, sms * per_sm);
        if (dev >= 0 && dev < 64)
            grid_blocks_cache[dev].store(resident, std::memory_order_relaxed);
    }
    const int64_t pairs = static_cast<int64_t>(k.T) * k.K;
    const int G = static_cast<int>(std::min<int64_t>(
        {static_cast<int64_t>(kGridMaxBlocks), static_cast<int64_t>(resident),
         std::max<int64_t>(1, (pairs + kGridPairsPerCta - 1) / kGridPairsPerCta)}));
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* tile_counts = reinterpret_cast<int32_t*>(ws + kWorkspaceHeaderBytes);
    int32_t* tile_ranks = tile_counts + static_cast<int64_t>(kGridMaxBlocks) * k.E;
    GridBar bar{reinterpret_cast<uint32_t*>(ws + 64), reinterpret_cast<uint32_t*>(ws + 128)};
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kGridThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, tc_layout_grid_kernel, k, tile_counts, tile_ranks, bar);
}

cudaError_t launch_tc_layout(const TcLayoutLaunch& a, cudaStream_t stream)
{
    TcArgs k{};
    k.topk_idx = a.topk_idx;
    k.T = a.T;
    k.K = a.K;
    k.E = a.E;
    k.R = a.R;
    k.per_rank = a.E / a.R;
    k.counts = a.counts;
    k.offsets = a.offsets;
    k.rank_counts = a.rank_counts;
    k.in_rank = a.in_rank;
    k.slot = a.slot;
    k.err = a.err;
    k.in_rank_words = (a.R % 4 == 0 && (reinterpret_cast<uintptr_t>(a.in_rank) & 3u) == 0) ? 1 : 0;
    k.trigger = a.trigger_dependents;

    if (static_cast<int64_t>(a.T) * a.K >= EP_LAYOUT_GRID_MIN_PAIRS && a.workspace != nullptr)
        return launch_tc_layout_grid(k, a.workspace, stream);

    const size_t smem =
        sizeof(int32_t) * (static_cast<size_t>(kLayoutWarps) * a.E + 3 * static_cast<size_t>(a.E) + 64 + 2 * kSmemIds);
    cudaError_t st = prepare_layout_kernel(smem);
    if (st != cudaSuccess)
        return st;
    const int64_t pairs = static_cast<int64_t>(a.T) * a.K;
    int cs = static_cast<int>(
        std::min<int64_t>(EP_LAYOUT_MAX_CLUSTER, std::max<int64_t>(1, (pairs + kPairsPerCta - 1) / kPairsPerCta)));
    if (cs > 8)
        cs = std::min(cs, max_layout_cluster(smem));

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(cs);
    cfg.blockDim = dim3(kLayoutThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (EP_LAYOUT_SINGLE_PLAIN && cs == 1) ? 0 : 1;
    return cudaLaunchKernelEx(&cfg, tc_layout_cluster_kernel, k);
}

size_t ec_layout_workspace_bytes(int64_t T, int64_t E, int64_t C)
{
    const size_t arrays = sizeof(int32_t) * static_cast<size_t>(2 * T + E * C);
    return kWorkspaceHeaderBytes + ((arrays + 255) / 256) * 256;
}

std::atomic<int> ec_smem_attr_dev[64];

cudaError_t launch_ec_layout_cluster(const EcLayoutLaunch& a, cudaStream_t stream, bool& launched)
{
    launched = false;
    const int64_t S = static_cast<int64_t>(a.E) * a.C;
    if (a.T > kEcClusterMaxT || S > kMaxCluster * kEcClusterSlotsPerCta)
        return cudaSuccess;
    // enough CTAs for <= 1024 slots and <= kEcClusterOwnMax owned tokens each, if possible
    const int64_t Tp = ec_padded_tokens(a.T);
    int cs = static_cast<int>(std::min<int64_t>(
        kMaxCluster, std::max<int64_t>({int64_t{1}, (S + 1023) / 1024, (Tp + kEcClusterOwnMax - 1) / kEcClusterOwnMax})));
    if (cs > 8 && max_ec_cluster() < 16)
        cs = 8;
    const int64_t spc = (S + cs - 1) / cs;
    const int64_t own = ((Tp / 4 + cs - 1) / cs) * 4;
    if (spc > kEcClusterSlotsPerCta || own > kEcClusterOwnMax || a.E > kEcClusterMaxE)
        return cudaSuccess; // too large for one cluster: the multi-kernel path below
    const size_t smem = ec_cluster_smem_bytes(a.T, spc, a.E);
    int dev = 0;
    cudaError_t st = cudaGetDevice(&dev);
    if (st != cudaSuccess)
        return st;
    if (dev < 0 || dev >= 64 || ec_smem_attr_dev[dev] == 0) {
        st = cudaFuncSetAttribute(ec_layout_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(ec_cluster_smem_bytes(kEcClusterMaxT, kEcClusterSlotsPerCta, kEcClusterMaxE)));
        if (st == cudaSuccess)
            st = cudaFuncSetAttribute(ec_layout_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (st != cudaSuccess)
            return st;
        if (dev >= 0 && dev < 64)
            ec_smem_attr_dev[dev] = 1;
    }
    EcClusterArgs k{a.token_indices, a.T, a.E, a.C, a.R, a.E / a.R, a.counts, a.rank_counts, a.in_rank,
                    a.token_offsets, a.token_slots, a.err, a.trigger_dependents};
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(cs);
    cfg.blockDim = dim3(kEcClusterThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    launched = true;
    return cudaLaunchKernelEx(&cfg, ec_layout_cluster_kernel, k, static_cast<int32_t>(spc));
}

cudaError_t launch_ec_layout(const EcLayoutLaunch& a, cudaStream_t stream)
{
    bool launched = false;
    cudaError_t cst = launch_ec_layout_cluster(a, stream, launched);
    if (cst != cudaSuccess || launched)
        return cst;
    EcArgs k{};
    k.ti = a.token_indices;
    k.T = a.T;
    k.E = a.E;
    k.C = a.C;
    k.R = a.R;
    k.per_rank = a.E / a.R;
    k.counts = a.counts;
    k.rank_counts = a.rank_counts;
    k.in_rank = a.in_rank;
    k.token_offsets = a.token_offsets;
    k.token_slots = a.token_slots;
    uint8_t* ws = static_cast<uint8_t*>(a.workspace) + kWorkspaceHeaderBytes;
    k.tmask = reinterpret_cast<uint32_t*>(ws);
    k.fill = reinterpret_cast<int32_t*>(ws) + a.T;
    k.scratch = reinterpret_cast<int32_t*>(ws) + 2 * static_cast<int64_t>(a.T);
    k.err = a.err;

    cudaError_t st = cudaMemsetAsync(a.token_offsets, 0, sizeof(int32_t) * (static_cast<size_t>(a.T) + 1), stream);
    if (st == cudaSuccess)
        st = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * static_cast<size_t>(a.E), stream);
    if (st == cudaSuccess && a.T > 0)
        st = cudaMemsetAsync(ws, 0, sizeof(int32_t) * 2 * static_cast<size_t>(a.T), stream);
    if (st != cudaSuccess)
        return st;
    const int32_t cblocks = (a.C + kEcThreads - 1) / kEcThreads;
    const int64_t count_blocks = static_cast<int64_t>(a.E) * cblocks;
    if (count_blocks >= (int64_t{1} << 31))
        return cudaErrorInvalidValue;
    ec_count_kernel<<<static_cast<unsigned>(count_blocks), kEcThreads, 0, stream>>>(k, cblocks);
    ec_scan_kernel<<<1, kScanThreads, 0, stream>>>(k);
    const int64_t S = static_cast<int64_t>(a.E) * a.C;
    ec_fill_kernel<<<static_cast<unsigned>((S + kEcThreads - 1) / kEcThreads), kEcThreads, 0, stream>>>(k);
    if (a.T > 0) {
        const int64_t warps_per_block = kEcThreads / 32;
        ec_sort_kernel<<<static_cast<unsigned>((a.T + warps_per_block - 1) / warps_per_block), kEcThreads, 0,
                         stream>>>(k);
    }
    return cudaGetLastError();
}

} // namespace ep
