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

#include <cooperative_groups.h>

#include "ep_device.cuh"
#include "ep_internal.h"

namespace cg = cooperative_groups;

namespace ep {

namespace {

constexpr int kLayoutThreads = 1024;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kPrefetch = 8; // 32-pair steps a warp loads before ranking them
constexpr int64_t kPairsPerCta = 2048;
constexpr int kMaxCluster = 16;

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
};

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
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = static_cast<int>(cluster.num_blocks());
    const int b = static_cast<int>(cluster.block_rank());
    extern __shared__ __align__(16) int32_t smem[];
    int32_t* wtab = smem;                      // [32][E] per-warp counters, later prefixes
    int32_t* tot = wtab + kLayoutWarps * a.E;  // [E] this CTA's pairs per expert
    int32_t* srank = tot + a.E;                // [32] this CTA's tokens per rank
    int32_t* sscan = srank + 32;               // [32] scan scratch
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
    // one prefetch batch (<= 256 pairs) the ids and ranks stay in registers;
    // longer runs park the rank in slot[] and re-read it in phase 3.
    const bool in_regs = (we - wb) <= 32 * kPrefetch;
    int ev[kPrefetch]; // expert id, or -1 for a pair that is not routed
    int loc[kPrefetch];
    for (int64_t base = wb; base < we; base += 32 * kPrefetch) {
        int64_t raw[kPrefetch];
#pragma unroll
        for (int j = 0; j < kPrefetch; ++j) {
            const int64_t p = base + j * 32 + lane;
            raw[j] = p < we ? __ldg(a.topk_idx + p) : -1;
        }
#pragma unroll
        for (int j = 0; j < kPrefetch; ++j) {
            const bool ok = raw[j] >= 0 && raw[j] < a.E;
            bad |= !ok && raw[j] != -1;
            ev[j] = ok ? static_cast<int>(raw[j]) : -1;
        }
#pragma unroll
        for (int j = 0; j < kPrefetch; ++j) {
            loc[j] = -1;
            const int64_t step = base + j * 32;
            if (step >= we)
                break; // warp-uniform
            const int64_t p = step + lane;
            const bool in = p < we;
            const int e = ev[j];
            const bool good = e >= 0;
            const uint32_t peers = __match_any_sync(kFullMask, e);
            int prior = 0;
            if (good)
                prior = mine[e];
            __syncwarp();
            if (good) {
                const int r = __popc(peers & lanes_below);
                loc[j] = prior + r;
                if (r == 0)
                    mine[e] = prior + __popc(peers);
            }
            if (!in_regs && in)
                a.slot[p] = loc[j];
            __syncwarp();
        }
    }

    // phase 1b: rank membership of this CTA's tokens (ids re-read from L1/L2,
    // all of a token's loads issued before any is used)
    constexpr int kMaskBatch = 8;
    for (int64_t tb = t0 + static_cast<int64_t>(warp) * 32; tb < t1; tb += kLayoutThreads) {
        const int64_t t = tb + lane;
        uint32_t mask = 0;
        if (t < t1) {
            for (int k0 = 0; k0 < a.K; k0 += kMaskBatch) {
                int64_t ids[kMaskBatch];
#pragma unroll
                for (int k = 0; k < kMaskBatch; ++k)
                    ids[k] = k0 + k < a.K ? __ldg(a.topk_idx + t * a.K + k0 + k) : -1;
#pragma unroll
                for (int k = 0; k < kMaskBatch; ++k)
                    if (ids[k] >= 0 && ids[k] < a.E)
                        mask |= 1u << static_cast<uint32_t>(ids[k] / a.per_rank);
            }
            uint8_t* row = a.in_rank + t * a.R;
            if (a.in_rank_words) {
                for (int r = 0; r < a.R; r += 4) {
                    uint32_t w = ((mask >> r) & 1u) | (((mask >> (r + 1)) & 1u) << 8) |
                                 (((mask >> (r + 2)) & 1u) << 16) | (((mask >> (r + 3)) & 1u) << 24);
                    *reinterpret_cast<uint32_t*>(row + r) = w;
                }
            } else {
                for (int r = 0; r < a.R; ++r)
                    row[r] = static_cast<uint8_t>((mask >> r) & 1u);
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

    // phase 2: counters -> exclusive prefix down the warps; CTA totals
    const int e = tid; // E <= kLayoutThreads
    if (e < a.E) {
        int run = 0;
        for (int w = 0; w < kLayoutWarps; ++w) {
            const int c = wtab[w * a.E + e];
            wtab[w * a.E + e] = run;
            run += c;
        }
        tot[e] = run;
    }
    cluster.sync();

    // totals of every CTA of the cluster, all loads in flight together
    int base = 0, all = 0;
    if (e < a.E) {
        int v[kMaxCluster];
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j)
            v[j] = j < cs ? cluster.map_shared_rank(tot, j)[e] : 0;
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j) {
            base += j < b ? v[j] : 0;
            all += v[j];
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
    cluster.sync(); // no CTA leaves or reuses its shared memory while others read it

    if (b == 0) {
        int total = 0;
        const int excl = block_exclusive_scan(e < a.E ? all : 0, sscan, total);
        if (e < a.E) {
            a.counts[e] = all;
            a.offsets[e] = excl;
        }
        if (tid == 0)
            a.offsets[a.E] = total;
        if (tid < a.R)
            a.rank_counts[tid] = rank_total;
    }
    if (e < a.E) {
        for (int w = 0; w < kLayoutWarps; ++w)
            wtab[w * a.E + e] += base;
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

int cluster_limit_cache[64];
size_t smem_attr_cache[64];

// Kernel attributes (dynamic shared memory limit, 16-CTA clusters) are set
// once per device and shared-memory size; later calls skip the driver calls.
cudaError_t prepare_layout_kernel(size_t smem)
{
    int dev = 0;
    cudaError_t st = cudaGetDevice(&dev);
    if (st != cudaSuccess)
        return st;
    if (dev >= 0 && dev < 64 && smem_attr_cache[dev] >= smem)
        return cudaSuccess;
    const size_t want = std::max<size_t>(smem, sizeof(int32_t) * (kLayoutWarps * 256 + 256 + 64));
    st = cudaFuncSetAttribute(tc_layout_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(want));
    if (st != cudaSuccess)
        return st;
    st = cudaFuncSetAttribute(tc_layout_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (st != cudaSuccess)
        return st;
    if (dev >= 0 && dev < 64)
        smem_attr_cache[dev] = want;
    return cudaSuccess;
}

int max_layout_cluster(size_t smem_bytes)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 8;
    int cached = cluster_limit_cache[dev];
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
    cluster_limit_cache[dev] = best;
    return best;
}

} // namespace

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

    const size_t smem = sizeof(int32_t) * (static_cast<size_t>(kLayoutWarps) * a.E + a.E + 64);
    cudaError_t st = prepare_layout_kernel(smem);
    if (st != cudaSuccess)
        return st;
    const int64_t pairs = static_cast<int64_t>(a.T) * a.K;
    int cs = static_cast<int>(std::min<int64_t>(16, std::max<int64_t>(1, (pairs + kPairsPerCta - 1) / kPairsPerCta)));
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
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, tc_layout_cluster_kernel, k);
}

size_t ec_layout_workspace_bytes(int64_t T, int64_t E, int64_t C)
{
    const size_t arrays = sizeof(int32_t) * static_cast<size_t>(2 * T + E * C);
    return kWorkspaceHeaderBytes + ((arrays + 255) / 256) * 256;
}

cudaError_t launch_ec_layout(const EcLayoutLaunch& a, cudaStream_t stream)
{
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
