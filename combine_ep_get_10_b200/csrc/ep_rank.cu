// ep_rank.cu -- rank layout of the per-rank (deduplicated) path.
//
// DeepEP-Ascend README, API Overview: normal-mode dispatch sends each token
// to the expert *ranks* that need it (is_token_in_rank from
// get_dispatch_layout).  Rank r receives its tokens in ascending order, and
// the ranks' row ranges are laid end to end, so token t's row in rank r is
//   rank_offsets[r] + #{t' < t : is_token_in_rank[t', r]}.
//
// A grid of CTAs of 1024 threads, one token per thread, one 1024-token tile
// per CTA.  A CTA first counts, per rank, the tokens of all earlier tiles
// (warp ballots of each rank's bit over those tokens' rank masks: a few
// L2-resident KB per tile, no inter-CTA synchronisation, deterministic), then
// ranks its own tokens: a ballot per rank gives each lane its rank inside
// the warp and one warp per rank scans the 32 warps' counts.  The rank
// offsets come from the layout's num_tokens_per_rank (one warp scan).
//
// The per-rank path over peer memory also starts here: every rank publishes
// its num_tokens_per_rank as one row of every rank's [R, R] counts matrix,
// from which each rank's dispatch and combine find where its rows sit in
// the other ranks' buffers.
#include <algorithm>

#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kRankThreads = 1024;
constexpr int kRankWarps = kRankThreads / 32;

// Rank mask of token t: bit r set when is_token_in_rank[t, r] != 0.
__device__ __forceinline__ uint32_t token_mask(const uint8_t* in_rank, int64_t t, int R)
{
    uint32_t mask = 0;
    const uint8_t* m = in_rank + t * R;
    if ((R & 3) == 0 && (reinterpret_cast<uintptr_t>(in_rank) & 3u) == 0) { // rows of whole aligned words
        for (int i = 0; i < R / 4; ++i) {
            const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(m) + i);
#pragma unroll
            for (int b = 0; b < 4; ++b)
                mask |= (((v >> (8 * b)) & 0xFFu) != 0u ? 1u : 0u) << (4 * i + b);
        }
    } else {
        for (int r = 0; r < R; ++r)
            mask |= (__ldg(m + r) != 0 ? 1u : 0u) << r;
    }
    return mask;
}

__global__ void __launch_bounds__(kRankThreads) rank_layout_kernel(RankLayoutLaunch a)
{
    if (a.trigger_dependents)
        pdl_launch_dependents(); // the per-rank dispatch of the same call may load its rows now
    __shared__ int32_t s_base[32];             // first row of each rank in this tile
    __shared__ int32_t s_wpre[kRankWarps][33]; // per warp, per rank: counts, then rows before the warp
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int R = a.R;
    const int64_t tile = static_cast<int64_t>(blockIdx.x) * kRankThreads;

    for (int i = tid; i < kRankWarps * 33; i += kRankThreads)
        (&s_wpre[0][0])[i] = 0;
    __syncthreads();
    // tokens of the earlier tiles, per rank (four tiles' masks loaded at once)
    for (int64_t base = 0; base < tile; base += 4 * kRankThreads) {
        uint32_t m4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t u = base + i * kRankThreads + tid;
            m4[i] = u < tile ? token_mask(a.in_rank, u, R) : 0u;
        }
        for (int r = 0; r < R; ++r) {
            int c = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                c += __popc(__ballot_sync(kFullMask, (m4[i] >> r) & 1u));
            if (lane == 0)
                s_wpre[warp][r] += c;
        }
    }
    __syncthreads();
    if (warp == 0) {
        const int32_t c = lane < R ? __ldg(a.rank_counts + lane) : 0;
        int32_t inc = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t o = __shfl_up_sync(kFullMask, inc, d);
            if (lane >= d)
                inc += o;
        }
        if (lane < R && blockIdx.x == 0) {
            a.rank_offsets[lane] = inc - c;
            if (lane == R - 1)
                a.rank_offsets[R] = inc;
        }
        if (lane < R)
            s_base[lane] = inc - c;
    }
    __syncthreads();
    if (warp < R) { // warp r adds the earlier tiles' tokens of rank r
        int32_t v = s_wpre[lane][warp];
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1)
            v += __shfl_xor_sync(kFullMask, v, d);
        if (lane == 0)
            s_base[warp] += v;
    }
    __syncthreads();

    // this tile
    const int64_t t = tile + tid;
    const uint32_t mask = t < a.T ? token_mask(a.in_rank, t, R) : 0u;
    for (int r = 0; r < R; ++r) {
        const uint32_t b = __ballot_sync(kFullMask, (mask >> r) & 1u);
        if (lane == 0)
            s_wpre[warp][r] = __popc(b);
    }
    __syncthreads();
    if (warp < R) { // warp r scans rank r's counts over the 32 warps
        const int32_t c = s_wpre[lane][warp];
        int32_t inc = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t o = __shfl_up_sync(kFullMask, inc, d);
            if (lane >= d)
                inc += o;
        }
        s_wpre[lane][warp] = inc - c;
    }
    __syncthreads();
    const uint32_t lt = (1u << lane) - 1u;
    for (int r = 0; r < R; ++r) {
        const bool in = (mask >> r) & 1u;
        const uint32_t b = __ballot_sync(kFullMask, in);
        if (t < a.T)
            a.rank_row[t * R + r] = in ? s_base[r] + s_wpre[warp][r] + __popc(b & lt) : -1;
    }
}

// Row `me` of every rank's [R, R] counts matrix <- this rank's
// num_tokens_per_rank: thread (j, c) stores entry c into rank j's matrix.
__global__ void __launch_bounds__(1024) publish_counts_kernel(PublishCountsLaunch a)
{
    const int i = threadIdx.x;
    if (i >= a.R * a.R)
        return;
    const int j = i / a.R;
    const int c = i - j * a.R;
    int32_t* m = reinterpret_cast<int32_t*>(__ldg(a.rank_counts + j));
    m[a.me * a.R + c] = __ldg(a.num_tokens_per_rank + c);
}

} // namespace

cudaError_t launch_publish_counts(const PublishCountsLaunch& a, cudaStream_t stream)
{
    publish_counts_kernel<<<1, 1024, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_rank_layout(const RankLayoutLaunch& a, cudaStream_t stream)
{
    const int64_t tiles = std::max<int64_t>(1, (static_cast<int64_t>(a.T) + kRankThreads - 1) / kRankThreads);
    rank_layout_kernel<<<static_cast<unsigned>(tiles), kRankThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

} // namespace ep
