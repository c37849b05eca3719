// ep_combine.cu -- combine (gather-reduce) kernels.
//
// Token choice: DeepEP-Ascend README, API Overview, combine and
// low_latency_combine (the reduce weighted by topk_weights); the same
// kernel reduces the per-rank rows of the deduplicated path (weight 1,
// ascending rank).  Expert choice:
// DeepEP issue #595, Solution 1 (the reduce over the slots that picked the
// token, no [T, K] padding, no cap on their number).  Both skip -1 entries
// (issue #595, Solution 2).
//
// One warp per (token, hidden segment).  A segment is kVecPerLane 16-byte
// vectors per lane (8 bf16 each; 4 vectors = 2 KB of a row per warp); the
// warp fetches the token's entries (row, weight) once, 32 at a time,
// broadcasts them by shuffles and, for groups of kGroup entries, issues every
// 16-byte load of the group before any FMA so that kGroup * kVecPerLane loads
// per lane are in flight.  Each accumulator sees its entries in ascending
// order: acc = fmaf(w, y, acc) from 0 in fp32.  (A TMA-pipelined variant --
// a producer warp streaming row chunks into a shared-memory ring -- measured
// no faster at 4096 tokens and slower under expert-choice skew.)
#include <algorithm>

#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

#ifndef EP_COMBINE_VEC
#define EP_COMBINE_VEC 4
#endif
#ifndef EP_COMBINE_GROUP
#define EP_COMBINE_GROUP 4
#endif
#ifndef EP_COMBINE_THREADS
#define EP_COMBINE_THREADS 256
#endif

constexpr int kCombineThreads = EP_COMBINE_THREADS;
constexpr int kWarpsPerCta = kCombineThreads / 32;
// token choice: kTcVec 16-byte vectors per lane per segment, kTcGroup
// entries whose loads are issued together (K is small and uniform)
constexpr int kTcVec = EP_COMBINE_VEC;
constexpr int kTcGroup = EP_COMBINE_GROUP;
// expert choice: most tokens have few or no picks and a few have long lists
#ifndef EP_COMBINE_EC_VEC
#define EP_COMBINE_EC_VEC 2
#endif
#ifndef EP_COMBINE_EC_GROUP
#define EP_COMBINE_EC_GROUP 8
#endif
// token choice: uniform items, so one resident wave of persistent warps;
// expert choice: item cost varies by 100x, so blocks are scheduled dynamically
#ifndef EP_COMBINE_PERSIST_TC
#define EP_COMBINE_PERSIST_TC 1
#endif
#ifndef EP_COMBINE_PERSIST_EC
#define EP_COMBINE_PERSIST_EC 0
#endif
#ifndef EP_COMBINE_HEAVY_FIRST
#define EP_COMBINE_HEAVY_FIRST 1
#endif
constexpr int kEcVec = EP_COMBINE_EC_VEC;
constexpr int kEcGroup = EP_COMBINE_EC_GROUP;

struct CombineArgs {
    const uint8_t* y;
    int32_t T, H, nvec, nseg;
    int64_t num_y_rows;
    // token choice
    const int64_t* topk_idx;
    const int32_t* slot;
    const int32_t* offsets;
    int32_t K, E, mode, max_tokens;
    const float* topk_weights;
    // expert choice
    const int32_t* token_offsets;
    const int32_t* token_slots;
    const float* expert_weights;
    // per rank: [T, K] rows (K = R), weight 1
    const int32_t* rank_row;
    void* out;
    uint32_t* err;
    int64_t warp_base; // first (token, segment) item of this launch
    int32_t heavy_first; // expert choice: list heavy tokens first (persistent launch)
};

// expert choice, heavy first (see combine_kernel)
constexpr int kHeavyDeg = 16;
constexpr int kMaxHeavy = 2048;
constexpr int kHeavyFirstMaxT = 65536;

enum CombineSrc : int {
    kSrcTopk = 0,  // entries: the token's K (expert, slot) pairs, gate weights
    kSrcEc = 1,    // entries: the token's CSR slots, expert weights
    kSrcRanks = 2  // entries: the token's R rank rows, weight 1 (fmaf(1, y, acc) == acc + y)
};

template <int kSrc>
__device__ __forceinline__ void entry(const CombineArgs& a, int64_t t, int64_t beg, int j, int64_t& row, float& w,
                                      uint32_t& errbits)
{
    row = -1;
    w = 0.0f;
    if constexpr (kSrc == kSrcRanks) {
        const int64_t r = __ldg(a.rank_row + t * a.K + j);
        if (r < 0)
            return;
        if (r >= a.num_y_rows) {
            errbits |= EP_DEVERR_OVERFLOW;
            return;
        }
        row = r;
        w = 1.0f;
    } else if constexpr (kSrc == kSrcEc) {
        const int64_t s = __ldg(a.token_slots + beg + j);
        if (s < 0 || s >= a.num_y_rows) {
            errbits |= EP_DEVERR_OVERFLOW;
            return;
        }
        row = s;
        w = __ldg(a.expert_weights + s);
    } else {
        const int64_t e = __ldg(a.topk_idx + t * a.K + j);
        const int32_t s = __ldg(a.slot + t * a.K + j);
        if (e < 0 || e >= a.E || s < 0) {
            if (e < -1 || e >= a.E)
                errbits |= EP_DEVERR_BAD_INDEX;
            return;
        }
        int64_t r;
        if (a.mode == EP_LAYOUT_PADDED) {
            if (s >= a.max_tokens) {
                errbits |= EP_DEVERR_OVERFLOW;
                return;
            }
            r = e * a.max_tokens + s;
        } else {
            r = static_cast<int64_t>(__ldg(a.offsets + e)) + s;
        }
        if (r >= a.num_y_rows) {
            errbits |= EP_DEVERR_OVERFLOW;
            return;
        }
        row = r;
        w = __ldg(a.topk_weights + t * a.K + j);
    }
}

// Expert choice: virtual item g -> (token, segment); the first heavy_items
// items are the listed heavy tokens' segments, then every token in order.
__device__ __forceinline__ void item_token(int64_t g, int64_t heavy_items, int nseg, const int* heavy, int64_t& t,
                                           int& seg)
{
    if (g < heavy_items) {
        t = heavy[g / nseg];
        seg = static_cast<int>(g % nseg);
    } else {
        t = (g - heavy_items) / nseg;
        seg = static_cast<int>((g - heavy_items) - t * nseg);
    }
}

template <int kSrc, bool kOutF32, int kVecPerLane, int kGroup>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineArgs a)
{
    constexpr bool kExpertChoice = kSrc == kSrcEc;
    constexpr int kSegVec = 32 * kVecPerLane;
    // token choice lists are short (K); expert-choice lists reach E entries
    constexpr int kLookup = kExpertChoice ? 2 : 1;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kWarpsPerCta;
    uint32_t errbits = 0;

    // Expert choice, heavy first: every CTA lists, in token order, the tokens
    // with at least kHeavyDeg picks (the same list in every CTA); warps take
    // their items before all others, so the long lists start in the first
    // wave and overlap the light work instead of trailing it.
    __shared__ int s_heavy[kMaxHeavy];
    __shared__ uint32_t s_flags[kHeavyFirstMaxT / 32];
    __shared__ int s_wbase[kWarpsPerCta + 1];
    int n_heavy = 0;
    if (kExpertChoice && a.heavy_first) {
        const int64_t per_warp = ((static_cast<int64_t>(a.T) + kWarpsPerCta * 32 - 1) / (kWarpsPerCta * 32)) * 32;
        const int64_t w0 = min(static_cast<int64_t>(a.T), warp * per_warp);
        const int64_t w1 = min(static_cast<int64_t>(a.T), w0 + per_warp);
        int cnt = 0;
        for (int64_t base = w0; base < w1; base += 32) {
            const int64_t t = base + lane;
            const bool heavy = t < w1 && __ldg(a.token_offsets + t + 1) - __ldg(a.token_offsets + t) >= kHeavyDeg;
            const uint32_t bits = __ballot_sync(kFullMask, heavy);
            if (lane == 0)
                s_flags[base / 32] = bits;
            cnt += __popc(bits);
        }
        if (lane == 0)
            s_wbase[warp + 1] = cnt;
        __syncthreads();
        if (threadIdx.x == 0) {
            s_wbase[0] = 0;
            for (int w = 0; w < kWarpsPerCta; ++w)
                s_wbase[w + 1] += s_wbase[w];
        }
        __syncthreads();
        n_heavy = s_wbase[kWarpsPerCta];
        if (n_heavy <= kMaxHeavy) {
            int pos = s_wbase[warp];
            for (int64_t base = w0; base < w1; base += 32) {
                const uint32_t bits = s_flags[base / 32];
                if ((bits >> lane) & 1u)
                    s_heavy[pos + __popc(bits & ((1u << lane) - 1u))] = static_cast<int>(base + lane);
                pos += __popc(bits);
            }
        } else {
            n_heavy = 0; // too many to list: plain token order
        }
        __syncthreads();
    }
    const int64_t heavy_items = static_cast<int64_t>(n_heavy) * a.nseg;
    const int64_t items = heavy_items + static_cast<int64_t>(a.T) * a.nseg;
    for (int64_t gw = a.warp_base + static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + warp; gw < items;
         gw += stride) {
        int64_t t;
        int seg;
        int64_t beg = 0;
        int n;
        if constexpr (kExpertChoice) {
            item_token(gw, heavy_items, a.nseg, s_heavy, t, seg);
            beg = __ldg(a.token_offsets + t);
            n = __ldg(a.token_offsets + t + 1) - static_cast<int>(beg);
        } else {
            t = gw / a.nseg;
            seg = static_cast<int>(gw - t * a.nseg);
            n = a.K;
        }
        if (kExpertChoice && n_heavy > 0 && gw >= heavy_items && n >= kHeavyDeg)
            continue; // done in the heavy phase

        int v[kVecPerLane];
        bool vin[kVecPerLane];
#pragma unroll
        for (int j = 0; j < kVecPerLane; ++j) {
            v[j] = seg * kSegVec + j * 32 + lane;
            vin[j] = v[j] < a.nvec;
        }
        float acc[kVecPerLane][8];
#pragma unroll
        for (int j = 0; j < kVecPerLane; ++j)
#pragma unroll
            for (int i = 0; i < 8; ++i)
                acc[j][i] = 0.0f;

        const int64_t row_bytes = static_cast<int64_t>(a.H) * 2;
        // entries are looked up kLookup at a time (all of their loads in flight),
        // then folded kGroup at a time in ascending order
        for (int k0 = 0; k0 < n; k0 += 32 * kLookup) {
            int64_t my_row[kLookup];
            float my_w[kLookup];
#pragma unroll
            for (int i = 0; i < kLookup; ++i) {
                my_row[i] = -1;
                my_w[i] = 0.0f;
                const int j = k0 + 32 * i + lane;
                if (j < n)
                    entry<kSrc>(a, t, beg, j, my_row[i], my_w[i], errbits);
            }
#pragma unroll
            for (int i = 0; i < kLookup; ++i) {
                const int kb = k0 + 32 * i;
                if (kb >= n)
                    break; // warp-uniform
                const int m = min(32, n - kb);
                for (int g0 = 0; g0 < m; g0 += kGroup) {
                    int64_t rows[kGroup];
                    float ws[kGroup];
#pragma unroll
                    for (int g = 0; g < kGroup; ++g) {
                        const int src = (g0 + g) & 31;
                        rows[g] = __shfl_sync(kFullMask, my_row[i], src);
                        ws[g] = __shfl_sync(kFullMask, my_w[i], src);
                        if (g0 + g >= m)
                            rows[g] = -1;
                    }
                    uint4 d[kGroup][kVecPerLane];
#pragma unroll
                    for (int g = 0; g < kGroup; ++g)
#pragma unroll
                        for (int j = 0; j < kVecPerLane; ++j)
                            d[g][j] = (rows[g] >= 0 && vin[j])
                                          ? ld_nc_v4(a.y + rows[g] * row_bytes + static_cast<int64_t>(v[j]) * 16)
                                          : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int g = 0; g < kGroup; ++g) {
                        if (rows[g] < 0)
                            continue;
#pragma unroll
                        for (int j = 0; j < kVecPerLane; ++j) {
                            acc[j][0] = fmaf(ws[g], bf16_lo(d[g][j].x), acc[j][0]);
                            acc[j][1] = fmaf(ws[g], bf16_hi(d[g][j].x), acc[j][1]);
                            acc[j][2] = fmaf(ws[g], bf16_lo(d[g][j].y), acc[j][2]);
                            acc[j][3] = fmaf(ws[g], bf16_hi(d[g][j].y), acc[j][3]);
                            acc[j][4] = fmaf(ws[g], bf16_lo(d[g][j].z), acc[j][4]);
                            acc[j][5] = fmaf(ws[g], bf16_hi(d[g][j].z), acc[j][5]);
                            acc[j][6] = fmaf(ws[g], bf16_lo(d[g][j].w), acc[j][6]);
                            acc[j][7] = fmaf(ws[g], bf16_hi(d[g][j].w), acc[j][7]);
                        }
                    }
                }
            }
        }

#pragma unroll
        for (int j = 0; j < kVecPerLane; ++j) {
            if (!vin[j])
                continue;
            if (kOutF32) {
                float* o = static_cast<float*>(a.out) + t * a.H + static_cast<int64_t>(v[j]) * 8;
                st_cs_v4(o, make_uint4(__float_as_uint(acc[j][0]), __float_as_uint(acc[j][1]), __float_as_uint(acc[j][2]),
                                       __float_as_uint(acc[j][3])));
                st_cs_v4(o + 4, make_uint4(__float_as_uint(acc[j][4]), __float_as_uint(acc[j][5]),
                                           __float_as_uint(acc[j][6]), __float_as_uint(acc[j][7])));
            } else {
                uint8_t* o = static_cast<uint8_t*>(a.out) + t * row_bytes + static_cast<int64_t>(v[j]) * 16;
                st_cs_v4(o, make_uint4(pack_bf16x2(acc[j][0], acc[j][1]), pack_bf16x2(acc[j][2], acc[j][3]),
                                       pack_bf16x2(acc[j][4], acc[j][5]), pack_bf16x2(acc[j][6], acc[j][7])));
            }
        }
    }
    const uint32_t any = __reduce_or_sync(kFullMask, errbits);
    if (lane == 0)
        flag_error(a.err, any);
}

// Blocks of 256 threads of `kernel` resident on the whole device (SMs x
// blocks per SM), cached per device in `cache`.
template <typename Kernel>
int64_t resident_blocks(Kernel kernel, int* cache)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 0;
    if (cache[dev] == 0) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kCombineThreads, 0) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        cache[dev] = sms * std::max(per_sm, 1);
    }
    return cache[dev];
}

// persistent: one resident wave of warps loops over the (token, segment)
// items instead of one short-lived block per 8 items
template <int kSrc, int kVec, int kGrp>
cudaError_t launch_combine(CombineArgs k, bool out_f32, bool persistent, cudaStream_t stream)
{
    constexpr int64_t kMaxBlocks = int64_t{1} << 30;
    k.nseg = (k.nvec + 32 * kVec - 1) / (32 * kVec);
    const int64_t warps = static_cast<int64_t>(k.T) * k.nseg;
    int64_t blocks = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
    if (persistent) {
        static int cache_bf16[64], cache_f32[64];
        const int64_t res = out_f32 ? resident_blocks(combine_kernel<kSrc, true, kVec, kGrp>, cache_f32)
                                    : resident_blocks(combine_kernel<kSrc, false, kVec, kGrp>, cache_bf16);
        if (res > 0)
            blocks = std::min(blocks, res);
    }
    for (int64_t b0 = 0; b0 < blocks; b0 += kMaxBlocks) {
        k.warp_base = b0 * kWarpsPerCta;
        const unsigned n = static_cast<unsigned>(blocks - b0 < kMaxBlocks ? blocks - b0 : kMaxBlocks);
        if (out_f32)
            combine_kernel<kSrc, true, kVec, kGrp><<<n, kCombineThreads, 0, stream>>>(k);
        else
            combine_kernel<kSrc, false, kVec, kGrp><<<n, kCombineThreads, 0, stream>>>(k);
        cudaError_t st = cudaGetLastError();
        if (st != cudaSuccess)
            return st;
    }
    return cudaSuccess;
}

} // namespace

cudaError_t launch_tc_combine(const TcCombineLaunch& a, cudaStream_t stream)
{
    CombineArgs k{};
    k.y = static_cast<const uint8_t*>(a.y);
    k.T = a.T;
    k.H = a.H;
    k.nvec = a.H / 8;
    k.num_y_rows = a.rows.num_rows;
    k.topk_idx = a.rows.topk_idx;
    k.slot = a.rows.slot;
    k.offsets = a.rows.offsets;
    k.K = a.rows.K;
    k.E = a.rows.E;
    k.mode = a.rows.mode;
    k.max_tokens = a.rows.max_tokens;
    k.topk_weights = a.topk_weights;
    k.out = a.out;
    k.err = a.err;
    return launch_combine<kSrcTopk, kTcVec, kTcGroup>(k, a.out_dtype == EP_FP32, EP_COMBINE_PERSIST_TC != 0, stream);
}

cudaError_t launch_ec_combine(const EcCombineLaunch& a, cudaStream_t stream)
{
    CombineArgs k{};
    k.y = static_cast<const uint8_t*>(a.y);
    k.T = a.T;
    k.H = a.H;
    k.nvec = a.H / 8;
    k.num_y_rows = a.num_y_rows;
    k.token_offsets = a.token_offsets;
    k.token_slots = a.token_slots;
    k.expert_weights = a.expert_weights;
    k.out = a.out;
    k.err = a.err;
    k.heavy_first = EP_COMBINE_HEAVY_FIRST && a.T <= kHeavyFirstMaxT ? 1 : 0;
    return launch_combine<kSrcEc, kEcVec, kEcGroup>(k, a.out_dtype == EP_FP32,
                                                    k.heavy_first != 0 || EP_COMBINE_PERSIST_EC != 0, stream);
}

cudaError_t launch_rank_combine(const RankCombineLaunch& a, cudaStream_t stream)
{
    CombineArgs k{};
    k.y = static_cast<const uint8_t*>(a.y);
    k.T = a.T;
    k.H = a.H;
    k.nvec = a.H / 8;
    k.num_y_rows = a.num_y_rows;
    k.K = a.R;
    k.rank_row = a.rank_row;
    k.out = a.out;
    k.err = a.err;
    return launch_combine<kSrcRanks, kTcVec, kTcGroup>(k, a.out_dtype == EP_FP32, EP_COMBINE_PERSIST_TC != 0, stream);
}

} // namespace ep
