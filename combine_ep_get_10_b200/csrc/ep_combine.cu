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
#include <atomic>
#include <type_traits>

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
// token choice: uniform items, so one resident wave of persistent warps
#ifndef EP_COMBINE_PERSIST_TC
#define EP_COMBINE_PERSIST_TC 1
#endif
#ifndef EP_COMBINE_HEAVY_FIRST
#define EP_COMBINE_HEAVY_FIRST 1
#endif
constexpr int kEcVec = EP_COMBINE_EC_VEC;
constexpr int kEcGroup = EP_COMBINE_EC_GROUP;
// expert choice, heavy tokens: narrower segments and longer groups keep more
// loads in flight on the long lists
#ifndef EP_COMBINE_HEAVY_VEC
#define EP_COMBINE_HEAVY_VEC 2
#endif
#ifndef EP_COMBINE_HEAVY_GROUP
#define EP_COMBINE_HEAVY_GROUP 8
#endif
#ifndef EP_COMBINE_EC_RUN
#define EP_COMBINE_EC_RUN 32
#endif
constexpr int kHeavyVec = EP_COMBINE_HEAVY_VEC;
constexpr int kHeavyGroup = EP_COMBINE_HEAVY_GROUP;
constexpr int kEcRun = EP_COMBINE_EC_RUN; // tokens per light item
static_assert(kEcRun >= 1 && kEcRun <= 32, "a light item's tokens are held one per lane");

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
    int32_t wide;        // rows and y 32-byte aligned: pairs of vectors by one 32-byte load
    PeerTables peers;    // per rank over peer memory: the ranks' y buffers
};

// expert choice, heavy first (see combine_kernel)
#ifndef EP_COMBINE_EC_HEAVY_DEG
#define EP_COMBINE_EC_HEAVY_DEG 16
#endif
constexpr int kHeavyDeg = EP_COMBINE_EC_HEAVY_DEG; // picks that make a token "heavy"
constexpr int kMaxHeavy = 2048;
constexpr int kHeavyFirstMaxT = 65536;
// heavy tokens listed by degree class, longest lists first (1: token order)
#ifndef EP_COMBINE_HEAVY_SORT
#define EP_COMBINE_HEAVY_SORT 1
#endif
constexpr int kHeavyClasses = EP_COMBINE_HEAVY_SORT ? 3 : 1;
// entries a heavy item looks up at once, in units of 32
#ifndef EP_COMBINE_HEAVY_LOOKUP
#define EP_COMBINE_HEAVY_LOOKUP 1
#endif
[[maybe_unused]] constexpr int kHeavyLookup = EP_COMBINE_HEAVY_LOOKUP; // used without EP_COMBINE_HEAVY_PIPE
// light runs: one list over the run's tokens (1) or one token at a time (0)
#ifndef EP_COMBINE_EC_FLAT
#define EP_COMBINE_EC_FLAT 1
#endif
#ifndef EP_COMBINE_EC_LOOKUP
#define EP_COMBINE_EC_LOOKUP 1
#endif
constexpr int kEcLookup = EP_COMBINE_EC_LOOKUP;
// resident CTAs per SM the expert-choice kernel is compiled for
#ifndef EP_COMBINE_EC_MINB
#define EP_COMBINE_EC_MINB 2
#endif
constexpr int kEcMinBlocks = EP_COMBINE_EC_MINB;
// expert choice: each group's weights (looked up from its slots, one more
// round trip) are taken from their lanes after the group's row loads are
// issued, not before (fp32 out 61.4 -> 60.4 us; bf16 unchanged)
#ifndef EP_COMBINE_EC_LATE_W
#define EP_COMBINE_EC_LATE_W 1
#endif
// per-rank combines: when a token's rank rows are spread over more groups
// than they fill, they are packed to the front (ascending rank kept) so that
// their loads go out in fewer rounds.  Measured on the skewed 16384-token
// batch (2.7 ranks per token): 153.6 -> 148.5 us; unchanged at 4096 tokens
// (5.3 ranks per token; packing every token measured 2 us slower there)
#ifndef EP_COMBINE_RANKS_COMPACT
#define EP_COMBINE_RANKS_COMPACT 1
#endif
// per-rank and peer combines: 16-byte vectors per lane and rows per load round
#ifndef EP_COMBINE_RANKS_VEC
#define EP_COMBINE_RANKS_VEC EP_COMBINE_VEC
#endif
#ifndef EP_COMBINE_RANKS_GROUP
#define EP_COMBINE_RANKS_GROUP EP_COMBINE_GROUP
#endif
constexpr int kRanksVec = EP_COMBINE_RANKS_VEC;
constexpr int kRanksGroup = EP_COMBINE_RANKS_GROUP;
// heavy items: lookups pipelined (reduce_heavy) or not (reduce_segment)
#ifndef EP_COMBINE_HEAVY_PIPE
#define EP_COMBINE_HEAVY_PIPE 1
#endif
// the longest lists (>= 4 kHeavyDeg picks, when listed by class) take
// narrower segments and longer groups: twice the warps, half the rounds
#ifndef EP_COMBINE_HEAVY0_VEC
#define EP_COMBINE_HEAVY0_VEC 1
#endif
#ifndef EP_COMBINE_HEAVY0_GROUP
#define EP_COMBINE_HEAVY0_GROUP 16
#endif
constexpr int kHeavy0Vec = EP_COMBINE_HEAVY0_VEC;
constexpr int kHeavy0Group = EP_COMBINE_HEAVY0_GROUP;
// 16-byte vectors of CSR bounds each thread loads per round of the heavy listing
constexpr int kHeavyVecs = 8;
// expert choice: the rows of unpicked tokens are written whole by TMA bulk
// stores from a zeroed shared buffer while the heavy tokens are listed (1),
// or by the light runs' vector stores (0)
#ifndef EP_COMBINE_EC_ZERO_BULK
#define EP_COMBINE_EC_ZERO_BULK 1
#endif
constexpr int kZeroBytes = 4096; // zeroed shared memory behind the bulk stores

enum CombineSrc : int {
    kSrcTopk = 0,  // entries: the token's K (expert, slot) pairs, gate weights
    kSrcEc = 1,    // entries: the token's CSR slots, expert weights
    kSrcRanks = 2, // entries: the token's R rank rows, weight 1 (fmaf(1, y, acc) == acc + y)
    kSrcPeers = 3  // entries: the token's rows in the R ranks' y buffers, weight 1; row = its address
};

template <int kSrc>
__device__ __forceinline__ void entry(const CombineArgs& a, int64_t t, int64_t beg, int j, int64_t& row, float& w,
                                      uint32_t& errbits)
{
    row = -1;
    w = 0.0f;
    if constexpr (kSrc == kSrcPeers) {
        // rank j's rows: those of ranks 0 .. me-1 first, then this rank's in send order
        const int64_t r = __ldg(a.rank_row + t * a.K + j);
        if (r < 0)
            return;
        const int32_t* counts = reinterpret_cast<const int32_t*>(__ldg(a.peers.rank_counts + a.peers.me));
        int64_t local = r - __ldg(a.peers.rank_offsets + j);
        for (int i = 0; i < a.peers.me; ++i)
            local += __ldg(counts + i * a.K + j);
        if (local < 0 || local >= a.num_y_rows) {
            errbits |= EP_DEVERR_OVERFLOW;
            return;
        }
        row = static_cast<int64_t>(__ldg(a.peers.y + j)) + local * (static_cast<int64_t>(a.H) * 2);
        w = 1.0f;
    } else if constexpr (kSrc == kSrcRanks) {
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

// out[t, segment seg] = sum over the token's n entries (ascending) of
// w * y[row], one warp.  A segment is kVecPerLane 16-byte vectors per lane;
// entries are looked up kLookup * 32 at a time (all of their loads in
// flight), broadcast by shuffles and folded kGroup at a time, every 16-byte
// load of a group issued before its FMAs.
template <int kSrc, bool kOutF32, int kVecPerLane, int kGroup, int kLookup>
__device__ __forceinline__ void reduce_segment(const CombineArgs& a, int64_t t, int seg, int64_t beg, int n, int lane,
                                               uint32_t& errbits)
{
    constexpr int kSegVec = 32 * kVecPerLane;
    const bool wide = kVecPerLane % 2 == 0 && a.wide != 0;
    int v[kVecPerLane];
    bool vin[kVecPerLane];
#pragma unroll
    for (int j = 0; j < kVecPerLane; ++j) {
        // 32-byte loads: lane covers vectors 2 lane, 2 lane + 1 of each 64-vector run
        v[j] = wide ? seg * kSegVec + (j >> 1) * 64 + 2 * lane + (j & 1) : seg * kSegVec + j * 32 + lane;
        vin[j] = v[j] < a.nvec;
    }
    float acc[kVecPerLane][8];
#pragma unroll
    for (int j = 0; j < kVecPerLane; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[j][i] = 0.0f;

    // expert-choice rows are slot ids below E*C < 2^31: 32-bit row registers
    using RowT = typename std::conditional<kSrc == kSrcEc, int32_t, int64_t>::type;
    const int64_t row_bytes = static_cast<int64_t>(a.H) * 2;
    for (int k0 = 0; k0 < n; k0 += 32 * kLookup) {
        RowT my_row[kLookup];
        float my_w[kLookup];
#pragma unroll
        for (int i = 0; i < kLookup; ++i) {
            my_row[i] = -1;
            my_w[i] = 0.0f;
            const int j = k0 + 32 * i + lane;
            if (j < n) {
                int64_t r = -1;
                entry<kSrc>(a, t, beg, j, r, my_w[i], errbits);
                my_row[i] = static_cast<RowT>(r);
            }
        }
        int m_valid = 32;
#if EP_COMBINE_RANKS_COMPACT
        if constexpr ((kSrc == kSrcRanks || kSrc == kSrcPeers) && kLookup == 1 && kGroup == 4) {
            // the token's ranks first, in ascending order: its loads then fill
            // the first group instead of spreading over all of them (group
            // occupancy counted by nibbles)
            const uint32_t valid = __ballot_sync(kFullMask, my_row[0] >= 0);
            const int cnt = __popc(valid);
            // groups (aligned nibbles) holding at least one of the token's ranks
            const int touched = __popc((valid | (valid >> 1) | (valid >> 2) | (valid >> 3)) & 0x11111111u);
            if ((cnt + kGroup - 1) / kGroup < touched) { // packing saves a round of loads
                m_valid = cnt;
                const int src = lane < cnt ? static_cast<int>(__fns(valid, 0, lane + 1)) : lane;
                const RowT r = __shfl_sync(kFullMask, my_row[0], src);
                const float wv = __shfl_sync(kFullMask, my_w[0], src);
                my_row[0] = lane < cnt ? r : -1;
                my_w[0] = lane < cnt ? wv : 0.0f;
            }
        }
#endif
#pragma unroll
        for (int i = 0; i < kLookup; ++i) {
            const int kb = k0 + 32 * i;
            if (kb >= n)
                break; // warp-uniform
            const int m = min(m_valid, n - kb);
            for (int g0 = 0; g0 < m; g0 += kGroup) {
                RowT rows[kGroup];
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
                for (int g = 0; g < kGroup; ++g) {
                    const bool on = rows[g] >= 0;
                    const uint8_t* src = kSrc == kSrcPeers
                                             ? reinterpret_cast<const uint8_t*>(static_cast<uintptr_t>(rows[g]))
                                             : a.y + static_cast<int64_t>(on ? rows[g] : 0) * row_bytes;
                    if (wide) {
#pragma unroll
                        for (int j = 0; j < kVecPerLane; j += 2) {
                            if (on && vin[j])
                                ld_nc_v8(src + static_cast<int64_t>(v[j]) * 16, d[g][j], d[g][j + 1]);
                            else
                                d[g][j] = d[g][j + 1] = make_uint4(0, 0, 0, 0);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < kVecPerLane; ++j)
                            d[g][j] = (on && vin[j]) ? ld_nc_v4(src + static_cast<int64_t>(v[j]) * 16) : make_uint4(0, 0, 0, 0);
                    }
                }
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

// out[t, segment] <- acc (kVecPerLane 16-byte vectors per lane, as in
// reduce_segment)
template <bool kOutF32, int kVecPerLane>
__device__ __forceinline__ void store_segment(const CombineArgs& a, int64_t t, const int (&v)[kVecPerLane],
                                              const bool (&vin)[kVecPerLane], const float (&acc)[kVecPerLane][8])
{
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
            uint8_t* o = static_cast<uint8_t*>(a.out) + t * static_cast<int64_t>(a.H) * 2 + static_cast<int64_t>(v[j]) * 16;
            st_cs_v4(o, make_uint4(pack_bf16x2(acc[j][0], acc[j][1]), pack_bf16x2(acc[j][2], acc[j][3]),
                                   pack_bf16x2(acc[j][4], acc[j][5]), pack_bf16x2(acc[j][6], acc[j][7])));
        }
    }
}

// Expert choice, a run of light tokens t0 .. t0 + cnt - 1 (cnt <= 32, lane j
// holds token j's CSR bounds), one segment.  The entries of the run's tokens
// (skipping heavy ones when skip_heavy) make one list in token order, each
// token's CSR slots in order.  Lanes look the list up kLookup * 32 entries at
// a time; the warp folds it kGroup entries at a time with every load of a
// group issued together, also when the group spans tokens, so a run costs
// one load round per kGroup entries instead of one per token.  A token's
// accumulators start from zero at its first entry and are stored after its
// last: each token's sum is the fmaf chain over its own entries in ascending
// CSR order, as in reduce_segment.  Tokens without entries store zeros.
template <bool kOutF32, int kVecPerLane, int kGroup, int kLookup>
__device__ __forceinline__ void reduce_run(const CombineArgs& a, int64_t t0, int cnt, int seg, bool skip_heavy,
                                           bool zeros_written, int lane, uint32_t& errbits)
{
    constexpr int kSegVec = 32 * kVecPerLane;
    const bool wide = kVecPerLane % 2 == 0 && a.wide != 0;
    int v[kVecPerLane];
    bool vin[kVecPerLane];
#pragma unroll
    for (int j = 0; j < kVecPerLane; ++j) {
        // 32-byte loads: lane covers vectors 2 lane, 2 lane + 1 of each 64-vector run
        v[j] = wide ? seg * kSegVec + (j >> 1) * 64 + 2 * lane + (j & 1) : seg * kSegVec + j * 32 + lane;
        vin[j] = v[j] < a.nvec;
    }
    float acc[kVecPerLane][8];
#pragma unroll
    for (int j = 0; j < kVecPerLane; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[j][i] = 0.0f;

    int my_beg = 0, my_n = 0;
    if (lane < cnt) {
        my_beg = __ldg(a.token_offsets + t0 + lane);
        my_n = __ldg(a.token_offsets + t0 + lane + 1) - my_beg;
    }
    const bool mine = lane < cnt && !(skip_heavy && my_n >= kHeavyDeg);
    const int my_cnt = mine ? max(my_n, 0) : 0;
    uint32_t zeros = zeros_written ? 0u : __ballot_sync(kFullMask, mine && my_cnt == 0);
    while (zeros) { // warp-uniform
        const int j = __ffs(zeros) - 1;
        zeros &= zeros - 1u;
        store_segment<kOutF32, kVecPerLane>(a, t0 + j, v, vin, acc);
    }
    int incl = my_cnt; // list positions up to and including this lane's token
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(kFullMask, incl, d);
        if (lane >= d)
            incl += o;
    }
    const int total = __shfl_sync(kFullMask, incl, 31);
    const int my_start = incl - my_cnt;

    int cur = -1; // lane (token) whose sum is open
    for (int c0 = 0; c0 < total; c0 += 32 * kLookup) {
        int32_t my_row[kLookup];
        float my_w[kLookup];
        int my_tok[kLookup];
        uint32_t first[kLookup]; // bit g: list position 32 * i + g opens a token
#pragma unroll
        for (int i = 0; i < kLookup; ++i) {
            const int e = c0 + 32 * i + lane;
            // owner of list position e: the number of lanes whose entries end
            // at or before e (incl is non-decreasing over the lanes)
            int j = 0;
#pragma unroll
            for (int step = 16; step >= 1; step >>= 1) {
                const int end = __shfl_sync(kFullMask, incl, j + step - 1);
                if (end <= e)
                    j += step;
            }
            const int jbeg = __shfl_sync(kFullMask, my_beg, j);
            const int jstart = __shfl_sync(kFullMask, my_start, j);
            my_tok[i] = j;
            first[i] = __ballot_sync(kFullMask, e < total && e == jstart);
            my_row[i] = -1;
            my_w[i] = 0.0f;
            if (e < total) {
                const int32_t s = __ldg(a.token_slots + jbeg + (e - jstart));
                if (s < 0 || s >= a.num_y_rows) {
                    errbits |= EP_DEVERR_OVERFLOW;
                } else {
                    my_row[i] = s;
                    my_w[i] = __ldg(a.expert_weights + s);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kLookup; ++i) {
            const int kb = c0 + 32 * i;
            if (kb >= total)
                break; // warp-uniform
            const int m = min(32, total - kb);
            for (int g0 = 0; g0 < m; g0 += kGroup) {
                int32_t rows[kGroup];
                float ws[kGroup];
#pragma unroll
                for (int g = 0; g < kGroup; ++g) {
                    const int src = (g0 + g) & 31;
                    rows[g] = __shfl_sync(kFullMask, my_row[i], src);
                    if (!EP_COMBINE_EC_LATE_W)
                        ws[g] = __shfl_sync(kFullMask, my_w[i], src);
                    if (g0 + g >= m)
                        rows[g] = -1;
                }
                uint4 d[kGroup][kVecPerLane];
#pragma unroll
                for (int g = 0; g < kGroup; ++g) {
                    const bool on = rows[g] >= 0;
                    const uint8_t* src = a.y + static_cast<int64_t>(on ? rows[g] : 0) * (static_cast<int64_t>(a.H) * 2);
                    if (wide) {
#pragma unroll
                        for (int j = 0; j < kVecPerLane; j += 2) {
                            if (on && vin[j])
                                ld_nc_v8(src + static_cast<int64_t>(v[j]) * 16, d[g][j], d[g][j + 1]);
                            else
                                d[g][j] = d[g][j + 1] = make_uint4(0, 0, 0, 0);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < kVecPerLane; ++j)
                            d[g][j] = (on && vin[j]) ? ld_nc_v4(src + static_cast<int64_t>(v[j]) * 16) : make_uint4(0, 0, 0, 0);
                    }
                }
                if (EP_COMBINE_EC_LATE_W) { // the weights' lookups finish under the row loads
#pragma unroll
                    for (int g = 0; g < kGroup; ++g)
                        ws[g] = __shfl_sync(kFullMask, my_w[i], (g0 + g) & 31);
                }
#pragma unroll
                for (int g = 0; g < kGroup; ++g) {
                    if (g0 + g >= m)
                        break; // warp-uniform
                    if ((first[i] >> ((g0 + g) & 31)) & 1u) { // warp-uniform: a token opens, the open one ended
                        if (cur >= 0)
                            store_segment<kOutF32, kVecPerLane>(a, t0 + cur, v, vin, acc);
#pragma unroll
                        for (int j = 0; j < kVecPerLane; ++j)
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                acc[j][q] = 0.0f;
                        cur = __shfl_sync(kFullMask, my_tok[i], (g0 + g) & 31);
                    }
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
    if (cur >= 0)
        store_segment<kOutF32, kVecPerLane>(a, t0 + cur, v, vin, acc);
}

// Expert choice, one heavy token's segment: the same fmaf chain as
// reduce_segment (entries in ascending CSR order, from zero), with the
// entry lookups taken off the chain: the slots of the next 32 entries are in
// flight while the current 32 are folded, and their weights are fetched
// while the first group of the current 32 is in flight, so a long list costs
// one load round per kGroup entries plus two at the start.
template <bool kOutF32, int kVecPerLane, int kGroup>
__device__ __forceinline__ void reduce_heavy(const CombineArgs& a, int64_t t, int seg, int beg, int n, int lane,
                                             uint32_t& errbits)
{
    constexpr int kSegVec = 32 * kVecPerLane;
    static_assert(32 % kGroup == 0, "a group never straddles two lookups");
    const bool wide = kVecPerLane % 2 == 0 && a.wide != 0;
    int v[kVecPerLane];
    bool vin[kVecPerLane];
#pragma unroll
    for (int j = 0; j < kVecPerLane; ++j) {
        // 32-byte loads: lane covers vectors 2 lane, 2 lane + 1 of each 64-vector run
        v[j] = wide ? seg * kSegVec + (j >> 1) * 64 + 2 * lane + (j & 1) : seg * kSegVec + j * 32 + lane;
        vin[j] = v[j] < a.nvec;
    }
    float acc[kVecPerLane][8];
#pragma unroll
    for (int j = 0; j < kVecPerLane; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[j][i] = 0.0f;

    const int64_t row_bytes = static_cast<int64_t>(a.H) * 2;
    // slot of entry j (-1 past the list); a slot outside y is flagged and skipped
    auto slot_at = [&](int j) -> int32_t { return j < n ? __ldg(a.token_slots + beg + j) : -1; };
    auto valid = [&](int j, int32_t s) -> bool {
        if (j >= n)
            return false;
        if (s < 0 || s >= a.num_y_rows) {
            errbits |= EP_DEVERR_OVERFLOW;
            return false;
        }
        return true;
    };
    int32_t s_cur = slot_at(lane);
    int32_t s_nxt = slot_at(32 + lane);
    int32_t r_cur = valid(lane, s_cur) ? s_cur : -1;
    float w_cur = r_cur >= 0 ? __ldg(a.expert_weights + r_cur) : 0.0f;
    for (int k0 = 0; k0 < n; k0 += 32) {
        const int m = min(32, n - k0);
        int32_t r_nxt = -1, s_after = -1;
        float w_nxt = 0.0f;
        for (int g0 = 0; g0 < m; g0 += kGroup) {
            int32_t rows[kGroup];
            float ws[kGroup];
#pragma unroll
            for (int g = 0; g < kGroup; ++g) {
                rows[g] = __shfl_sync(kFullMask, r_cur, g0 + g);
                if (!EP_COMBINE_EC_LATE_W)
                    ws[g] = __shfl_sync(kFullMask, w_cur, g0 + g);
                if (g0 + g >= m)
                    rows[g] = -1;
            }
            uint4 d[kGroup][kVecPerLane];
#pragma unroll
            for (int g = 0; g < kGroup; ++g) {
                const bool on = rows[g] >= 0;
                const uint8_t* src = a.y + static_cast<int64_t>(on ? rows[g] : 0) * row_bytes;
                if (wide) {
#pragma unroll
                    for (int j = 0; j < kVecPerLane; j += 2) {
                        if (on && vin[j])
                            ld_nc_v8(src + static_cast<int64_t>(v[j]) * 16, d[g][j], d[g][j + 1]);
                        else
                            d[g][j] = d[g][j + 1] = make_uint4(0, 0, 0, 0);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < kVecPerLane; ++j)
                        d[g][j] = (on && vin[j]) ? ld_nc_v4(src + static_cast<int64_t>(v[j]) * 16) : make_uint4(0, 0, 0, 0);
                }
            }
            if (g0 == 0) { // the next 32 entries' weights, and the slots of the 32 after them
                r_nxt = valid(k0 + 32 + lane, s_nxt) ? s_nxt : -1;
                w_nxt = r_nxt >= 0 ? __ldg(a.expert_weights + r_nxt) : 0.0f;
                s_after = slot_at(k0 + 64 + lane);
            }
            if (EP_COMBINE_EC_LATE_W) { // the weights' lookups finish under the row loads
#pragma unroll
                for (int g = 0; g < kGroup; ++g)
                    ws[g] = __shfl_sync(kFullMask, w_cur, g0 + g);
            }
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
        r_cur = r_nxt;
        w_cur = w_nxt;
        s_nxt = s_after;
    }
    store_segment<kOutF32, kVecPerLane>(a, t, v, vin, acc);
}

// Token choice and per-rank rows: one warp per (token, segment) item; the
// items are taken with a fixed stride by a persistent grid (uniform cost).
template <int kSrc, bool kOutF32, int kVecPerLane, int kGroup>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineArgs a)
{
    pdl_wait(); // every input is final once the kernel before has finished
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kWarpsPerCta;
    uint32_t errbits = 0;
    const int64_t items = static_cast<int64_t>(a.T) * a.nseg;
    for (int64_t gw = a.warp_base + static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + warp; gw < items;
         gw += stride) {
        const int64_t t = gw / a.nseg;
        const int seg = static_cast<int>(gw - t * a.nseg);
        reduce_segment<kSrc, kOutF32, kVecPerLane, kGroup, 1>(a, t, seg, 0, a.K, lane, errbits);
    }
    const uint32_t any = __reduce_or_sync(kFullMask, errbits);
    if (lane == 0)
        flag_error(a.err, any);
}

// Expert choice.  A few tokens are picked by up to all E experts and most by
// none, so the work per token varies by 100x.  Every CTA first lists the
// tokens with at least kHeavyDeg picks (the same list in every CTA, which
// the items below rely on): by degree class, longest first (>= 4x, >= 2x,
// >= 1x kHeavyDeg), in token order inside a class.  The items are then: one per (heavy token, segment),
// followed by one per (run of kEcRun tokens, segment); a run item folds its
// light tokens' entries as one list (reduce_run) and leaves the heavy tokens
// to the heavy items.  The items, in that order (roughly longest first), are
// dealt to the CTAs one round of gridDim items at a time in a serpentine (CTA
// c takes item c of an even round and item gridDim - 1 - c of an odd one), so
// every CTA holds a like mix of long and short work; a CTA's warps take its
// rounds in order from a shared-memory ticket, so a warp that finishes early
// takes the next item instead of the tail waiting on fixed shares.
template <bool kOutF32>
__global__ void __launch_bounds__(kCombineThreads, kEcMinBlocks) ec_combine_kernel(CombineArgs a)
{
    pdl_wait(); // every input is final once the kernel before has finished
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    uint32_t errbits = 0;

    __shared__ int s_heavy[kMaxHeavy];
    __shared__ uint32_t s_flags[kHeavyClasses][kHeavyFirstMaxT / 32];
    __shared__ int s_wsum[kWarpsPerCta];
    __shared__ int s_ticket; // this CTA's next round of items
    __shared__ __align__(128) uint8_t s_zero[EP_COMBINE_EC_ZERO_BULK ? kZeroBytes : 16];
    if (threadIdx.x == 0)
        s_ticket = 0;
    __syncthreads();
    int n_heavy = 0, n_long = 0;
    if (a.heavy_first) {
        // Every CTA reads the whole CSR bound array once, coalesced and all at
        // once (16-byte vectors, kHeavyVecs per thread, plus the bound after
        // each vector), flags the heavy tokens in one shared bit mask per
        // degree class, then lists them class by class (count per 32-token
        // word, CTA scan).
        const int tid = threadIdx.x;
        const int nwords = (a.T + 31) / 32;
        for (int i = tid; i < nwords; i += kCombineThreads)
#pragma unroll
            for (int c = 0; c < kHeavyClasses; ++c)
                s_flags[c][i] = 0u;
        if (EP_COMBINE_EC_ZERO_BULK) {
            for (int i = tid; i < kZeroBytes / 16; i += kCombineThreads)
                reinterpret_cast<uint4*>(s_zero)[i] = make_uint4(0, 0, 0, 0);
            fence_proxy_async_shared(); // the bulk stores below read it
        }
        __syncthreads();
        // this CTA also writes the whole output rows of the unpicked tokens in
        // [z0, z1), by bulk stores from the zeroed buffer
        const int64_t z0 = static_cast<int64_t>(a.T) * blockIdx.x / gridDim.x;
        const int64_t z1 = static_cast<int64_t>(a.T) * (blockIdx.x + 1) / gridDim.x;
        const int64_t out_row = static_cast<int64_t>(a.H) * (kOutF32 ? 4 : 2);
        bool issued = false;
        // 4 bounds per 16-byte vector (1 when the array is not 16-byte aligned),
        // kHeavyVecs vectors per thread per round, all loads of a round at once
        const int per = (reinterpret_cast<uintptr_t>(a.token_offsets) & 15u) == 0 ? 4 : 1;
        const int nv = (a.T + per - 1) / per; // vectors holding bounds 0 .. T-1
        for (int base = 0; base < nv; base += kHeavyVecs * kCombineThreads) {
            int4 q[kHeavyVecs];
            int nxt[kHeavyVecs];
#pragma unroll
            for (int k = 0; k < kHeavyVecs; ++k) {
                const int v = base + k * kCombineThreads + tid;
                q[k] = make_int4(0, 0, 0, 0);
                nxt[k] = 0;
                if (v < nv) {
                    const int b = per * v;
                    if (per == 4 && b + 3 <= a.T) {
                        q[k] = __ldg(reinterpret_cast<const int4*>(a.token_offsets) + v);
                    } else { // the array's last bounds: no read past index T
                        q[k].x = __ldg(a.token_offsets + b);
                        if (per == 4) {
                            q[k].y = b + 1 <= a.T ? __ldg(a.token_offsets + b + 1) : 0;
                            q[k].z = b + 2 <= a.T ? __ldg(a.token_offsets + b + 2) : 0;
                        }
                    }
                    nxt[k] = __ldg(a.token_offsets + min(b + per, a.T));
                }
            }
#pragma unroll
            for (int k = 0; k < kHeavyVecs; ++k) {
                const int v = base + k * kCombineThreads + tid;
                if (v >= nv)
                    continue;
                const int o[5] = {q[k].x, q[k].y, q[k].z, q[k].w, nxt[k]};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int t = per * v + j;
                    const int deg = (j + 1 < per ? o[j + 1] : o[4]) - o[j];
                    if (j < per && t < a.T && deg >= kHeavyDeg) {
                        const int c = kHeavyClasses == 1 ? 0 : deg >= 4 * kHeavyDeg ? 0 : deg >= 2 * kHeavyDeg ? 1 : 2;
                        atomicOr(&s_flags[c][t / 32], 1u << (t % 32));
                    }
                    if (EP_COMBINE_EC_ZERO_BULK && j < per && t >= z0 && t < z1 && deg == 0) {
                        uint8_t* row = static_cast<uint8_t*>(a.out) + t * out_row;
                        for (int64_t b0 = 0; b0 < out_row; b0 += kZeroBytes)
                            bulk_store_s2g(row + b0, s_zero,
                                           static_cast<uint32_t>(min(static_cast<int64_t>(kZeroBytes), out_row - b0)));
                        issued = true;
                    }
                }
            }
        }
        if (issued)
            bulk_commit();
        __syncthreads();
        // words w0 .. w1 of this thread, scanned over the CTA, class by class
        const int wpt = (nwords + kCombineThreads - 1) / kCombineThreads;
        const int w0 = min(nwords, tid * wpt);
        const int w1 = min(nwords, w0 + wpt);
        int listed = 0;
#pragma unroll 1
        for (int c = 0; c < kHeavyClasses; ++c) {
            if (c == 1)
                n_long = listed; // class 0: the longest lists
            int cnt = 0;
            for (int w = w0; w < w1; ++w)
                cnt += __popc(s_flags[c][w]);
            int inc = cnt;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int v = __shfl_up_sync(kFullMask, inc, d);
                if (lane >= d)
                    inc += v;
            }
            if (lane == 31)
                s_wsum[warp] = inc;
            __syncthreads();
            int before = 0, n_c = 0;
            for (int w = 0; w < kWarpsPerCta; ++w) {
                before += w < warp ? s_wsum[w] : 0;
                n_c += s_wsum[w];
            }
            if (listed + n_c <= kMaxHeavy) {
                int pos = listed + before + inc - cnt;
                for (int w = w0; w < w1; ++w) {
                    uint32_t bits = s_flags[c][w];
                    while (bits) {
                        const int i = __ffs(bits) - 1;
                        bits &= bits - 1u;
                        s_heavy[pos++] = w * 32 + i;
                    }
                }
            }
            listed += n_c;
            __syncthreads(); // s_wsum is reused by the next class
        }
        n_heavy = listed <= kMaxHeavy ? listed : 0; // too many to list: every token goes through the runs
        if (n_heavy == 0 || kHeavyClasses == 1)
            n_long = 0;
    }
    const int nseg_h = (a.nvec + 32 * kHeavyVec - 1) / (32 * kHeavyVec);
    const int nseg_l = (a.nvec + 32 * kHeavy0Vec - 1) / (32 * kHeavy0Vec);
    const int64_t long_items = static_cast<int64_t>(n_long) * nseg_l;
    const int64_t heavy_items = long_items + static_cast<int64_t>(n_heavy - n_long) * nseg_h;
    const int64_t runs = (static_cast<int64_t>(a.T) + kEcRun - 1) / kEcRun;
    const int64_t items = heavy_items + runs * a.nseg;
    // this CTA's round k holds item k * G + c (k even) or k * G + G - 1 - c (k odd)
    const int64_t G = gridDim.x;
    auto take = [&]() -> int {
        int k = 0;
        if (lane == 0)
            k = atomicAdd(&s_ticket, 1);
        return __shfl_sync(kFullMask, k, 0);
    };
    for (int k = take();; k = take()) {
        const int64_t it = static_cast<int64_t>(k) * G + ((k & 1) ? G - 1 - blockIdx.x : blockIdx.x);
        if (it >= items)
            break; // every later round of this CTA lies past the end too
        if (it < heavy_items) {
            const bool is_long = it < long_items;
            const int64_t h = is_long ? it : it - long_items;
            const int ns = is_long ? nseg_l : nseg_h;
            const int64_t t = s_heavy[(is_long ? 0 : n_long) + h / ns];
            const int seg = static_cast<int>(h % ns);
            const int beg = __ldg(a.token_offsets + t);
            const int n = __ldg(a.token_offsets + t + 1) - beg;
#if EP_COMBINE_HEAVY_PIPE
            if (is_long)
                reduce_heavy<kOutF32, kHeavy0Vec, kHeavy0Group>(a, t, seg, beg, n, lane, errbits);
            else
                reduce_heavy<kOutF32, kHeavyVec, kHeavyGroup>(a, t, seg, beg, n, lane, errbits);
#else
            if (is_long)
                reduce_segment<kSrcEc, kOutF32, kHeavy0Vec, kHeavy0Group, kHeavyLookup>(a, t, seg, beg, n, lane,
                                                                                       errbits);
            else
                reduce_segment<kSrcEc, kOutF32, kHeavyVec, kHeavyGroup, kHeavyLookup>(a, t, seg, beg, n, lane, errbits);
#endif
            continue;
        }
        const int64_t l = it - heavy_items; // a light item
        const int64_t r = l / a.nseg;
        const int seg = static_cast<int>(l - r * a.nseg);
        const int64_t t0 = r * kEcRun;
        const int cnt = static_cast<int>(min(static_cast<int64_t>(kEcRun), a.T - t0));
#if EP_COMBINE_EC_FLAT
        reduce_run<kOutF32, kEcVec, kEcGroup, kEcLookup>(a, t0, cnt, seg, n_heavy > 0,
                                                         EP_COMBINE_EC_ZERO_BULK && a.heavy_first, lane, errbits);
#else
        // lane j holds the CSR bounds of the run's j-th token; one token at a time
        int my_beg = 0, my_n = 0;
        if (lane < cnt) {
            my_beg = __ldg(a.token_offsets + t0 + lane);
            my_n = __ldg(a.token_offsets + t0 + lane + 1) - my_beg;
        }
        for (int j = 0; j < cnt; ++j) {
            const int n = __shfl_sync(kFullMask, my_n, j);
            const int beg = __shfl_sync(kFullMask, my_beg, j);
            if (n_heavy > 0 && n >= kHeavyDeg)
                continue; // done as a heavy item
            reduce_segment<kSrcEc, kOutF32, kEcVec, kEcGroup, 2>(a, t0 + j, seg, beg, n, lane, errbits);
        }
#endif
    }
    const uint32_t any = __reduce_or_sync(kFullMask, errbits);
    if (lane == 0)
        flag_error(a.err, any);
    if (EP_COMBINE_EC_ZERO_BULK)
        bulk_wait_read_all(); // the zero rows' bulk stores have read s_zero
}

// Combine kernels are launched with programmatic stream serialisation: their
// CTAs may be placed while the kernel before them (normally the dispatch)
// retires its last CTAs, and wait in griddepcontrol.wait before any read, so
// only the launch latency is hidden.
#ifndef EP_COMBINE_PDL
#define EP_COMBINE_PDL 1
#endif

template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kernel)(KArgs...), unsigned grid, cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kCombineThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = EP_COMBINE_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Blocks of 256 threads of `kernel` resident on the whole device (SMs x
// blocks per SM), cached per device in `cache` (host threads may race to
// fill an entry; they store the same value).
template <typename Kernel>
int64_t resident_blocks(Kernel kernel, std::atomic<int>* cache)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 0;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kCombineThreads, 0) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        n = sms * std::max(per_sm, 1);
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
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
        static std::atomic<int> cache_bf16[64], cache_f32[64];
        const int64_t res = out_f32 ? resident_blocks(combine_kernel<kSrc, true, kVec, kGrp>, cache_f32)
                                    : resident_blocks(combine_kernel<kSrc, false, kVec, kGrp>, cache_bf16);
        if (res > 0)
            blocks = std::min(blocks, res);
    }
    for (int64_t b0 = 0; b0 < blocks; b0 += kMaxBlocks) {
        k.warp_base = b0 * kWarpsPerCta;
        const unsigned n = static_cast<unsigned>(blocks - b0 < kMaxBlocks ? blocks - b0 : kMaxBlocks);
        cudaError_t st = out_f32 ? launch_after(combine_kernel<kSrc, true, kVec, kGrp>, n, stream, k)
                                 : launch_after(combine_kernel<kSrc, false, kVec, kGrp>, n, stream, k);
        if (st != cudaSuccess)
            return st;
    }
    return cudaSuccess;
}

// Expert choice: one resident wave of warps over the heavy and run items.
cudaError_t launch_ec(CombineArgs k, bool out_f32, cudaStream_t stream)
{
    k.nseg = (k.nvec + 32 * kEcVec - 1) / (32 * kEcVec);
    const int64_t runs = (static_cast<int64_t>(k.T) + kEcRun - 1) / kEcRun;
    const int64_t items = std::max<int64_t>(1, runs * k.nseg);
    static std::atomic<int> cache_bf16[64], cache_f32[64];
    const int64_t res = out_f32 ? resident_blocks(ec_combine_kernel<true>, cache_f32)
                                : resident_blocks(ec_combine_kernel<false>, cache_bf16);
    int64_t blocks = res > 0 ? res : (items + kWarpsPerCta - 1) / kWarpsPerCta;
    blocks = std::min<int64_t>(blocks, int64_t{1} << 30);
    k.warp_base = 0;
    return out_f32 ? launch_after(ec_combine_kernel<true>, static_cast<unsigned>(blocks), stream, k)
                   : launch_after(ec_combine_kernel<false>, static_cast<unsigned>(blocks), stream, k);
}

// Pairs of 16-byte vectors by one 32-byte load (sm_100's 256-bit loads) in
// the token-choice and per-rank combines from this many tokens on: measured
// faster at 16384 tokens (skewed workload 305 -> 293 us) and slower at 4096
// (91 -> 99 us); the expert-choice combine measured no gain and keeps 16-byte
// loads.  32-byte loads need y aligned to 32 and rows a multiple of 32 bytes.
#ifndef EP_COMBINE_WIDE_MIN_TOKENS
#define EP_COMBINE_WIDE_MIN_TOKENS 8192
#endif
int32_t wide_loads(const void* y, int32_t H, int32_t T)
{
    return T >= EP_COMBINE_WIDE_MIN_TOKENS && H % 16 == 0 && (reinterpret_cast<uintptr_t>(y) & 31u) == 0 ? 1 : 0;
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
    k.wide = wide_loads(a.y, a.H, a.T);
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
    k.wide = 0;
    if (a.T == 0)
        return cudaSuccess;
    return launch_ec(k, a.out_dtype == EP_FP32, stream);
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
    if (a.peers.y != nullptr) {
        // the ranks' buffers: 16-byte loads (their alignment to 32 is not known here)
        k.peers = a.peers;
        k.num_y_rows = a.peers.capacity;
        k.wide = 0;
        return launch_combine<kSrcPeers, kRanksVec, kRanksGroup>(k, a.out_dtype == EP_FP32,
                                                                  EP_COMBINE_PERSIST_TC != 0, stream);
    }
    k.wide = wide_loads(a.y, a.H, a.T);
    return launch_combine<kSrcRanks, kRanksVec, kRanksGroup>(k, a.out_dtype == EP_FP32, EP_COMBINE_PERSIST_TC != 0,
                                                              stream);
}

} // namespace ep
