// ep_dispatch.cu -- dispatch kernels.
//
// bf16 dispatch (token choice: DeepEP-Ascend README, API Overview,
// dispatch / low_latency_dispatch, per expert or deduplicated per rank;
// expert choice: DeepEP issue #595, Solution 1) is a pure row copy: each
// source row chunk (a whole row up to 16 KB) is read from HBM exactly once by
// the TMA engine (cp.async.bulk global->shared, completion on an mbarrier)
// and written to every destination row by bulk stores (cp.async.bulk
// shared->global), one per destination, issued by different lanes.  A CTA is
// one warp and moves one (row, chunk) item; up to 14 CTAs of 16 KB per SM
// keep ~200 KB of copies in flight per SM and the block scheduler balances
// the tail.  (8 KB chunks measured 2% slower on 14 KB rows; a persistent
// variant streaming each CTA's items through a 3-4 stage ring 10-15% slower.)
//
// Quantised dispatch (README, "Quantization Modes in Normal Dispatch": FP8
// with one fp32 scale per 128 channels, per-token INT8 and FP8, MX FP8/FP4
// with an e8m0 scale per 32): one CTA per token stages the row in shared memory
// (all loads issued at once), reduces the amax over each scale group by
// shuffles (or over the CTA for per-token scales), encodes every element once
// with the cvt.rn.satfinite packing instructions, and stores the code runs
// and scales to each destination row of the token.
#include <algorithm>

#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

#ifndef EP_DISPATCH_CHUNK
#define EP_DISPATCH_CHUNK 16384
#endif

constexpr int64_t kChunkTarget = EP_DISPATCH_CHUNK; // bytes per bulk-copy item

#ifndef EP_QUANT_BULK_SCALES
#define EP_QUANT_BULK_SCALES 0
#endif

// Dispatch kernels are launched with programmatic stream serialisation.  By
// default a dispatch waits for the kernel before it (griddepcontrol.wait)
// before it reads anything: that kernel may have written x or the routing,
// and its writes are only guaranteed visible after the wait.  When the
// library itself has just launched the layout on the stream
// (ep_layout_dispatch: the kernel before is that layout, which lets its
// dependents start at once and writes neither x nor the routing), the
// dispatch's CTAs start while the layout runs, load their source rows, and
// wait only before reading the layout's results (early_load).  The
// expert-choice copy reads no layout result at all
// (ep_layout_dispatch_expert_choice): its CTAs run under the whole layout
// and only the grid's last CTA waits, before it ends, so that the grid never
// completes before the layout does (a kernel launched after it in the same
// way then sees the layout's CSR) while the other CTAs leave at once.
#ifndef EP_DISPATCH_PDL
#define EP_DISPATCH_PDL 1
#endif

// <<<grid, block, smem, stream>>> with programmatic stream serialisation.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = EP_DISPATCH_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

struct RowMap {
    const int64_t* topk_idx;
    const int32_t* slot;
    const int32_t* offsets;
    int32_t K, E, mode, max_tokens;
    int64_t num_rows;

    // Destination row of pair (t,k), or -1 (not routed / no room).
    __device__ __forceinline__ int64_t row(int64_t t, int k, uint32_t& errbits) const
    {
        const int64_t e = __ldg(topk_idx + t * K + k);
        const int32_t s = ld_meta(slot + t * K + k);
        if (e < 0 || e >= E || s < 0) {
            if (e < -1 || e >= E)
                errbits |= EP_DEVERR_BAD_INDEX;
            return -1;
        }
        int64_t r;
        if (mode == EP_LAYOUT_PADDED) {
            if (s >= max_tokens) {
                errbits |= EP_DEVERR_OVERFLOW;
                return -1;
            }
            r = e * max_tokens + s;
        } else {
            r = static_cast<int64_t>(ld_meta(offsets + e)) + s;
        }
        if (r >= num_rows) {
            errbits |= EP_DEVERR_OVERFLOW;
            return -1;
        }
        return r;
    }
};

struct BulkArgs {
    const uint8_t* src;
    uint8_t* dst;
    int64_t row_bytes;
    int64_t chunk_bytes;
    int32_t nchunks;
    RowMap map;                 // token choice
    const float* topk_weights;  // token choice, optional outputs
    int32_t* recv_src;
    float* recv_weights;
    const int32_t* token_indices; // expert choice
    int32_t T;
    const int32_t* rank_row;      // per rank: [T, R] destination rows
    int32_t R;
    int64_t* recv_topk_idx;
    float* recv_topk_weights;
    uint32_t* err;
    int64_t item_base; // first item of this launch
    int32_t early_load; // load source rows before waiting for the kernel before (see launch_pdl)
    PeerTables peers;   // per rank over peer memory
};

enum BulkSrc : int {
    kSrcTopk = 0,  // item row = token t; destinations = its K routed pairs
    kSrcEc = 1,    // item row = slot s; source token_indices[s]; destination row s
    kSrcRanks = 2, // item row = token t; destinations = its ranks' rows
    kSrcPeers = 3  // item row = token t; destinations = its rows in the ranks' buffers
};

template <typename T>
__device__ __forceinline__ T* table_at(const unsigned long long* table, int r)
{
    return reinterpret_cast<T*>(__ldg(table + r));
}

// Row of token t (rank_row[t, j] = row in this rank's send order) in rank
// j's receive buffer: base(me, j) + rank_row - rank_offsets[j], base from
// this rank's copy of every rank's counts; -1 with EP_DEVERR_OVERFLOW when
// it falls outside the buffer.
__device__ __forceinline__ int64_t peer_row(const PeerTables& p, int R, int j, int64_t row, uint32_t& errbits)
{
    const int32_t* counts = table_at<const int32_t>(p.rank_counts, p.me);
    int64_t local = row - ld_meta(p.rank_offsets + j);
    for (int i = 0; i < p.me; ++i)
        local += ld_meta(counts + i * R + j);
    if (local < 0 || local >= p.capacity) {
        errbits |= EP_DEVERR_OVERFLOW;
        return -1;
    }
    return local;
}

// Top-k entries of token t as rank r sees them (per-rank dispatch): local
// expert id and weight for the experts of rank r, -1 and 0 for the others.
__device__ __forceinline__ void write_rank_topk(const BulkArgs& a, int64_t t, int lane)
{
    const int K = a.map.K;
    const int per_rank = a.map.E / a.R;
    for (int j = lane; j < a.R * K; j += 32) {
        const int r = j / K;
        const int k = j - r * K;
        const int64_t row = ld_meta(a.rank_row + t * a.R + r);
        if (row < 0 || row >= a.map.num_rows)
            continue;
        const int64_t e = __ldg(a.map.topk_idx + t * K + k);
        const bool local = e >= 0 && e < a.map.E && e / per_rank == r;
        if (a.recv_topk_idx != nullptr)
            a.recv_topk_idx[row * K + k] = local ? e - static_cast<int64_t>(r) * per_rank : -1;
        if (a.recv_topk_weights != nullptr)
            a.recv_topk_weights[row * K + k] = local ? __ldg(a.topk_weights + t * K + k) : 0.0f;
    }
}

// The token's K entries as each of its ranks sees them, written into the
// ranks' buffers: lane j holds the token's row in rank j's buffer (or -1).
__device__ __forceinline__ void write_peer_topk(const BulkArgs& a, int64_t t, int lane, int64_t my_row)
{
    const int K = a.map.K;
    const int per_rank = a.map.E / a.R;
    const int n = a.R * K;
    for (int j0 = 0; j0 < n; j0 += 32) { // warp-uniform trip count: every lane takes the shuffle
        const int j = j0 + lane;
        const int r = min(j / K, a.R - 1);
        const int64_t row = __shfl_sync(kFullMask, my_row, r);
        if (j >= n || row < 0)
            continue;
        const int k = j - r * K;
        const int64_t e = __ldg(a.map.topk_idx + t * K + k);
        const bool local = e >= 0 && e < a.map.E && e / per_rank == r;
        if (a.peers.recv_topk_idx != nullptr)
            table_at<int64_t>(a.peers.recv_topk_idx, r)[row * K + k] =
                local ? e - static_cast<int64_t>(r) * per_rank : -1;
        if (a.peers.recv_topk_weights != nullptr)
            table_at<float>(a.peers.recv_topk_weights, r)[row * K + k] =
                local ? __ldg(a.topk_weights + t * K + k) : 0.0f;
    }
}

// One warp per (row, chunk) item; kSrc says what an item row is.
template <int kSrc>
__global__ void __launch_bounds__(32) bulk_dispatch_kernel(BulkArgs a)
{
    constexpr bool kExpertChoice = kSrc == kSrcEc;
    __shared__ __align__(8) uint64_t bar;
    extern __shared__ __align__(128) uint8_t buf[];
    const int lane = threadIdx.x;
    const int64_t item = a.item_base + blockIdx.x;
    const int64_t r = item / a.nchunks;
    const int c = static_cast<int>(item - r * a.nchunks);
    const int64_t off = static_cast<int64_t>(c) * a.chunk_bytes;
    const uint32_t bytes = static_cast<uint32_t>(min(a.chunk_bytes, a.row_bytes - off));
    uint32_t errbits = 0;

    if (!a.early_load)
        pdl_wait(); // the kernel before may have written x or the routing
    int64_t src_row;
    if (kExpertChoice) {
        const int t = __ldg(a.token_indices + r);
        if (t < 0 || t >= a.T) {
            if (lane == 0 && c == 0 && t != -1)
                flag_error(a.err, EP_DEVERR_BAD_INDEX);
            if (a.early_load && blockIdx.x == gridDim.x - 1)
                pdl_wait(); // this grid ends only after the layout before it
            return;
        }
        src_row = t;
    } else {
        src_row = r;
    }

    if (lane == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar, bytes);
        bulk_load_g2s(buf, a.src + src_row * a.row_bytes + off, bytes, &bar);
    }
    // the layout's results (slot, offsets) are final from here on; the
    // expert-choice copy reads none of them and waits only before it ends
    if (a.early_load && !kExpertChoice)
        pdl_wait();
    // destination rows of the first 32 pairs while the load is in flight
    int64_t dst_row = -1;
    uint8_t* dst = a.dst;
    if constexpr (kSrc == kSrcEc) {
        dst_row = lane == 0 ? r : -1;
    } else if constexpr (kSrc == kSrcPeers) {
        if (lane < a.R) {
            const int64_t row = ld_meta(a.rank_row + r * a.R + lane);
            if (row >= 0) {
                dst_row = peer_row(a.peers, a.R, lane, row, errbits);
                dst = table_at<uint8_t>(a.peers.recv_x, lane);
            }
        }
    } else if constexpr (kSrc == kSrcRanks) {
        if (lane < a.R) {
            dst_row = ld_meta(a.rank_row + r * a.R + lane);
            if (dst_row >= a.map.num_rows) {
                errbits |= EP_DEVERR_OVERFLOW;
                dst_row = -1;
            }
        }
    } else if (lane < a.map.K) {
        dst_row = a.map.row(r, lane, errbits);
    }
    __syncwarp();
    const bool ok = mbar_wait_bounded(&bar, 0, a.err);
    if (ok) {
        if (dst_row >= 0)
            bulk_store_s2g(dst + dst_row * a.row_bytes + off, buf, bytes);
        if constexpr (kSrc == kSrcTopk) {
            for (int k = lane + 32; k < a.map.K; k += 32) {
                const int64_t rk = a.map.row(r, k, errbits);
                if (rk >= 0)
                    bulk_store_s2g(a.dst + rk * a.row_bytes + off, buf, bytes);
            }
        }
        bulk_commit();
        bulk_wait_read_all();
    }
    if constexpr (kSrc == kSrcRanks) {
        if (c == 0) {
            if (dst_row >= 0 && a.recv_src != nullptr)
                a.recv_src[dst_row] = static_cast<int32_t>(r);
            if (a.recv_topk_idx != nullptr || a.recv_topk_weights != nullptr)
                write_rank_topk(a, r, lane);
        }
    }
    if constexpr (kSrc == kSrcPeers) {
        if (c == 0) {
            if (dst_row >= 0 && a.peers.recv_src != nullptr)
                table_at<int32_t>(a.peers.recv_src, lane)[dst_row] = static_cast<int32_t>(r);
            if (a.peers.recv_topk_idx != nullptr || a.peers.recv_topk_weights != nullptr)
                write_peer_topk(a, r, lane, dst_row);
        }
    }
    if (kSrc == kSrcTopk && c == 0 && (a.recv_src != nullptr || a.recv_weights != nullptr)) {
        uint32_t ignored = 0;
        for (int k = lane; k < a.map.K; k += 32) {
            const int64_t rk = k < 32 ? dst_row : a.map.row(r, k, ignored);
            if (rk < 0)
                continue;
            if (a.recv_src != nullptr)
                a.recv_src[rk] = static_cast<int32_t>(r);
            if (a.recv_weights != nullptr)
                a.recv_weights[rk] = __ldg(a.topk_weights + r * a.map.K + k);
        }
    }
    if (c == 0) {
        const uint32_t any = __reduce_or_sync(kFullMask, errbits);
        if (lane == 0)
            flag_error(a.err, any);
    }
    // this grid ends only after the layout before it (for the kernels after
    // it): its last CTA waits; the others leave at once and free their slots
    if (kExpertChoice && a.early_load && blockIdx.x == gridDim.x - 1)
        pdl_wait();
}

// Quantised payload formats (values of ep_dtype_t handled by the kernel).
enum QuantFmt : int {
    kQFp8G128 = EP_FP8_E4M3,        // e4m3, fp32 scale per 128 channels
    kQInt8Tok = EP_INT8_PER_TOKEN,  // int8, fp32 scale per row
    kQFp8Tok = EP_FP8_E4M3_PER_TOKEN, // e4m3, fp32 scale per row
    kQMxE4m3 = EP_MXFP8_E4M3,       // e4m3, e8m0 scale per 32
    kQMxE5m2 = EP_MXFP8_E5M2,       // e5m2, e8m0 scale per 32
    kQMxE2m1 = EP_MXFP4_E2M1,       // e2m1 x2, e8m0 scale per 32
    kQBf16 = EP_BF16                // bf16 copy (fused low-latency dispatch only)
};

struct QuantArgs {
    const uint16_t* x;
    int32_t H;
    RowMap map;
    uint8_t* recv;
    void* scales;
    const float* topk_weights;
    int32_t* recv_src;
    float* recv_weights;
    uint32_t* err;
    int32_t early_load; // load the row before waiting for the kernel before (see launch_pdl)
    // fused low-latency mode: the layout is computed in the same launch
    int32_t T, R;
    int32_t* slot;
    uint8_t* in_rank;
    int32_t* counts;
    int32_t* offsets;
    int32_t* rank_counts;
};

// fused low-latency dispatch limits: a CTA scans the ids of all earlier pairs
constexpr int kFusedMaxPairs = 8192;
constexpr int kFusedMaxK = 32;
constexpr int kFusedMaxE = 1024;

#ifndef EP_QUANT_THREADS
#define EP_QUANT_THREADS 256
#endif
constexpr int kQuantThreads = EP_QUANT_THREADS; // threads per token CTA

__device__ __forceinline__ float amax8(uint4 r)
{
    // |x| of a bf16 is its bit pattern without the sign; max over floats
    const float a0 = fmaxf(fabsf(bf16_lo(r.x)), fabsf(bf16_hi(r.x)));
    const float a1 = fmaxf(fabsf(bf16_lo(r.y)), fabsf(bf16_hi(r.y)));
    const float a2 = fmaxf(fabsf(bf16_lo(r.z)), fabsf(bf16_hi(r.z)));
    const float a3 = fmaxf(fabsf(bf16_lo(r.w)), fabsf(bf16_hi(r.w)));
    return fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
}

// Eight bf16 values times `mul` (one IEEE multiply each) encoded in format
// kFmt: 8 bytes (int8 / fp8) in .x/.y, or 4 bytes (fp4) in .x.
template <int kFmt>
__device__ __forceinline__ uint2 encode8(uint4 r, float mul)
{
    float p[8];
    p[0] = __fmul_rn(bf16_lo(r.x), mul);
    p[1] = __fmul_rn(bf16_hi(r.x), mul);
    p[2] = __fmul_rn(bf16_lo(r.y), mul);
    p[3] = __fmul_rn(bf16_hi(r.y), mul);
    p[4] = __fmul_rn(bf16_lo(r.z), mul);
    p[5] = __fmul_rn(bf16_hi(r.z), mul);
    p[6] = __fmul_rn(bf16_lo(r.w), mul);
    p[7] = __fmul_rn(bf16_hi(r.w), mul);
    uint2 q;
    if constexpr (kFmt == kQInt8Tok) {
        uint32_t b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            b[i] = static_cast<uint32_t>(max(-127, min(127, __float2int_rn(p[i])))) & 0xFFu;
        q.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
        q.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
    } else if constexpr (kFmt == kQMxE5m2) {
        q.x = pack_e5m2x2(p[0], p[1]) | (pack_e5m2x2(p[2], p[3]) << 16);
        q.y = pack_e5m2x2(p[4], p[5]) | (pack_e5m2x2(p[6], p[7]) << 16);
    } else if constexpr (kFmt == kQMxE2m1) {
        q.x = pack_e2m1x2(p[0], p[1]) | (pack_e2m1x2(p[2], p[3]) << 8) | (pack_e2m1x2(p[4], p[5]) << 16) |
              (pack_e2m1x2(p[6], p[7]) << 24);
        q.y = 0;
    } else {
        q.x = pack_e4m3x2(p[0], p[1]) | (pack_e4m3x2(p[2], p[3]) << 16);
        q.y = pack_e4m3x2(p[4], p[5]) | (pack_e4m3x2(p[6], p[7]) << 16);
    }
    return q;
}

// One CTA per token, its row staged in shared memory: a TMA bulk load brings
// the bf16 row in (completion on an mbarrier, bounded wait) while the
// threads look up the token's destination rows.  Threads then walk the
// 16-byte vectors of the row (vector v = j*nthr + tid) and reduce the amax
// over each scale group by shuffles -- 16 lanes (128 channels), 4 lanes (32,
// MX) -- or over the CTA for a per-token scale (an extra pass over shared
// memory), encode every element once into a shared code row and scale row,
// and hand those to the TMA engine: one bulk store per destination row,
// issued by different threads.  Rows whose byte size is not a multiple of 16
// are written with 8-byte stores instead.  Registers stay low, so many CTAs
// (and their row loads) are resident per SM.
//   shared memory: x row [2H] | codes [code_row] | scales [scale_row -> 16] | rows [K]
// Shared-memory bytes of one token CTA: x row | codes | scales | rows [K]
// (| fused layout: expert -> k mask [E], histogram [E], per-token rank bits
// [T], small arrays [4 x 32]).
__host__ __device__ inline size_t quant_smem_bytes(int fmt, int H, int K, int E, int T, bool fused)
{
    const size_t nvec = static_cast<size_t>(H) / 8;
    const bool mx = fmt == kQMxE4m3 || fmt == kQMxE5m2 || fmt == kQMxE2m1;
    const size_t code_row = fmt == kQBf16 ? 0 : nvec * (fmt == kQMxE2m1 ? 4 : 8);
    const size_t scale_row =
        fmt == kQBf16 ? 0 : (mx ? nvec / 4 : ((fmt == kQInt8Tok || fmt == kQFp8Tok) ? 4 : nvec / 16 * 4));
    size_t n = nvec * 16 + code_row + ((scale_row + 15) & ~static_cast<size_t>(15)) + sizeof(int64_t) * K;
    if (fused)
        n += sizeof(uint32_t) * (2 * static_cast<size_t>(E) + static_cast<size_t>(T) + 4 * 32);
    return n;
}

// Fused low-latency layout of token t (padded rows e * max_tokens + slot).
// The slot of pair (t, k) is the number of earlier pairs (token-major) routed
// to the same expert: the CTA counts them itself over the ids of tokens
// 0..t, with a shared expert -> k mask.  The last token's CTA scans every id
// anyway, so it also builds the per-expert histogram (counts, offsets by a
// CTA scan) and each token's rank bits (per-rank token counts).  No
// inter-CTA synchronisation: every output is computed from topk_idx alone.
__device__ __forceinline__ void fused_layout(const QuantArgs& a, int64_t t, int64_t* rows, uint32_t* sm,
                                             uint32_t& errbits)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = a.map.K, E = a.map.E;
    const bool last = t == a.T - 1;
    const int per_rank = E / a.R;
    uint32_t* s_kmask = sm;             // [E] which of this token's k route to expert e
    uint32_t* s_hist = sm + E;          // [E] last CTA: pairs per expert
    uint32_t* s_tmask = sm + 2 * E;     // [T] last CTA: rank bits per token
    int* s_cnt = reinterpret_cast<int*>(s_tmask + a.T); // [32] earlier pairs per k
    int* s_e = s_cnt + 32;              // [32] this token's ids (-1 if not routed)
    int* s_rank = s_cnt + 64;           // [32] last CTA: tokens per rank
    int* s_wsum = s_cnt + 96;           // [32] last CTA: scan scratch
    for (int i = tid; i < E; i += kQuantThreads) {
        s_kmask[i] = 0u;
        s_hist[i] = 0u;
    }
    if (last)
        for (int i = tid; i < a.T; i += kQuantThreads)
            s_tmask[i] = 0u;
    if (tid < 32) {
        s_cnt[tid] = 0;
        s_rank[tid] = 0;
    }
    __syncthreads();
    if (tid < K) {
        const int64_t e = __ldg(a.map.topk_idx + t * K + tid);
        const bool ok = e >= 0 && e < E;
        if (!ok && e != -1)
            errbits |= EP_DEVERR_BAD_INDEX;
        s_e[tid] = ok ? static_cast<int>(e) : -1;
        if (ok)
            atomicOr(&s_kmask[e], 1u << tid);
    }
    __syncthreads();
    const int64_t lim = last ? static_cast<int64_t>(a.T) * K : t * K + K;
#pragma unroll 4
    for (int64_t p = tid; p < lim; p += kQuantThreads) {
        const int64_t e = __ldg(a.map.topk_idx + p);
        if (e < 0 || e >= E)
            continue;
        uint32_t m = s_kmask[e];
        while (m) {
            const int k = __ffs(m) - 1;
            m &= m - 1u;
            if (p < t * K + k)
                atomicAdd(&s_cnt[k], 1);
        }
        if (last) {
            atomicAdd(&s_hist[e], 1u);
            atomicOr(&s_tmask[p / K], 1u << static_cast<uint32_t>(e / per_rank));
        }
    }
    __syncthreads();
    if (tid < K) {
        const int e = s_e[tid];
        const int sl = e >= 0 ? s_cnt[tid] : -1;
        a.slot[t * K + tid] = sl;
        int64_t rk = -1;
        if (e >= 0) {
            if (sl < a.map.max_tokens)
                rk = static_cast<int64_t>(e) * a.map.max_tokens + sl;
            else
                errbits |= EP_DEVERR_OVERFLOW;
        }
        rows[tid] = rk;
        if (rk >= 0) {
            if (a.recv_src != nullptr)
                a.recv_src[rk] = static_cast<int32_t>(t);
            if (a.recv_weights != nullptr)
                a.recv_weights[rk] = __ldg(a.topk_weights + t * K + tid);
        }
    }
    if (tid < a.R) {
        bool in = false;
        for (int k = 0; k < K; ++k)
            in |= s_e[k] >= 0 && s_e[k] / per_rank == tid;
        a.in_rank[t * a.R + tid] = in ? 1 : 0;
    }
    if (last) {
        for (int64_t u = tid; u < a.T; u += kQuantThreads) {
            uint32_t m = s_tmask[u];
            while (m) {
                const int r = __ffs(m) - 1;
                m &= m - 1u;
                atomicAdd(&s_rank[r], 1);
            }
        }
        // counts and offsets: thread i owns experts [i*epc, (i+1)*epc)
        const int epc = (E + kQuantThreads - 1) / kQuantThreads;
        const int e0 = min(E, tid * epc), e1 = min(E, e0 + epc);
        int sum = 0;
        for (int e = e0; e < e1; ++e)
            sum += static_cast<int>(s_hist[e]);
        int inc = sum;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(kFullMask, inc, d);
            if (lane >= d)
                inc += v;
        }
        if (lane == 31)
            s_wsum[warp] = inc;
        __syncthreads();
        int run = inc - sum;
        for (int w = 0; w < warp; ++w)
            run += s_wsum[w];
        for (int e = e0; e < e1; ++e) {
            const int c = static_cast<int>(s_hist[e]);
            a.counts[e] = c;
            a.offsets[e] = run;
            run += c;
        }
        if (tid == kQuantThreads - 1)
            a.offsets[E] = run; // the last thread's run ends at the total
        if (tid < a.R)
            a.rank_counts[tid] = s_rank[tid];
    }
}

template <int kFmt, bool kFused>
__global__ void __launch_bounds__(kQuantThreads) quant_dispatch_kernel(QuantArgs a)
{
    constexpr bool kMx = kFmt == kQMxE4m3 || kFmt == kQMxE5m2 || kFmt == kQMxE2m1;
    constexpr bool kPerToken = kFmt == kQInt8Tok || kFmt == kQFp8Tok;
    constexpr bool kCopy = kFmt == kQBf16;
    constexpr int kGroupLanes = kFmt == kQFp8G128 ? 16 : 4; // group modes only
    constexpr int kCodeBytes = kFmt == kQMxE2m1 ? 4 : 8;  // bytes per 8 channels
    extern __shared__ __align__(128) uint8_t qsmem[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float warp_amax[kQuantThreads / 32];
    const int64_t t = blockIdx.x;
    const int tid = threadIdx.x;
    const int nvec = a.H / 8;
    const int row_bytes = a.H * 2;
    const int code_row = kCopy ? row_bytes : nvec * kCodeBytes;
    const int scale_row = kCopy ? 0 : (kMx ? nvec / 4 : (kPerToken ? 4 : nvec / 16 * 4));
    uint8_t* s_x = qsmem;
    uint8_t* s_codes = kCopy ? s_x : qsmem + row_bytes;
    uint8_t* s_scales = qsmem + row_bytes + (kCopy ? 0 : code_row);
    int64_t* rows = reinterpret_cast<int64_t*>(s_scales + ((scale_row + 15) & ~15));

    if (!a.early_load)
        pdl_wait(); // the kernel before may have written x or the routing
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(row_bytes));
        bulk_load_g2s(s_x, reinterpret_cast<const uint8_t*>(a.x) + t * static_cast<int64_t>(row_bytes),
                      static_cast<uint32_t>(row_bytes), &bar);
    }
    if (a.early_load)
        pdl_wait(); // the layout's results are final from here on
    uint32_t errbits = 0;
    if constexpr (kFused) {
        fused_layout(a, t, rows, reinterpret_cast<uint32_t*>(rows + a.map.K), errbits);
    } else {
        for (int k = tid; k < a.map.K; k += kQuantThreads) {
            const int64_t rk = a.map.row(t, k, errbits);
            rows[k] = rk;
            if (rk >= 0) {
                if (a.recv_src != nullptr)
                    a.recv_src[rk] = static_cast<int32_t>(t);
                if (a.recv_weights != nullptr)
                    a.recv_weights[rk] = __ldg(a.topk_weights + t * a.map.K + k);
            }
        }
    }
    if (errbits)
        flag_error(a.err, errbits);
    __syncthreads(); // barrier initialised (and rows written) before anyone reads them
    if (!mbar_wait_bounded(&bar, 0, a.err))
        return;

    float tok_mul = 0.0f;
    if constexpr (kPerToken) {
        float amax = 0.0f;
        for (int v = tid; v < nvec; v += kQuantThreads)
            amax = fmaxf(amax, amax8(*reinterpret_cast<const uint4*>(s_x + v * 16)));
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, d));
        if ((tid & 31) == 0)
            warp_amax[tid >> 5] = amax;
        __syncthreads();
        amax = 0.0f;
#pragma unroll
        for (int w = 0; w < kQuantThreads / 32; ++w)
            amax = fmaxf(amax, warp_amax[w]);
        constexpr float qmax = kFmt == kQInt8Tok ? 127.0f : 448.0f;
        float scale = 0.0f;
        if (amax > 0.0f) {
            scale = __fdiv_rn(amax, qmax);
            tok_mul = fminf(__fdiv_rn(qmax, amax), 3.40282347e38f);
        }
        if (tid == 0)
            *reinterpret_cast<float*>(s_scales) = scale;
    }

    // one vector per thread and step, uniform trip count: every lane takes
    // part in the group shuffles
    auto encode_step = [&](int base, uint4 raw) {
        const int v = base + tid;
        const bool active = v < nvec; // a scale group is all-in or all-out
        float mul = tok_mul;
        if constexpr (!kPerToken) {
            float amax = amax8(raw);
#pragma unroll
            for (int d = kGroupLanes / 2; d >= 1; d >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, d));
            if constexpr (kMx) {
                constexpr int kEmax = kFmt == kQMxE4m3 ? 8 : (kFmt == kQMxE5m2 ? 15 : 2);
                // floor(log2 amax) is the unbiased exponent of a normal amax; a
                // zero or subnormal amax clamps to -127 either way
                const int ef = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
                const int X = max(ef - 127 - kEmax, -127);
                mul = __uint_as_float(static_cast<uint32_t>(127 - X) << 23); // 2^-X, a normal float
                if (active && (tid & 3) == 0)
                    s_scales[v / 4] = static_cast<uint8_t>(X + 127);
            } else {
                float scale = 0.0f;
                mul = 0.0f;
                if (amax > 0.0f) {
                    scale = __fdiv_rn(amax, 448.0f);
                    mul = fminf(__fdiv_rn(448.0f, amax), 3.40282347e38f);
                }
                if (active && (tid & 15) == 0)
                    reinterpret_cast<float*>(s_scales)[v / 16] = scale;
            }
        }
        if (active) {
            // dynamic scales: a zero amax gives zero codes (no -0 codes either)
            const uint2 q = (kMx || mul != 0.0f) ? encode8<kFmt>(raw, mul) : make_uint2(0, 0);
            if constexpr (kCodeBytes == 8)
                sts_v2(s_codes + v * 8, q);
            else
                reinterpret_cast<uint32_t*>(s_codes)[v] = q.x;
        }
    };
    if constexpr (!kCopy) {
        for (int base = 0; base < nvec; base += kQuantThreads) {
            const int v = base + tid;
            encode_step(base, v < nvec ? *reinterpret_cast<const uint4*>(s_x + v * 16) : make_uint4(0, 0, 0, 0));
        }
    }
    fence_proxy_async_shared();
    __syncthreads();

    const bool bulk_codes = (code_row & 15) == 0;
    // A scale row is small (224 bytes at 7168 channels): one bulk copy each
    // would double the copy engine's operations per token for 3% of the
    // bytes, so scales leave by plain 16-byte stores from the threads (or by
    // the copy engine, EP_QUANT_BULK_SCALES)
    const bool bulk_scales =
        kCopy || (EP_QUANT_BULK_SCALES && (scale_row & 15) == 0 && (reinterpret_cast<uintptr_t>(a.scales) & 15) == 0);
    if (bulk_codes) {
        bool issued = false;
        for (int k = tid; k < a.map.K; k += kQuantThreads) {
            const int64_t rk = rows[k];
            if (rk < 0)
                continue;
            bulk_store_s2g(a.recv + rk * code_row, s_codes, static_cast<uint32_t>(code_row));
            if (bulk_scales && !kCopy)
                bulk_store_s2g(static_cast<uint8_t*>(a.scales) + rk * scale_row, s_scales,
                               static_cast<uint32_t>(scale_row));
            issued = true;
        }
        if (issued)
            bulk_commit();
    } else {
        for (int k = 0; k < a.map.K; ++k) {
            const int64_t rk = rows[k];
            if (rk < 0)
                continue;
            uint8_t* dst = a.recv + rk * code_row;
            for (int i = tid; i < code_row / 8; i += kQuantThreads)
                st_v2(dst + i * 8, *reinterpret_cast<const uint2*>(s_codes + i * 8));
        }
    }
    if (!kCopy && !(bulk_codes && bulk_scales) && (scale_row & 15) == 0 &&
        (reinterpret_cast<uintptr_t>(a.scales) & 15) == 0) {
        // every (destination, 16-byte vector) pair of the scale rows by one thread
        const int vpr = scale_row / 16;
        for (int i = tid; i < a.map.K * vpr; i += kQuantThreads) {
            const int k = i / max(vpr, 1); // vpr >= 1 here (a per-token scale row makes the loop empty)
            const int64_t rk = rows[k];
            if (rk >= 0)
                st_v4(static_cast<uint8_t*>(a.scales) + rk * scale_row + (i - k * vpr) * 16,
                      *reinterpret_cast<const uint4*>(s_scales + (i - k * vpr) * 16));
        }
    } else if (!kCopy && !(bulk_codes && bulk_scales)) {
        // scales by plain stores (per-token: 4 bytes; rows not 16-byte multiples)
        for (int k = 0; k < a.map.K; ++k) {
            const int64_t rk = rows[k];
            if (rk < 0)
                continue;
            uint8_t* dst = static_cast<uint8_t*>(a.scales) + rk * scale_row;
            if constexpr (kMx) {
                for (int i = tid; i < scale_row; i += kQuantThreads)
                    dst[i] = s_scales[i];
            } else {
                for (int i = tid; i < scale_row / 4; i += kQuantThreads)
                    reinterpret_cast<float*>(dst)[i] = reinterpret_cast<const float*>(s_scales)[i];
            }
        }
    }
    if (bulk_codes)
        bulk_wait_read_all(); // shared memory must outlive the copies' reads
}

template <int kFmt, bool kFused>
cudaError_t launch_quant(const QuantArgs& a, int32_t T, int32_t K, cudaStream_t stream)
{
    const size_t smem = quant_smem_bytes(kFmt, a.H, K, a.map.E, kFused ? T : 0, kFused);
    auto kernel = quant_dispatch_kernel<kFmt, kFused>;
    if (smem > 48 * 1024) {
        cudaError_t st = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (st != cudaSuccess)
            return st;
    }
    return launch_pdl(kernel, static_cast<unsigned>(T), kQuantThreads, smem, stream, a);
}

template <bool kFused>
cudaError_t launch_quant_fmt(int fmt, const QuantArgs& k, int32_t T, int32_t K, cudaStream_t stream)
{
    switch (fmt) {
    case EP_FP8_E4M3:
        return launch_quant<kQFp8G128, kFused>(k, T, K, stream);
    case EP_INT8_PER_TOKEN:
        return launch_quant<kQInt8Tok, kFused>(k, T, K, stream);
    case EP_FP8_E4M3_PER_TOKEN:
        return launch_quant<kQFp8Tok, kFused>(k, T, K, stream);
    case EP_MXFP8_E4M3:
        return launch_quant<kQMxE4m3, kFused>(k, T, K, stream);
    case EP_MXFP8_E5M2:
        return launch_quant<kQMxE5m2, kFused>(k, T, K, stream);
    case EP_MXFP4_E2M1:
        return launch_quant<kQMxE2m1, kFused>(k, T, K, stream);
    case EP_BF16:
        if constexpr (kFused)
            return launch_quant<kQBf16, true>(k, T, K, stream);
        return cudaErrorInvalidValue;
    default:
        return cudaErrorInvalidValue;
    }
}

constexpr int64_t kMaxGrid = int64_t{1} << 30;

template <int kSrc>
cudaError_t launch_bulk(BulkArgs k, int64_t items, cudaStream_t stream)
{
    for (int64_t base = 0; base < items; base += kMaxGrid) {
        k.item_base = base;
        const unsigned n = static_cast<unsigned>(std::min(kMaxGrid, items - base));
        cudaError_t st = launch_pdl(bulk_dispatch_kernel<kSrc>, n, 32, static_cast<size_t>(k.chunk_bytes), stream, k);
        if (st != cudaSuccess)
            return st;
    }
    return cudaSuccess;
}

} // namespace

bool ll_fusable(int32_t T, int32_t K, int32_t E, int32_t H, int out_dtype)
{
    return T > 0 && static_cast<int64_t>(T) * K <= kFusedMaxPairs && K <= kFusedMaxK && E <= kFusedMaxE &&
           quant_smem_bytes(out_dtype, H, K, E, T, true) <= 200 * 1024;
}

cudaError_t launch_ll_dispatch(const LowLatencyLaunch& a, cudaStream_t stream)
{
    RowMap m{a.topk_idx, nullptr, nullptr, a.K, a.E, EP_LAYOUT_PADDED, a.max_tokens,
             static_cast<int64_t>(a.E) * a.max_tokens};
    QuantArgs k{};
    k.x = static_cast<const uint16_t*>(a.x);
    k.H = a.H;
    k.map = m;
    k.recv = static_cast<uint8_t*>(a.recv_x);
    k.scales = a.recv_scales;
    k.topk_weights = a.topk_weights;
    k.recv_src = a.recv_src;
    k.recv_weights = a.recv_weights;
    k.err = a.err;
    k.T = a.T;
    k.R = a.R;
    k.slot = a.slot;
    k.in_rank = a.in_rank;
    k.counts = a.counts;
    k.offsets = a.offsets;
    k.rank_counts = a.rank_counts;
    return launch_quant_fmt<true>(a.out_dtype, k, a.T, a.K, stream);
}

cudaError_t launch_tc_dispatch(const TcDispatchLaunch& a, cudaStream_t stream)
{
    if (a.T == 0)
        return cudaSuccess;
    RowMap m{a.rows.topk_idx, a.rows.slot, a.rows.offsets, a.rows.K, a.rows.E, a.rows.mode, a.rows.max_tokens,
             a.rows.num_rows};
    if (a.out_dtype != EP_BF16) {
        QuantArgs k{};
        k.x = static_cast<const uint16_t*>(a.x);
        k.H = a.H;
        k.map = m;
        k.recv = static_cast<uint8_t*>(a.recv_x);
        k.scales = a.recv_scales;
        k.topk_weights = a.topk_weights;
        k.recv_src = a.recv_src;
        k.recv_weights = a.recv_weights;
        k.err = a.err;
        k.early_load = a.early_load;
        return launch_quant_fmt<false>(a.out_dtype, k, a.T, a.rows.K, stream);
    }
    BulkArgs k{};
    k.src = static_cast<const uint8_t*>(a.x);
    k.dst = static_cast<uint8_t*>(a.recv_x);
    k.row_bytes = static_cast<int64_t>(a.H) * 2;
    k.nchunks = static_cast<int32_t>((k.row_bytes + kChunkTarget - 1) / kChunkTarget);
    k.chunk_bytes = ((k.row_bytes / k.nchunks + 15) / 16) * 16;
    k.nchunks = static_cast<int32_t>((k.row_bytes + k.chunk_bytes - 1) / k.chunk_bytes);
    k.map = m;
    k.topk_weights = a.topk_weights;
    k.recv_src = a.recv_src;
    k.recv_weights = a.recv_weights;
    k.err = a.err;
    k.early_load = a.early_load;
    return launch_bulk<kSrcTopk>(k, static_cast<int64_t>(a.T) * k.nchunks, stream);
}

cudaError_t launch_ec_dispatch(const EcDispatchLaunch& a, cudaStream_t stream)
{
    const int64_t S = static_cast<int64_t>(a.E) * a.C;
    BulkArgs k{};
    k.src = static_cast<const uint8_t*>(a.x);
    k.dst = static_cast<uint8_t*>(a.recv_x);
    k.row_bytes = static_cast<int64_t>(a.H) * 2;
    k.nchunks = static_cast<int32_t>((k.row_bytes + kChunkTarget - 1) / kChunkTarget);
    k.chunk_bytes = ((k.row_bytes / k.nchunks + 15) / 16) * 16;
    k.nchunks = static_cast<int32_t>((k.row_bytes + k.chunk_bytes - 1) / k.chunk_bytes);
    k.token_indices = a.token_indices;
    k.T = a.T;
    k.err = a.err;
    k.early_load = a.early_load;
    return launch_bulk<kSrcEc>(k, S * k.nchunks, stream);
}

cudaError_t launch_rank_dispatch(const RankDispatchLaunch& a, cudaStream_t stream)
{
    if (a.T == 0)
        return cudaSuccess;
    BulkArgs k{};
    k.src = static_cast<const uint8_t*>(a.x);
    k.dst = static_cast<uint8_t*>(a.recv_x);
    k.row_bytes = static_cast<int64_t>(a.H) * 2;
    k.nchunks = static_cast<int32_t>((k.row_bytes + kChunkTarget - 1) / kChunkTarget);
    k.chunk_bytes = ((k.row_bytes / k.nchunks + 15) / 16) * 16;
    k.nchunks = static_cast<int32_t>((k.row_bytes + k.chunk_bytes - 1) / k.chunk_bytes);
    k.map.topk_idx = a.topk_idx;
    k.map.K = a.K;
    k.map.E = a.E;
    k.map.num_rows = a.num_rows;
    k.topk_weights = a.topk_weights;
    k.recv_src = a.recv_src;
    k.rank_row = a.rank_row;
    k.R = a.R;
    k.recv_topk_idx = a.recv_topk_idx;
    k.recv_topk_weights = a.recv_topk_weights;
    k.T = a.T;
    k.err = a.err;
    k.early_load = a.early_load;
    if (a.peers.recv_x != nullptr) {
        k.peers = a.peers;
        return launch_bulk<kSrcPeers>(k, static_cast<int64_t>(a.T) * k.nchunks, stream);
    }
    return launch_bulk<kSrcRanks>(k, static_cast<int64_t>(a.T) * k.nchunks, stream);
}

} // namespace ep
