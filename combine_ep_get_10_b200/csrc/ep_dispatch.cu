// ep_dispatch.cu -- dispatch kernels.
//
// bf16 dispatch (token choice: DeepEP-Ascend README, API Overview,
// dispatch / low_latency_dispatch; expert choice: DeepEP issue #595,
// Solution 1) is a pure row copy: each source row chunk is read from HBM
// exactly once by the TMA engine (cp.async.bulk global->shared, completion on
// an mbarrier) and written to every destination row by bulk stores
// (cp.async.bulk shared->global), one per destination, issued by different
// lanes.  A CTA is one warp and moves one (row, chunk) item; up to 28 CTAs
// per SM keep ~200 KB of copies in flight per SM and the block scheduler
// balances the tail.  (A persistent variant streaming each CTA's items
// through a 3-4 stage ring measured 10-15% slower.)
//
// Quantised dispatch (README, "Quantization Modes in Normal Dispatch": FP8
// with one fp32 scale per 128 channels, per-token INT8 and FP8, MX FP8/FP4
// with an e8m0 scale per 32): one CTA per token holds the row in registers
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
#define EP_DISPATCH_CHUNK 8192
#endif

constexpr int64_t kChunkTarget = EP_DISPATCH_CHUNK; // bytes per bulk-copy item

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
        const int32_t s = __ldg(slot + t * K + k);
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
            r = static_cast<int64_t>(__ldg(offsets + e)) + s;
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
    uint32_t* err;
    int64_t item_base; // first item of this launch
};

// One warp per (row, chunk) item.  kExpertChoice: item row = slot s, source
// token = token_indices[s], one destination (row s).  Otherwise item row =
// token t, destinations = its K routed pairs.
template <bool kExpertChoice>
__global__ void __launch_bounds__(32) bulk_dispatch_kernel(BulkArgs a)
{
    __shared__ __align__(8) uint64_t bar;
    extern __shared__ __align__(128) uint8_t buf[];
    const int lane = threadIdx.x;
    const int64_t item = a.item_base + blockIdx.x;
    const int64_t r = item / a.nchunks;
    const int c = static_cast<int>(item - r * a.nchunks);
    const int64_t off = static_cast<int64_t>(c) * a.chunk_bytes;
    const uint32_t bytes = static_cast<uint32_t>(min(a.chunk_bytes, a.row_bytes - off));
    uint32_t errbits = 0;

    int64_t src_row;
    if (kExpertChoice) {
        const int t = __ldg(a.token_indices + r);
        if (t < 0 || t >= a.T) {
            if (lane == 0 && c == 0 && t != -1)
                flag_error(a.err, EP_DEVERR_BAD_INDEX);
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
    // destination rows of the first 32 pairs while the load is in flight
    int64_t dst_row = -1;
    if (kExpertChoice) {
        dst_row = lane == 0 ? r : -1;
    } else if (lane < a.map.K) {
        dst_row = a.map.row(r, lane, errbits);
    }
    __syncwarp();
    const bool ok = mbar_wait_bounded(&bar, 0, a.err);
    if (ok) {
        if (dst_row >= 0)
            bulk_store_s2g(a.dst + dst_row * a.row_bytes + off, buf, bytes);
        if (!kExpertChoice) {
            for (int k = lane + 32; k < a.map.K; k += 32) {
                const int64_t rk = a.map.row(r, k, errbits);
                if (rk >= 0)
                    bulk_store_s2g(a.dst + rk * a.row_bytes + off, buf, bytes);
            }
        }
        bulk_commit();
        bulk_wait_read_all();
    }
    if (!kExpertChoice && c == 0 && (a.recv_src != nullptr || a.recv_weights != nullptr)) {
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
}

// Quantised payload formats (values of ep_dtype_t handled by the kernel).
enum QuantFmt : int {
    kQFp8G128 = EP_FP8_E4M3,        // e4m3, fp32 scale per 128 channels
    kQInt8Tok = EP_INT8_PER_TOKEN,  // int8, fp32 scale per row
    kQFp8Tok = EP_FP8_E4M3_PER_TOKEN, // e4m3, fp32 scale per row
    kQMxE4m3 = EP_MXFP8_E4M3,       // e4m3, e8m0 scale per 32
    kQMxE5m2 = EP_MXFP8_E5M2,       // e5m2, e8m0 scale per 32
    kQMxE2m1 = EP_MXFP4_E2M1        // e2m1 x2, e8m0 scale per 32
};

struct QuantArgs {
    const uint16_t* x;
    int32_t H;
    int32_t nper; // 16-byte vectors per thread (<= kQuantMaxVec)
    RowMap map;
    uint8_t* recv;
    void* scales;
    const float* topk_weights;
    int32_t* recv_src;
    float* recv_weights;
    uint32_t* err;
};

constexpr int kQuantMaxVec = 8;     // a row is held in registers: <= 8 vectors of 8 bf16 per thread
constexpr int kQuantVecTarget = 4;  // vectors per thread the launch aims for

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

// One CTA per token.  Thread i holds vectors i, i + nthr, ... of the row
// (all loads issued up front); the amax is reduced over the scale group --
// 16 lanes (128 channels), 4 lanes (32, MX) or the whole CTA (per token) --
// then every thread encodes its vectors once and stores them, with the
// group's scale, to each destination row of the token.
template <int kFmt>
__global__ void __launch_bounds__(512, 1) quant_dispatch_kernel(QuantArgs a)
{
    constexpr bool kMx = kFmt == kQMxE4m3 || kFmt == kQMxE5m2 || kFmt == kQMxE2m1;
    constexpr bool kPerToken = kFmt == kQInt8Tok || kFmt == kQFp8Tok;
    constexpr int kGroupLanes = kFmt == kQFp8G128 ? 16 : 4; // group modes only
    constexpr int kCodeBytes = kFmt == kQMxE2m1 ? 4 : 8;  // bytes per 8 channels
    extern __shared__ __align__(16) int64_t rows[];         // [K]
    __shared__ float warp_amax[32];
    const int64_t t = blockIdx.x;
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;
    const int nvec = a.H / 8;

    const uint8_t* xrow = reinterpret_cast<const uint8_t*>(a.x) + t * static_cast<int64_t>(a.H) * 2;
    uint4 raw[kQuantMaxVec];
#pragma unroll
    for (int j = 0; j < kQuantMaxVec; ++j) {
        const int v = j * nthr + tid;
        raw[j] = make_uint4(0, 0, 0, 0);
        if (j < a.nper && v < nvec)
            raw[j] = ld_nc_v4(xrow + static_cast<int64_t>(v) * 16);
    }

    uint32_t errbits = 0;
    for (int k = tid; k < a.map.K; k += nthr) {
        const int64_t rk = a.map.row(t, k, errbits);
        rows[k] = rk;
        if (rk >= 0) {
            if (a.recv_src != nullptr)
                a.recv_src[rk] = static_cast<int32_t>(t);
            if (a.recv_weights != nullptr)
                a.recv_weights[rk] = __ldg(a.topk_weights + t * a.map.K + k);
        }
    }
    if (errbits)
        flag_error(a.err, errbits);

    float tok_amax = 0.0f;
    if constexpr (kPerToken) {
#pragma unroll
        for (int j = 0; j < kQuantMaxVec; ++j)
            tok_amax = fmaxf(tok_amax, amax8(raw[j]));
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1)
            tok_amax = fmaxf(tok_amax, __shfl_xor_sync(kFullMask, tok_amax, d));
        if ((tid & 31) == 0)
            warp_amax[tid >> 5] = tok_amax;
    }
    __syncthreads();
    if constexpr (kPerToken) {
        tok_amax = 0.0f;
        for (int w = 0; w < (nthr >> 5); ++w)
            tok_amax = fmaxf(tok_amax, warp_amax[w]);
    }

    // codes and scale of each held vector
    uint2 code[kQuantMaxVec];
    float fscale[kQuantMaxVec];   // fp32 scale of the vector's group (128-channel mode)
    uint32_t xbyte[kQuantMaxVec]; // e8m0 byte of the vector's block (MX)
    float tok_scale = 0.0f, tok_mul = 0.0f;
    if constexpr (kPerToken) {
        constexpr float qmax = kFmt == kQInt8Tok ? 127.0f : 448.0f;
        if (tok_amax > 0.0f) {
            tok_scale = __fdiv_rn(tok_amax, qmax);
            tok_mul = fminf(__fdiv_rn(qmax, tok_amax), 3.40282347e38f);
        }
    }
#pragma unroll
    for (int j = 0; j < kQuantMaxVec; ++j) {
        float mul = tok_mul;
        fscale[j] = 0.0f;
        xbyte[j] = 0;
        if constexpr (!kPerToken) {
            float amax = amax8(raw[j]);
#pragma unroll
            for (int d = kGroupLanes / 2; d >= 1; d >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, d));
            if constexpr (kMx) {
                constexpr int kEmax = kFmt == kQMxE4m3 ? 8 : (kFmt == kQMxE5m2 ? 15 : 2);
                // floor(log2 amax) is the unbiased exponent of a normal amax; a
                // zero or subnormal amax clamps to -127 either way
                const int ef = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
                const int X = max(ef - 127 - kEmax, -127);
                xbyte[j] = static_cast<uint32_t>(X + 127);
                mul = __uint_as_float(static_cast<uint32_t>(127 - X) << 23); // 2^-X, a normal float
            } else {
                mul = 0.0f;
                if (amax > 0.0f) {
                    fscale[j] = __fdiv_rn(amax, 448.0f);
                    mul = fminf(__fdiv_rn(448.0f, amax), 3.40282347e38f);
                }
            }
        }
        // dynamic scales: a zero amax gives zero codes (no -0 codes either)
        code[j] = (kMx || mul != 0.0f) ? encode8<kFmt>(raw[j], mul) : make_uint2(0, 0);
    }

    const int64_t code_row = static_cast<int64_t>(nvec) * kCodeBytes;
    for (int k = 0; k < a.map.K; ++k) {
        const int64_t rk = rows[k];
        if (rk < 0)
            continue;
        uint8_t* dst = a.recv + rk * code_row;
#pragma unroll
        for (int j = 0; j < kQuantMaxVec; ++j) {
            const int v = j * nthr + tid;
            if (j >= a.nper || v >= nvec)
                continue;
            if constexpr (kCodeBytes == 8)
                st_v2(dst + static_cast<int64_t>(v) * 8, code[j]);
            else
                st_u32(dst + static_cast<int64_t>(v) * 4, code[j].x);
            if constexpr (kMx) {
                if ((tid & 3) == 0)
                    static_cast<uint8_t*>(a.scales)[rk * (nvec / 4) + v / 4] = static_cast<uint8_t>(xbyte[j]);
            } else if constexpr (kFmt == kQFp8G128) {
                if ((tid & 15) == 0)
                    static_cast<float*>(a.scales)[rk * (nvec / 16) + v / 16] = fscale[j];
            }
        }
        if constexpr (kPerToken) {
            if (tid == 0)
                static_cast<float*>(a.scales)[rk] = tok_scale;
        }
    }
}

template <int kFmt>
cudaError_t launch_quant(const QuantArgs& k, int32_t T, int32_t K, cudaStream_t stream)
{
    const int nvec = k.H / 8;
    int nthr = (nvec + kQuantVecTarget - 1) / kQuantVecTarget;
    nthr = ((nthr + 31) / 32) * 32;
    nthr = std::min(std::max(nthr, 32), 512);
    QuantArgs a = k;
    a.nper = (nvec + nthr - 1) / nthr;
    const size_t smem = sizeof(int64_t) * static_cast<size_t>(K);
    if (smem > 40 * 1024) {
        cudaError_t st = cudaFuncSetAttribute(quant_dispatch_kernel<kFmt>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(smem));
        if (st != cudaSuccess)
            return st;
    }
    quant_dispatch_kernel<kFmt><<<T, nthr, smem, stream>>>(a);
    return cudaGetLastError();
}

constexpr int64_t kMaxGrid = int64_t{1} << 30;

template <bool kExpertChoice>
cudaError_t launch_bulk(BulkArgs k, int64_t items, cudaStream_t stream)
{
    for (int64_t base = 0; base < items; base += kMaxGrid) {
        k.item_base = base;
        const unsigned n = static_cast<unsigned>(std::min(kMaxGrid, items - base));
        bulk_dispatch_kernel<kExpertChoice><<<n, 32, static_cast<size_t>(k.chunk_bytes), stream>>>(k);
        cudaError_t st = cudaGetLastError();
        if (st != cudaSuccess)
            return st;
    }
    return cudaSuccess;
}

} // namespace

cudaError_t launch_tc_dispatch(const TcDispatchLaunch& a, cudaStream_t stream)
{
    if (a.T == 0)
        return cudaSuccess;
    RowMap m{a.rows.topk_idx, a.rows.slot, a.rows.offsets, a.rows.K, a.rows.E, a.rows.mode, a.rows.max_tokens,
             a.rows.num_rows};
    if (a.out_dtype != EP_BF16) {
        QuantArgs k{static_cast<const uint16_t*>(a.x), a.H, 0, m, static_cast<uint8_t*>(a.recv_x), a.recv_scales,
                    a.topk_weights, a.recv_src, a.recv_weights, a.err};
        switch (a.out_dtype) {
        case EP_FP8_E4M3:
            return launch_quant<kQFp8G128>(k, a.T, a.rows.K, stream);
        case EP_INT8_PER_TOKEN:
            return launch_quant<kQInt8Tok>(k, a.T, a.rows.K, stream);
        case EP_FP8_E4M3_PER_TOKEN:
            return launch_quant<kQFp8Tok>(k, a.T, a.rows.K, stream);
        case EP_MXFP8_E4M3:
            return launch_quant<kQMxE4m3>(k, a.T, a.rows.K, stream);
        case EP_MXFP8_E5M2:
            return launch_quant<kQMxE5m2>(k, a.T, a.rows.K, stream);
        case EP_MXFP4_E2M1:
            return launch_quant<kQMxE2m1>(k, a.T, a.rows.K, stream);
        default:
            return cudaErrorInvalidValue;
        }
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
    return launch_bulk<false>(k, static_cast<int64_t>(a.T) * k.nchunks, stream);
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
    return launch_bulk<true>(k, S * k.nchunks, stream);
}

} // namespace ep
