// ep_api.cu -- the C ABI declared in include/ep.h: argument checks on the
// host, then one launcher per operation.  Nothing here allocates device
// memory except ep_peer_alloc (buffers other processes map); only
// ep_get_device_error, and a layout call given a num_valid_host pointer,
// synchronise.
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include <nvtx3/nvToolsExt.h>

#include "ep.h"
#include "ep_internal.h"

namespace {

// An NVTX range named after the entry point, around the whole call (checks
// and launches), so that profilers can attribute kernels to ABI calls.  With
// no tool attached the push and pop return at once.
struct CallRange {
    explicit CallRange(const char* name) { nvtxRangePushA(name); }
    ~CallRange() { nvtxRangePop(); }
    CallRange(const CallRange&) = delete;
    CallRange& operator=(const CallRange&) = delete;
};

using ep::kWorkspaceHeaderBytes;

bool aligned(const void* p, uintptr_t n)
{
    return (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0;
}

ep_status_t from_cuda(cudaError_t e)
{
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

ep_status_t check_routing(const ep_routing_desc_t* r)
{
    if (r == nullptr)
        return EP_ERR_INVALID_ARG;
    if (r->num_tokens < 0 || r->num_experts < 1 || r->num_ranks < 1 || r->num_ranks > 32 ||
        r->num_experts % r->num_ranks != 0)
        return EP_ERR_INVALID_ARG;
    if (r->routing == EP_ROUTING_TOPK) {
        if (r->num_topk < 1)
            return EP_ERR_INVALID_ARG;
        if (static_cast<int64_t>(r->num_tokens) * r->num_topk >= (int64_t{1} << 31))
            return EP_ERR_INVALID_ARG;
        if (r->num_tokens > 0 && (r->topk_idx == nullptr || !aligned(r->topk_idx, 8)))
            return EP_ERR_INVALID_ARG;
        return EP_OK;
    }
    if (r->routing == EP_ROUTING_EXPERT_CHOICE) {
        if (r->capacity < 1)
            return EP_ERR_INVALID_ARG;
        if (static_cast<int64_t>(r->num_experts) * r->capacity >= (int64_t{1} << 31))
            return EP_ERR_INVALID_ARG;
        if (r->token_indices == nullptr || !aligned(r->token_indices, 4))
            return EP_ERR_INVALID_ARG;
        return EP_OK;
    }
    return EP_ERR_INVALID_ARG;
}

size_t workspace_need(const ep_routing_desc_t* r)
{
    if (r->routing == EP_ROUTING_EXPERT_CHOICE)
        return ep::ec_layout_workspace_bytes(r->num_tokens, r->num_experts, r->capacity);
    return ep::tc_layout_workspace_bytes(r->num_experts);
}

// The layout needs its full workspace; dispatch and combine only the header
// (the device error word).
ep_status_t check_workspace(const ep_routing_desc_t* r, const ep_layout_t* l, bool full)
{
    if (l == nullptr)
        return EP_ERR_INVALID_ARG;
    const size_t need = full ? workspace_need(r) : kWorkspaceHeaderBytes;
    if (l->workspace == nullptr || !aligned(l->workspace, 256) || l->workspace_bytes < need)
        return EP_ERR_WORKSPACE;
    return EP_OK;
}

bool valid_mode(ep_buffer_mode_t m)
{
    return m == EP_LAYOUT_COMPACT || m == EP_LAYOUT_PADDED;
}

ep_status_t check_rows(const ep_routing_desc_t* r, const ep_layout_t* l, ep_buffer_mode_t mode, int32_t max_tokens,
                       int64_t num_rows)
{
    if (!valid_mode(mode) || num_rows < 0)
        return EP_ERR_INVALID_ARG;
    if (mode == EP_LAYOUT_PADDED && max_tokens < 1)
        return EP_ERR_INVALID_ARG;
    if (r->num_tokens > 0 && (l->slot == nullptr || !aligned(l->slot, 4)))
        return EP_ERR_INVALID_ARG;
    if (mode == EP_LAYOUT_COMPACT && (l->expert_offsets == nullptr || !aligned(l->expert_offsets, 4)))
        return EP_ERR_INVALID_ARG;
    return EP_OK;
}

ep::TcRows tc_rows(const ep_routing_desc_t* r, const ep_layout_t* l, ep_buffer_mode_t mode, int32_t max_tokens,
                   int64_t num_rows)
{
    ep::TcRows rows{};
    rows.topk_idx = r->topk_idx;
    rows.slot = l->slot;
    rows.offsets = l->expert_offsets;
    rows.K = r->num_topk;
    rows.E = r->num_experts;
    rows.mode = static_cast<int32_t>(mode);
    rows.max_tokens = max_tokens;
    rows.num_rows = num_rows;
    return rows;
}

// ep_get_layout without the host report: argument checks and the launch.
// trigger: the caller launches its own dispatch next, which may start while
// the layout runs (it reads the layout's results only after waiting for it,
// and through L2); without it the kernel launched next starts after the
// layout has finished.
ep_status_t get_layout(const ep_routing_desc_t* routing, const ep_layout_t* layout, ep_stream_t stream,
                       bool trigger = false);

} // namespace

namespace ep {

ep_status_t report_num_valid(const ep_routing_desc_t* routing, const ep_layout_t* layout, cudaStream_t stream)
{
    if (layout->num_valid_host == nullptr)
        return EP_OK;
    const int32_t* total = routing->routing == EP_ROUTING_TOPK ? layout->expert_offsets + routing->num_experts
                                                               : layout->token_offsets + routing->num_tokens;
    cudaError_t e = cudaMemcpyAsync(layout->num_valid_host, total, sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    return from_cuda(e);
}

} // namespace ep

extern "C" {

size_t ep_workspace_bytes(const ep_routing_desc_t* routing)
{
    if (check_routing(routing) != EP_OK)
        return 0;
    return workspace_need(routing);
}

ep_status_t ep_workspace_init(void* workspace, size_t bytes, ep_stream_t stream)
{
    CallRange range_("ep_workspace_init");
    if (workspace == nullptr || !aligned(workspace, 256) || bytes < kWorkspaceHeaderBytes)
        return EP_ERR_WORKSPACE;
    return from_cuda(cudaMemsetAsync(workspace, 0, bytes, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status_t ep_get_layout(const ep_routing_desc_t* routing, const ep_layout_t* layout, ep_stream_t stream)
{
    CallRange range_("ep_get_layout");
    const ep_status_t st = get_layout(routing, layout, stream);
    if (st != EP_OK)
        return st;
    return ep::report_num_valid(routing, layout, reinterpret_cast<cudaStream_t>(stream));
}

} // extern "C"

namespace {

ep_status_t get_layout(const ep_routing_desc_t* routing, const ep_layout_t* layout, ep_stream_t stream,
                       bool trigger)
{
    ep_status_t st = check_routing(routing);
    if (st != EP_OK)
        return st;
    st = check_workspace(routing, layout, true);
    if (st != EP_OK)
        return st;
    const int32_t T = routing->num_tokens, E = routing->num_experts, R = routing->num_ranks;
    if (layout->num_tokens_per_expert == nullptr || layout->num_tokens_per_rank == nullptr ||
        !aligned(layout->num_tokens_per_expert, 4) || !aligned(layout->num_tokens_per_rank, 4))
        return EP_ERR_INVALID_ARG;
    if (T > 0 && layout->is_token_in_rank == nullptr)
        return EP_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t* err = ep::error_word(layout->workspace);
    if (routing->routing == EP_ROUTING_TOPK) {
        if (E > ep::kMaxTopkLayoutExperts)
            return EP_ERR_UNSUPPORTED;
        if (layout->expert_offsets == nullptr || !aligned(layout->expert_offsets, 4))
            return EP_ERR_INVALID_ARG;
        if (T > 0 && (layout->slot == nullptr || !aligned(layout->slot, 4)))
            return EP_ERR_INVALID_ARG;
        ep::TcLayoutLaunch a{routing->topk_idx,
                             T,
                             routing->num_topk,
                             E,
                             R,
                             layout->num_tokens_per_expert,
                             layout->expert_offsets,
                             layout->num_tokens_per_rank,
                             layout->is_token_in_rank,
                             layout->slot,
                             err,
                             layout->workspace,
                             trigger ? 1 : 0};
        return from_cuda(ep::launch_tc_layout(a, s));
    }
    if (layout->token_offsets == nullptr || layout->token_slots == nullptr || !aligned(layout->token_offsets, 4) ||
        !aligned(layout->token_slots, 4))
        return EP_ERR_INVALID_ARG;
    ep::EcLayoutLaunch a{routing->token_indices,
                         T,
                         E,
                         routing->capacity,
                         R,
                         layout->num_tokens_per_expert,
                         layout->num_tokens_per_rank,
                         layout->is_token_in_rank,
                         layout->token_offsets,
                         layout->token_slots,
                         layout->workspace,
                         err,
                         trigger ? 1 : 0};
    return from_cuda(ep::launch_ec_layout(a, s));
}

// Host-side checks of a token-choice dispatch call (ep_dispatch and the
// dispatch half of ep_dispatch_low_latency).
ep_status_t check_dispatch_args(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                const ep_layout_t* layout, ep_buffer_mode_t mode, int32_t max_tokens_per_expert,
                                int64_t num_recv_rows, ep_dtype_t out_dtype, const float* topk_weights, void* recv_x,
                                void* recv_scales, int32_t* recv_src, float* recv_weights)
{
    ep_status_t st = check_routing(routing);
    if (st != EP_OK)
        return st;
    if (routing->routing != EP_ROUTING_TOPK)
        return EP_ERR_INVALID_ARG;
    st = check_workspace(routing, layout, false);
    if (st != EP_OK)
        return st;
    st = check_rows(routing, layout, mode, max_tokens_per_expert, num_recv_rows);
    if (st != EP_OK)
        return st;
    if (hidden < 1 || hidden % 8 != 0)
        return EP_ERR_INVALID_ARG;
    if (out_dtype == EP_FP32 || out_dtype < EP_BF16 || out_dtype > EP_MXFP4_E2M1)
        return EP_ERR_INVALID_ARG;
    if (out_dtype != EP_BF16) {
        const bool mx = out_dtype == EP_MXFP8_E4M3 || out_dtype == EP_MXFP8_E5M2 || out_dtype == EP_MXFP4_E2M1;
        const int group = out_dtype == EP_FP8_E4M3 ? 128 : (mx ? 32 : 8);
        if (hidden % group != 0 || (num_recv_rows > 0 && recv_scales == nullptr) || !aligned(recv_scales, mx ? 1 : 4))
            return EP_ERR_INVALID_ARG;
        if (hidden > ep::kMaxQuantHidden)
            return EP_ERR_UNSUPPORTED;
    }
    const int32_t T = routing->num_tokens;
    if (T > 0 && (x == nullptr || !aligned(x, 16)))
        return EP_ERR_INVALID_ARG;
    if (num_recv_rows > 0 && (recv_x == nullptr || !aligned(recv_x, 16)))
        return EP_ERR_INVALID_ARG;
    if (recv_weights != nullptr && (topk_weights == nullptr || !aligned(topk_weights, 4) || !aligned(recv_weights, 4)))
        return EP_ERR_INVALID_ARG;
    if (recv_src != nullptr && !aligned(recv_src, 4))
        return EP_ERR_INVALID_ARG;
    return EP_OK;
}

// The dispatch launch of ep_dispatch (early_load 0: wait for the kernel
// before, whatever it is, before reading anything) and of ep_layout_dispatch
// (early_load 1: the kernel before is this library's layout, launched just
// now on the same stream).  Arguments are checked by the caller.
ep_status_t launch_dispatch(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                            const ep_layout_t* layout, ep_buffer_mode_t mode, int32_t max_tokens_per_expert,
                            int64_t num_recv_rows, ep_dtype_t out_dtype, const float* topk_weights, void* recv_x,
                            void* recv_scales, int32_t* recv_src, float* recv_weights, ep_stream_t stream,
                            bool early_load)
{
    ep::TcDispatchLaunch a{x,
                           routing->num_tokens,
                           hidden,
                           tc_rows(routing, layout, mode, max_tokens_per_expert, num_recv_rows),
                           static_cast<int32_t>(out_dtype),
                           topk_weights,
                           recv_x,
                           recv_scales,
                           recv_src,
                           recv_weights,
                           ep::error_word(layout->workspace),
                           early_load ? 1 : 0};
    return from_cuda(ep::launch_tc_dispatch(a, reinterpret_cast<cudaStream_t>(stream)));
}

} // namespace

extern "C" {

ep_status_t ep_dispatch(const void* x, int32_t hidden, const ep_routing_desc_t* routing, const ep_layout_t* layout,
                        ep_buffer_mode_t mode, int32_t max_tokens_per_expert, int64_t num_recv_rows,
                        ep_dtype_t out_dtype, const float* topk_weights, void* recv_x, void* recv_scales,
                        int32_t* recv_src, float* recv_weights, ep_stream_t stream)
{
    CallRange range_("ep_dispatch");
    ep_status_t st = check_dispatch_args(x, hidden, routing, layout, mode, max_tokens_per_expert, num_recv_rows,
                                         out_dtype, topk_weights, recv_x, recv_scales, recv_src, recv_weights);
    if (st != EP_OK)
        return st;
    return launch_dispatch(x, hidden, routing, layout, mode, max_tokens_per_expert, num_recv_rows, out_dtype,
                           topk_weights, recv_x, recv_scales, recv_src, recv_weights, stream, false);
}

ep_status_t ep_layout_dispatch(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                               const ep_layout_t* layout, ep_buffer_mode_t mode, int32_t max_tokens_per_expert,
                               int64_t num_recv_rows, ep_dtype_t out_dtype, const float* topk_weights, void* recv_x,
                               void* recv_scales, int32_t* recv_src, float* recv_weights, ep_stream_t stream)
{
    CallRange range_("ep_layout_dispatch");
    // the dispatch's checks first: nothing is launched unless both calls can run
    ep_status_t st = check_dispatch_args(x, hidden, routing, layout, mode, max_tokens_per_expert, num_recv_rows,
                                         out_dtype, topk_weights, recv_x, recv_scales, recv_src, recv_weights);
    if (st != EP_OK)
        return st;
    st = get_layout(routing, layout, stream, true);
    if (st != EP_OK)
        return st;
    st = launch_dispatch(x, hidden, routing, layout, mode, max_tokens_per_expert, num_recv_rows, out_dtype,
                         topk_weights, recv_x, recv_scales, recv_src, recv_weights, stream, true);
    if (st != EP_OK)
        return st;
    return ep::report_num_valid(routing, layout, reinterpret_cast<cudaStream_t>(stream));
}

ep_status_t ep_dispatch_low_latency(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                    const ep_layout_t* layout, int32_t max_tokens_per_expert, ep_dtype_t out_dtype,
                                    const float* topk_weights, void* recv_x, void* recv_scales, int32_t* recv_src,
                                    float* recv_weights, ep_stream_t stream)
{
    CallRange range_("ep_dispatch_low_latency");
    ep_status_t st = check_routing(routing);
    if (st != EP_OK)
        return st;
    if (routing->routing != EP_ROUTING_TOPK)
        return EP_ERR_INVALID_ARG;
    st = check_workspace(routing, layout, true); // the unfused fallback runs ep_get_layout
    if (st != EP_OK)
        return st;
    if (max_tokens_per_expert < 1)
        return EP_ERR_INVALID_ARG;
    const int32_t T = routing->num_tokens, K = routing->num_topk, E = routing->num_experts, R = routing->num_ranks;
    if (E > ep::kMaxTopkLayoutExperts)
        return EP_ERR_UNSUPPORTED;
    if (layout->num_tokens_per_expert == nullptr || layout->num_tokens_per_rank == nullptr ||
        layout->expert_offsets == nullptr || !aligned(layout->num_tokens_per_expert, 4) ||
        !aligned(layout->num_tokens_per_rank, 4) || !aligned(layout->expert_offsets, 4))
        return EP_ERR_INVALID_ARG;
    if (T > 0 && (layout->is_token_in_rank == nullptr || layout->slot == nullptr || !aligned(layout->slot, 4)))
        return EP_ERR_INVALID_ARG;
    const int64_t rows = static_cast<int64_t>(E) * max_tokens_per_expert;
    st = check_dispatch_args(x, hidden, routing, layout, EP_LAYOUT_PADDED, max_tokens_per_expert, rows, out_dtype,
                             topk_weights, recv_x, recv_scales, recv_src, recv_weights);
    if (st != EP_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (ep::ll_fusable(T, K, E, hidden, static_cast<int>(out_dtype))) {
        ep::LowLatencyLaunch a{x,
                               T,
                               hidden,
                               K,
                               E,
                               R,
                               max_tokens_per_expert,
                               routing->topk_idx,
                               static_cast<int32_t>(out_dtype),
                               topk_weights,
                               recv_x,
                               recv_scales,
                               recv_src,
                               recv_weights,
                               layout->slot,
                               layout->is_token_in_rank,
                               layout->num_tokens_per_expert,
                               layout->expert_offsets,
                               layout->num_tokens_per_rank,
                               ep::error_word(layout->workspace)};
        st = from_cuda(ep::launch_ll_dispatch(a, s));
    } else {
        st = get_layout(routing, layout, stream, true);
        if (st == EP_OK)
            st = launch_dispatch(x, hidden, routing, layout, EP_LAYOUT_PADDED, max_tokens_per_expert, rows,
                                 out_dtype, topk_weights, recv_x, recv_scales, recv_src, recv_weights, stream, true);
    }
    if (st != EP_OK)
        return st;
    return ep::report_num_valid(routing, layout, s);
}

ep_status_t ep_combine(const void* y, int32_t hidden, int64_t num_y_rows, const ep_routing_desc_t* routing,
                       const ep_layout_t* layout, ep_buffer_mode_t mode, int32_t max_tokens_per_expert,
                       const float* topk_weights, void* out, ep_dtype_t out_dtype, ep_stream_t stream)
{
    CallRange range_("ep_combine");
    ep_status_t st = check_routing(routing);
    if (st != EP_OK)
        return st;
    if (routing->routing != EP_ROUTING_TOPK)
        return EP_ERR_INVALID_ARG;
    st = check_workspace(routing, layout, false);
    if (st != EP_OK)
        return st;
    st = check_rows(routing, layout, mode, max_tokens_per_expert, num_y_rows);
    if (st != EP_OK)
        return st;
    if (hidden < 1 || hidden % 8 != 0 || (out_dtype != EP_BF16 && out_dtype != EP_FP32))
        return EP_ERR_INVALID_ARG;
    const int32_t T = routing->num_tokens;
    if (num_y_rows > 0 && (y == nullptr || !aligned(y, 16)))
        return EP_ERR_INVALID_ARG;
    if (T > 0 && (out == nullptr || !aligned(out, 16) || topk_weights == nullptr || !aligned(topk_weights, 4)))
        return EP_ERR_INVALID_ARG;
    ep::TcCombineLaunch a{y,
                          T,
                          hidden,
                          tc_rows(routing, layout, mode, max_tokens_per_expert, num_y_rows),
                          topk_weights,
                          out,
                          static_cast<int32_t>(out_dtype),
                          ep::error_word(layout->workspace)};
    return from_cuda(ep::launch_tc_combine(a, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {

ep_status_t check_ec_dispatch(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                              const ep_layout_t* layout, const void* recv_x)
{
    ep_status_t st = check_routing(routing);
    if (st != EP_OK)
        return st;
    if (routing->routing != EP_ROUTING_EXPERT_CHOICE)
        return EP_ERR_INVALID_ARG;
    if (layout == nullptr || layout->workspace == nullptr || !aligned(layout->workspace, 256) ||
        layout->workspace_bytes < kWorkspaceHeaderBytes)
        return EP_ERR_WORKSPACE;
    if (hidden < 1 || hidden % 8 != 0)
        return EP_ERR_INVALID_ARG;
    if ((routing->num_tokens > 0 && (x == nullptr || !aligned(x, 16))) || recv_x == nullptr || !aligned(recv_x, 16))
        return EP_ERR_INVALID_ARG;
    return EP_OK;
}

ep_status_t launch_ec_dispatch(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                               const ep_layout_t* layout, void* recv_x, ep_stream_t stream, bool early_load)
{
    ep::EcDispatchLaunch a{x,
                           routing->num_tokens,
                           hidden,
                           routing->num_experts,
                           routing->capacity,
                           routing->token_indices,
                           recv_x,
                           ep::error_word(layout->workspace),
                           early_load ? 1 : 0};
    return from_cuda(ep::launch_ec_dispatch(a, reinterpret_cast<cudaStream_t>(stream)));
}

} // namespace

ep_status_t ep_dispatch_expert_choice(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                      const ep_layout_t* layout, void* recv_x, ep_stream_t stream)
{
    CallRange range_("ep_dispatch_expert_choice");
    const ep_status_t st = check_ec_dispatch(x, hidden, routing, layout, recv_x);
    if (st != EP_OK)
        return st;
    return launch_ec_dispatch(x, hidden, routing, layout, recv_x, stream, false);
}

ep_status_t ep_layout_dispatch_expert_choice(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                             const ep_layout_t* layout, void* recv_x, ep_stream_t stream)
{
    CallRange range_("ep_layout_dispatch_expert_choice");
    // the dispatch's checks first: nothing is launched unless both calls can run
    ep_status_t st = check_ec_dispatch(x, hidden, routing, layout, recv_x);
    if (st != EP_OK)
        return st;
    st = get_layout(routing, layout, stream, true);
    if (st != EP_OK)
        return st;
    st = launch_ec_dispatch(x, hidden, routing, layout, recv_x, stream, true);
    if (st != EP_OK)
        return st;
    return ep::report_num_valid(routing, layout, reinterpret_cast<cudaStream_t>(stream));
}

ep_status_t ep_combine_expert_choice(const void* y, int32_t hidden, const ep_routing_desc_t* routing,
                                     const ep_layout_t* layout, const float* expert_weights, void* out,
                                     ep_dtype_t out_dtype, ep_stream_t stream)
{
    CallRange range_("ep_combine_expert_choice");
    ep_status_t st = check_routing(routing);
    if (st != EP_OK)
        return st;
    if (routing->routing != EP_ROUTING_EXPERT_CHOICE)
        return EP_ERR_INVALID_ARG;
    if (layout == nullptr || layout->workspace == nullptr || !aligned(layout->workspace, 256) ||
        layout->workspace_bytes < kWorkspaceHeaderBytes)
        return EP_ERR_WORKSPACE;
    if (hidden < 1 || hidden % 8 != 0 || (out_dtype != EP_BF16 && out_dtype != EP_FP32))
        return EP_ERR_INVALID_ARG;
    if (y == nullptr || !aligned(y, 16) || expert_weights == nullptr || !aligned(expert_weights, 4))
        return EP_ERR_INVALID_ARG;
    if (layout->token_offsets == nullptr || layout->token_slots == nullptr || !aligned(layout->token_offsets, 4) ||
        !aligned(layout->token_slots, 4))
        return EP_ERR_INVALID_ARG;
    if (routing->num_tokens > 0 && (out == nullptr || !aligned(out, 16)))
        return EP_ERR_INVALID_ARG;
    ep::EcCombineLaunch a{y,
                          routing->num_tokens,
                          hidden,
                          static_cast<int64_t>(routing->num_experts) * routing->capacity,
                          layout->token_offsets,
                          layout->token_slots,
                          expert_weights,
                          out,
                          static_cast<int32_t>(out_dtype),
                          ep::error_word(layout->workspace)};
    return from_cuda(ep::launch_ec_combine(a, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {

// Checks shared by the per-rank entry points: routing, the error word of
// the layout workspace, and a rank layout with both arrays.
ep_status_t check_rank_call(const ep_routing_desc_t* routing, const ep_layout_t* layout,
                            const ep_rank_layout_t* rank_layout)
{
    ep_status_t st = check_routing(routing);
    if (st != EP_OK)
        return st;
    st = check_workspace(routing, layout, false);
    if (st != EP_OK)
        return st;
    if (rank_layout == nullptr || rank_layout->rank_offsets == nullptr || !aligned(rank_layout->rank_offsets, 4))
        return EP_ERR_INVALID_ARG;
    if (routing->num_tokens > 0 && (rank_layout->rank_row == nullptr || !aligned(rank_layout->rank_row, 4)))
        return EP_ERR_INVALID_ARG;
    return EP_OK;
}

// Peer tables: one process per rank of the routing; the required tables
// (recv_x, y, rank_counts) present, every table 8-byte aligned.
ep_status_t check_peers(const ep_routing_desc_t* routing, const ep_peers_t* p)
{
    if (p == nullptr || p->num_ranks != routing->num_ranks || p->rank < 0 || p->rank >= p->num_ranks ||
        p->capacity < 0)
        return EP_ERR_INVALID_ARG;
    const void* required[] = {p->recv_x, p->y, p->rank_counts};
    for (const void* t : required)
        if (t == nullptr || !aligned(t, 8))
            return EP_ERR_INVALID_ARG;
    const void* optional[] = {p->recv_topk_idx, p->recv_topk_weights, p->recv_src};
    for (const void* t : optional)
        if (t != nullptr && !aligned(t, 8))
            return EP_ERR_INVALID_ARG;
    return EP_OK;
}

ep::PeerTables peer_tables(const ep_peers_t* p, const ep_rank_layout_t* rank_layout)
{
    auto table = [](const void* t) { return static_cast<const unsigned long long*>(t); };
    ep::PeerTables k{};
    k.recv_x = table(p->recv_x);
    k.recv_topk_idx = table(p->recv_topk_idx);
    k.recv_topk_weights = table(p->recv_topk_weights);
    k.recv_src = table(p->recv_src);
    k.y = table(p->y);
    k.rank_counts = table(p->rank_counts);
    k.rank_offsets = rank_layout->rank_offsets;
    k.me = p->rank;
    k.capacity = p->capacity;
    return k;
}

} // namespace

ep_status_t ep_get_rank_layout(const ep_routing_desc_t* routing, const ep_layout_t* layout,
                               const ep_rank_layout_t* rank_layout, ep_stream_t stream)
{
    CallRange range_("ep_get_rank_layout");
    ep_status_t st = check_rank_call(routing, layout, rank_layout);
    if (st != EP_OK)
        return st;
    if (layout->num_tokens_per_rank == nullptr || !aligned(layout->num_tokens_per_rank, 4) ||
        (routing->num_tokens > 0 && layout->is_token_in_rank == nullptr))
        return EP_ERR_INVALID_ARG;
    ep::RankLayoutLaunch a{layout->is_token_in_rank,
                           layout->num_tokens_per_rank,
                           routing->num_tokens,
                           routing->num_ranks,
                           rank_layout->rank_offsets,
                           rank_layout->rank_row};
    return from_cuda(ep::launch_rank_layout(a, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {

ep_status_t check_rank_dispatch(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                const ep_layout_t* layout, const ep_rank_layout_t* rank_layout, int64_t num_recv_rows,
                                const float* topk_weights, const void* recv_x, const int64_t* recv_topk_idx,
                                const float* recv_topk_weights, const int32_t* recv_src);

ep_status_t launch_rank_dispatch(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                 const ep_layout_t* layout, const ep_rank_layout_t* rank_layout,
                                 int64_t num_recv_rows, const float* topk_weights, void* recv_x,
                                 int64_t* recv_topk_idx, float* recv_topk_weights, int32_t* recv_src,
                                 ep_stream_t stream, bool early_load)
{
    ep::RankDispatchLaunch a{x,
                             routing->num_tokens,
                             hidden,
                             routing->num_topk,
                             routing->num_experts,
                             routing->num_ranks,
                             routing->topk_idx,
                             topk_weights,
                             rank_layout->rank_row,
                             num_recv_rows,
                             recv_x,
                             recv_topk_idx,
                             recv_topk_weights,
                             recv_src,
                             ep::error_word(layout->workspace),
                             ep::PeerTables{},
                             early_load ? 1 : 0};
    return from_cuda(ep::launch_rank_dispatch(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status_t launch_rank_layout(const ep_routing_desc_t* routing, const ep_layout_t* layout,
                               const ep_rank_layout_t* rank_layout, ep_stream_t stream)
{
    ep::RankLayoutLaunch a{layout->is_token_in_rank,
                           layout->num_tokens_per_rank,
                           routing->num_tokens,
                           routing->num_ranks,
                           rank_layout->rank_offsets,
                           rank_layout->rank_row,
                           1}; // the per-rank dispatch of the same call follows
    return from_cuda(ep::launch_rank_layout(a, reinterpret_cast<cudaStream_t>(stream)));
}

} // namespace

ep_status_t ep_layout_dispatch_ranks(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                     const ep_layout_t* layout, const ep_rank_layout_t* rank_layout,
                                     int64_t num_recv_rows, const float* topk_weights, void* recv_x,
                                     int64_t* recv_topk_idx, float* recv_topk_weights, int32_t* recv_src,
                                     ep_stream_t stream)
{
    CallRange range_("ep_layout_dispatch_ranks");
    // every call's checks first: nothing is launched unless all three can run
    ep_status_t st = check_rank_dispatch(x, hidden, routing, layout, rank_layout, num_recv_rows, topk_weights,
                                         recv_x, recv_topk_idx, recv_topk_weights, recv_src);
    if (st != EP_OK)
        return st;
    st = check_workspace(routing, layout, true);
    if (st != EP_OK)
        return st;
    if (layout->num_tokens_per_rank == nullptr || !aligned(layout->num_tokens_per_rank, 4) ||
        (routing->num_tokens > 0 && layout->is_token_in_rank == nullptr))
        return EP_ERR_INVALID_ARG;
    st = get_layout(routing, layout, stream);
    if (st != EP_OK)
        return st;
    st = launch_rank_layout(routing, layout, rank_layout, stream);
    if (st != EP_OK)
        return st;
    st = launch_rank_dispatch(x, hidden, routing, layout, rank_layout, num_recv_rows, topk_weights, recv_x,
                              recv_topk_idx, recv_topk_weights, recv_src, stream, true);
    if (st != EP_OK)
        return st;
    return ep::report_num_valid(routing, layout, reinterpret_cast<cudaStream_t>(stream));
}

ep_status_t ep_dispatch_ranks(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                              const ep_layout_t* layout, const ep_rank_layout_t* rank_layout, int64_t num_recv_rows,
                              const float* topk_weights, void* recv_x, int64_t* recv_topk_idx,
                              float* recv_topk_weights, int32_t* recv_src, ep_stream_t stream)
{
    CallRange range_("ep_dispatch_ranks");
    const ep_status_t st = check_rank_dispatch(x, hidden, routing, layout, rank_layout, num_recv_rows, topk_weights,
                                               recv_x, recv_topk_idx, recv_topk_weights, recv_src);
    if (st != EP_OK)
        return st;
    return launch_rank_dispatch(x, hidden, routing, layout, rank_layout, num_recv_rows, topk_weights, recv_x,
                                recv_topk_idx, recv_topk_weights, recv_src, stream, false);
}

namespace {

ep_status_t check_rank_dispatch(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                                const ep_layout_t* layout, const ep_rank_layout_t* rank_layout, int64_t num_recv_rows,
                                const float* topk_weights, const void* recv_x, const int64_t* recv_topk_idx,
                                const float* recv_topk_weights, const int32_t* recv_src)
{
    ep_status_t st = check_rank_call(routing, layout, rank_layout);
    if (st != EP_OK)
        return st;
    if (routing->routing != EP_ROUTING_TOPK || hidden < 1 || hidden % 8 != 0 || num_recv_rows < 0)
        return EP_ERR_INVALID_ARG;
    const int32_t T = routing->num_tokens;
    if (T > 0 && (x == nullptr || !aligned(x, 16)))
        return EP_ERR_INVALID_ARG;
    if (num_recv_rows > 0 && (recv_x == nullptr || !aligned(recv_x, 16)))
        return EP_ERR_INVALID_ARG;
    if (recv_topk_idx != nullptr && !aligned(recv_topk_idx, 8))
        return EP_ERR_INVALID_ARG;
    if (recv_topk_weights != nullptr &&
        ((T > 0 && topk_weights == nullptr) || !aligned(topk_weights, 4) || !aligned(recv_topk_weights, 4)))
        return EP_ERR_INVALID_ARG;
    if (recv_src != nullptr && !aligned(recv_src, 4))
        return EP_ERR_INVALID_ARG;
    return EP_OK;
}

} // namespace

ep_status_t ep_combine_ranks(const void* y, int32_t hidden, int64_t num_y_rows, const ep_routing_desc_t* routing,
                             const ep_layout_t* layout, const ep_rank_layout_t* rank_layout, void* out,
                             ep_dtype_t out_dtype, ep_stream_t stream)
{
    CallRange range_("ep_combine_ranks");
    ep_status_t st = check_rank_call(routing, layout, rank_layout);
    if (st != EP_OK)
        return st;
    if (hidden < 1 || hidden % 8 != 0 || num_y_rows < 0 || (out_dtype != EP_BF16 && out_dtype != EP_FP32))
        return EP_ERR_INVALID_ARG;
    const int32_t T = routing->num_tokens;
    if (num_y_rows > 0 && (y == nullptr || !aligned(y, 16)))
        return EP_ERR_INVALID_ARG;
    if (T > 0 && (out == nullptr || !aligned(out, 16)))
        return EP_ERR_INVALID_ARG;
    if (T == 0)
        return EP_OK;
    ep::RankCombineLaunch a{y,
                            T,
                            hidden,
                            routing->num_ranks,
                            num_y_rows,
                            rank_layout->rank_row,
                            out,
                            static_cast<int32_t>(out_dtype),
                            ep::error_word(layout->workspace)};
    return from_cuda(ep::launch_rank_combine(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status_t ep_peer_alloc(size_t bytes, void** ptr, void* handle)
{
    CallRange range_("ep_peer_alloc");
    if (bytes == 0 || ptr == nullptr || handle == nullptr)
        return EP_ERR_INVALID_ARG;
    static_assert(sizeof(cudaIpcMemHandle_t) == EP_IPC_HANDLE_BYTES, "IPC handle size");
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
        cudaGetLastError();
        return EP_ERR_CUDA;
    }
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, p) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(p);
        return EP_ERR_CUDA;
    }
    std::memcpy(handle, &h, sizeof(h));
    *ptr = p;
    return EP_OK;
}

ep_status_t ep_peer_free(void* ptr)
{
    CallRange range_("ep_peer_free");
    if (ptr == nullptr)
        return EP_ERR_INVALID_ARG;
    return from_cuda(cudaFree(ptr));
}

ep_status_t ep_peer_open(const void* handle, void** ptr)
{
    CallRange range_("ep_peer_open");
    if (handle == nullptr || ptr == nullptr)
        return EP_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    void* p = nullptr;
    if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
        cudaGetLastError();
        return EP_ERR_CUDA;
    }
    *ptr = p;
    return EP_OK;
}

ep_status_t ep_peer_close(void* ptr)
{
    CallRange range_("ep_peer_close");
    if (ptr == nullptr)
        return EP_ERR_INVALID_ARG;
    return from_cuda(cudaIpcCloseMemHandle(ptr));
}

ep_status_t ep_peer_publish_counts(const ep_routing_desc_t* routing, const ep_layout_t* layout,
                                   const ep_peers_t* peers, ep_stream_t stream)
{
    CallRange range_("ep_peer_publish_counts");
    ep_status_t st = check_routing(routing);
    if (st != EP_OK)
        return st;
    st = check_peers(routing, peers);
    if (st != EP_OK)
        return st;
    if (layout == nullptr || layout->num_tokens_per_rank == nullptr || !aligned(layout->num_tokens_per_rank, 4))
        return EP_ERR_INVALID_ARG;
    ep::PublishCountsLaunch a{layout->num_tokens_per_rank, static_cast<const unsigned long long*>(
                                                               static_cast<const void*>(peers->rank_counts)),
                              peers->num_ranks, peers->rank};
    return from_cuda(ep::launch_publish_counts(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status_t ep_dispatch_peers(const void* x, int32_t hidden, const ep_routing_desc_t* routing,
                              const ep_layout_t* layout, const ep_rank_layout_t* rank_layout,
                              const float* topk_weights, const ep_peers_t* peers, ep_stream_t stream)
{
    CallRange range_("ep_dispatch_peers");
    ep_status_t st = check_rank_call(routing, layout, rank_layout);
    if (st != EP_OK)
        return st;
    st = check_peers(routing, peers);
    if (st != EP_OK)
        return st;
    if (routing->routing != EP_ROUTING_TOPK || hidden < 1 || hidden % 8 != 0)
        return EP_ERR_INVALID_ARG;
    const int32_t T = routing->num_tokens;
    if (T > 0 && (x == nullptr || !aligned(x, 16)))
        return EP_ERR_INVALID_ARG;
    if (peers->recv_topk_weights != nullptr && ((T > 0 && topk_weights == nullptr) || !aligned(topk_weights, 4)))
        return EP_ERR_INVALID_ARG;
    ep::RankDispatchLaunch a{x,
                             T,
                             hidden,
                             routing->num_topk,
                             routing->num_experts,
                             routing->num_ranks,
                             routing->topk_idx,
                             topk_weights,
                             rank_layout->rank_row,
                             peers->capacity,
                             nullptr,
                             nullptr,
                             nullptr,
                             nullptr,
                             ep::error_word(layout->workspace),
                             peer_tables(peers, rank_layout)};
    return from_cuda(ep::launch_rank_dispatch(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status_t ep_combine_peers(int32_t hidden, const ep_routing_desc_t* routing, const ep_layout_t* layout,
                             const ep_rank_layout_t* rank_layout, const ep_peers_t* peers, void* out,
                             ep_dtype_t out_dtype, ep_stream_t stream)
{
    CallRange range_("ep_combine_peers");
    ep_status_t st = check_rank_call(routing, layout, rank_layout);
    if (st != EP_OK)
        return st;
    st = check_peers(routing, peers);
    if (st != EP_OK)
        return st;
    if (hidden < 1 || hidden % 8 != 0 || (out_dtype != EP_BF16 && out_dtype != EP_FP32))
        return EP_ERR_INVALID_ARG;
    const int32_t T = routing->num_tokens;
    if (T > 0 && (out == nullptr || !aligned(out, 16)))
        return EP_ERR_INVALID_ARG;
    if (T == 0)
        return EP_OK;
    ep::RankCombineLaunch a{nullptr,
                            T,
                            hidden,
                            routing->num_ranks,
                            peers->capacity,
                            rank_layout->rank_row,
                            out,
                            static_cast<int32_t>(out_dtype),
                            ep::error_word(layout->workspace),
                            peer_tables(peers, rank_layout)};
    return from_cuda(ep::launch_rank_combine(a, reinterpret_cast<cudaStream_t>(stream)));
}

ep_status_t ep_get_device_error(const ep_layout_t* layout, uint32_t* flags, int clear, ep_stream_t stream)
{
    CallRange range_("ep_get_device_error");
    if (layout == nullptr || layout->workspace == nullptr || !aligned(layout->workspace, 256) ||
        layout->workspace_bytes < kWorkspaceHeaderBytes)
        return EP_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, layout->workspace, sizeof(word), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess && clear)
        e = cudaMemsetAsync(layout->workspace, 0, sizeof(uint32_t), s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return EP_ERR_CUDA;
    if (flags != nullptr)
        *flags = word;
    if (word & EP_DEVERR_BAD_INDEX)
        return EP_ERR_BAD_INDEX;
    if (word & EP_DEVERR_OVERFLOW)
        return EP_ERR_OVERFLOW;
    if (word & EP_DEVERR_TIMEOUT)
        return EP_ERR_TIMEOUT;
    return EP_OK;
}

const char* ep_status_string(ep_status_t status)
{
    switch (status) {
    case EP_OK:
        return "ok";
    case EP_ERR_INVALID_ARG:
        return "invalid argument";
    case EP_ERR_BAD_INDEX:
        return "routing index out of range";
    case EP_ERR_OVERFLOW:
        return "destination row beyond the buffer";
    case EP_ERR_WORKSPACE:
        return "workspace missing, misaligned or too small";
    case EP_ERR_CUDA:
        return "CUDA runtime error";
    case EP_ERR_UNSUPPORTED:
        return "unsupported configuration";
    case EP_ERR_TIMEOUT:
        return "device wait timed out";
    }
    return "unknown status";
}

int ep_version(void)
{
    return EP_ABI_VERSION;
}

} // extern "C"
