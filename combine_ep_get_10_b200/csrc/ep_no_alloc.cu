// ep_no_alloc.cu -- ep_get_layout_no_alloc: the layout entry point for
// callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they need a layout: a plugin inside an inference server or framework that
// only hands the plugin its input and output tensors and owns every other
// byte of device memory, or a latency-critical decode loop where an
// allocation could synchronise the device.  ep_get_layout needs a
// caller-provided workspace (the expert-choice layout keeps per-token
// counters and an unordered slot list there); this variant takes its
// scratch from a fixed-size array in the library's own device memory
// instead.
//
// The array is a file-scope __device__ object: every GPU that loads the
// library holds kStaticWorkspaceBytes of it until the process exits.  Its
// device address is looked up once per device (cudaGetSymbolAddress with that
// device current); host code must never pass the symbol itself to a kernel.
// All calls share the one array, so calls whose kernels overlap on the GPU
// (two streams, or two host threads) race on it and must be serialised by
// the caller.  Every call zeroes the array's 256-byte header first (the
// error word and the grid barrier's arrival and generation words), so a call
// whose barrier wait ran out leaves nothing behind for the next one.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "ep.h"
#include "ep_internal.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = EP_STATIC_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::mutex g_setup_mutex;
void* g_static_ptr[kMaxDevices] = {};

// Device address of g_static_workspace on the current device (looked up on
// the first call for that device), or nullptr on failure.
void* static_workspace_on_current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_static_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return nullptr;
        }
        g_static_ptr[dev] = p;
    }
    return g_static_ptr[dev];
}

bool aligned4(const void* p)
{
    return (reinterpret_cast<uintptr_t>(p) & 3u) == 0;
}

} // namespace

extern "C" {

ep_status_t ep_get_layout_no_alloc(const ep_routing_desc_t* routing, const ep_layout_t* layout,
                                   uint32_t* device_error_flags, ep_stream_t stream)
{
    if (routing == nullptr || layout == nullptr)
        return EP_ERR_INVALID_ARG;
    // the ordinary argument rules, checked by ep_workspace_bytes (0 = invalid)
    const size_t need = ep_workspace_bytes(routing);
    if (need == 0)
        return EP_ERR_INVALID_ARG;
    if (need > kStaticWorkspaceBytes)
        return EP_ERR_WORKSPACE; // the problem needs more scratch than the fixed array holds
    if (device_error_flags != nullptr && !aligned4(device_error_flags))
        return EP_ERR_INVALID_ARG;
    const int32_t T = routing->num_tokens, E = routing->num_experts, R = routing->num_ranks;
    if (layout->num_tokens_per_expert == nullptr || layout->num_tokens_per_rank == nullptr ||
        !aligned4(layout->num_tokens_per_expert) || !aligned4(layout->num_tokens_per_rank))
        return EP_ERR_INVALID_ARG;
    if (T > 0 && layout->is_token_in_rank == nullptr)
        return EP_ERR_INVALID_ARG;

    const bool topk = routing->routing == EP_ROUTING_TOPK;
    if (topk) {
        if (E > ep::kMaxTopkLayoutExperts)
            return EP_ERR_UNSUPPORTED;
        if (layout->expert_offsets == nullptr || !aligned4(layout->expert_offsets))
            return EP_ERR_INVALID_ARG;
        if (T > 0 && (layout->slot == nullptr || !aligned4(layout->slot)))
            return EP_ERR_INVALID_ARG;
    } else if (layout->token_offsets == nullptr || layout->token_slots == nullptr ||
               !aligned4(layout->token_offsets) || !aligned4(layout->token_slots)) {
        return EP_ERR_INVALID_ARG;
    }

    void* ws = static_workspace_on_current_device();
    if (ws == nullptr)
        return EP_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the header (error word, grid-barrier words) starts every call at zero,
    // and so does the caller's error word when one is given (the kernels
    // report there instead of in the header, where nobody reads it)
    if (cudaMemsetAsync(ws, 0, ep::kWorkspaceHeaderBytes, s) != cudaSuccess)
        return EP_ERR_CUDA;
    uint32_t* err = device_error_flags != nullptr ? device_error_flags : ep::error_word(ws);
    if (device_error_flags != nullptr && cudaMemsetAsync(err, 0, sizeof(uint32_t), s) != cudaSuccess)
        return EP_ERR_CUDA;

    if (topk) {
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
                             ws};
        if (ep::launch_tc_layout(a, s) != cudaSuccess)
            return EP_ERR_CUDA;
        return ep::report_num_valid(routing, layout, s);
    }
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
                         ws,
                         err};
    if (ep::launch_ec_layout(a, s) != cudaSuccess)
        return EP_ERR_CUDA;
    return ep::report_num_valid(routing, layout, s);
}

} // extern "C"
