// ep_internal.h -- host-side launch interfaces between the C-ABI layer
// (ep_api.cu) and the kernel files.  Arguments reaching these launchers have
// been validated by ep_api.cu.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "ep.h"

namespace ep {

constexpr size_t kWorkspaceHeaderBytes = 256; // error word + reserved
constexpr int kMaxTopkLayoutExperts = 1024;   // token-choice layout keeps E counters per warp
constexpr int kMaxQuantHidden = 32768;        // quantising dispatch stages a row (2H + H bytes) in shared memory

inline uint32_t* error_word(void* workspace)
{
    return static_cast<uint32_t*>(workspace);
}

// When layout->num_valid_host is set: copy the routing's filled-row count
// (expert_offsets[E] or token_offsets[T]) to it and synchronise the stream.
ep_status_t report_num_valid(const ep_routing_desc_t* routing, const ep_layout_t* layout, cudaStream_t stream);

// ------------------------------------------------------------------ layout
struct TcLayoutLaunch {
    const int64_t* topk_idx;
    int32_t T, K, E, R;
    int32_t* counts;
    int32_t* offsets;
    int32_t* rank_counts;
    uint8_t* in_rank;
    int32_t* slot;
    uint32_t* err;
    void* workspace; // header + per-CTA totals of the grid-wide kernel
    // let the kernel launched next start at once (a dispatch of the same call
    // that reads the layout's results through L2 only after griddepcontrol.wait)
    int32_t trigger_dependents;
};
size_t tc_layout_workspace_bytes(int64_t E);
cudaError_t launch_tc_layout(const TcLayoutLaunch& a, cudaStream_t stream);

struct EcLayoutLaunch {
    const int32_t* token_indices;
    int32_t T, E, C, R;
    int32_t* counts;
    int32_t* rank_counts;
    uint8_t* in_rank;
    int32_t* token_offsets;
    int32_t* token_slots;
    void* workspace; // header, then tmask[T], fill[T], scratch[E*C]
    uint32_t* err;
    int32_t trigger_dependents; // as for TcLayoutLaunch
};
size_t ec_layout_workspace_bytes(int64_t T, int64_t E, int64_t C);
cudaError_t launch_ec_layout(const EcLayoutLaunch& a, cudaStream_t stream);

struct RankLayoutLaunch {
    const uint8_t* in_rank;
    const int32_t* rank_counts;
    int32_t T, R;
    int32_t* rank_offsets;
    int32_t* rank_row;
    int32_t trigger_dependents; // as for TcLayoutLaunch
};
cudaError_t launch_rank_layout(const RankLayoutLaunch& a, cudaStream_t stream);

// --------------------------------------------------------------- dispatch
// Token-choice destination rows (shared by dispatch and combine).
struct TcRows {
    const int64_t* topk_idx;
    const int32_t* slot;
    const int32_t* offsets;
    int32_t K, E, mode, max_tokens;
    int64_t num_rows;
};

struct TcDispatchLaunch {
    const void* x;
    int32_t T, H;
    TcRows rows;
    int32_t out_dtype;
    const float* topk_weights;
    void* recv_x;
    void* recv_scales;
    int32_t* recv_src;
    float* recv_weights;
    uint32_t* err;
    int32_t early_load; // 1 only right after this library's own layout launch on the stream
};
cudaError_t launch_tc_dispatch(const TcDispatchLaunch& a, cudaStream_t stream);

// Fused low-latency dispatch: the token-choice layout and a padded dispatch
// (bf16 or any quantised format) in one launch, for small batches.
struct LowLatencyLaunch {
    const void* x;
    int32_t T, H, K, E, R, max_tokens;
    const int64_t* topk_idx;
    int32_t out_dtype;
    const float* topk_weights;
    void* recv_x;
    void* recv_scales;
    int32_t* recv_src;
    float* recv_weights;
    int32_t* slot;
    uint8_t* in_rank;
    int32_t* counts;
    int32_t* offsets;
    int32_t* rank_counts;
    uint32_t* err;
};
bool ll_fusable(int32_t T, int32_t K, int32_t E, int32_t H, int out_dtype);
cudaError_t launch_ll_dispatch(const LowLatencyLaunch& a, cudaStream_t stream);

struct EcDispatchLaunch {
    const void* x;
    int32_t T, H, E, C;
    const int32_t* token_indices;
    void* recv_x;
    uint32_t* err;
    int32_t early_load; // the layout kernel was launched just before by the library (see launch_pdl)
};
cudaError_t launch_ec_dispatch(const EcDispatchLaunch& a, cudaStream_t stream);

// Per rank over peer memory: device tables of R addresses (rank r's buffer
// as this process reaches it) and this rank's place among the ranks.  A
// source's row for rank j lands at base(me, j) + rank_row[t, j] -
// rank_offsets[j] of rank j's buffer, base(me, j) = sum over i < me of
// rank_counts[i, j] (this rank's own copy of the counts).
struct PeerTables {
    const unsigned long long* recv_x;            // nullptr: not the peer path
    const unsigned long long* recv_topk_idx;     // or nullptr
    const unsigned long long* recv_topk_weights; // or nullptr
    const unsigned long long* recv_src;          // or nullptr
    const unsigned long long* y;
    const unsigned long long* rank_counts;
    const int32_t* rank_offsets; // this rank's rank layout
    int32_t me;
    int64_t capacity; // rows of every rank's recv_x and y
};

struct PublishCountsLaunch {
    const int32_t* num_tokens_per_rank; // [R]
    const unsigned long long* rank_counts; // table of R [R, R] matrices
    int32_t R, me;
};
cudaError_t launch_publish_counts(const PublishCountsLaunch& a, cudaStream_t stream);

struct RankDispatchLaunch {
    const void* x;
    int32_t T, H, K, E, R;
    const int64_t* topk_idx;
    const float* topk_weights;
    const int32_t* rank_row;
    int64_t num_rows;
    void* recv_x;
    int64_t* recv_topk_idx;
    float* recv_topk_weights;
    int32_t* recv_src;
    uint32_t* err;
    PeerTables peers;   // peers.recv_x != nullptr: rows go to the ranks' buffers
    int32_t early_load; // the rank layout was launched just before by the library (see launch_pdl)
};
cudaError_t launch_rank_dispatch(const RankDispatchLaunch& a, cudaStream_t stream);

// ---------------------------------------------------------------- combine
struct TcCombineLaunch {
    const void* y;
    int32_t T, H;
    TcRows rows;
    const float* topk_weights;
    void* out;
    int32_t out_dtype;
    uint32_t* err;
};
cudaError_t launch_tc_combine(const TcCombineLaunch& a, cudaStream_t stream);

struct EcCombineLaunch {
    const void* y;
    int32_t T, H;
    int64_t num_y_rows;
    const int32_t* token_offsets;
    const int32_t* token_slots;
    const float* expert_weights;
    void* out;
    int32_t out_dtype;
    uint32_t* err;
};
cudaError_t launch_ec_combine(const EcCombineLaunch& a, cudaStream_t stream);

struct RankCombineLaunch {
    const void* y;
    int32_t T, H, R;
    int64_t num_y_rows;
    const int32_t* rank_row;
    void* out;
    int32_t out_dtype;
    uint32_t* err;
    PeerTables peers; // peers.y != nullptr: rows read from the ranks' buffers
};
cudaError_t launch_rank_combine(const RankCombineLaunch& a, cudaStream_t stream);

} // namespace ep
