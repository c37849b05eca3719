/*
 * A plain C consumer of the library's C ABI (include/ep.h): no Python, no
 * PyTorch.  Built by tests/test_c_consumer.py with gcc against the header
 * and linked against libep_b200.so.
 *
 *   abi_consumer host   -- host-only calls: version, status strings,
 *                          workspace sizing and argument rejection
 *   abi_consumer gpu    -- one small token-choice layout -> dispatch ->
 *                          combine on device memory from the CUDA runtime,
 *                          then the per-rank path over peer memory with two
 *                          ranks in this process, checked on the host
 *                          against hand-computed values
 *
 * Exit status 0 on success; each failed check prints a line and exits 1.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "ep.h"

#include <cuda_runtime_api.h>

#define H2D cudaMemcpyHostToDevice
#define D2H cudaMemcpyDeviceToHost

#define CHECK(cond, what)                                                                                   \
    do {                                                                                                    \
        if (!(cond)) {                                                                                      \
            printf("FAIL %s (line %d)\n", what, __LINE__);                                                  \
            exit(1);                                                                                        \
        }                                                                                                   \
    } while (0)

static int host_mode(void)
{
    CHECK(ep_version() == EP_ABI_VERSION, "version");
    CHECK(strcmp(ep_status_string(EP_OK), "") != 0, "status string");
    ep_routing_desc_t r;
    memset(&r, 0, sizeof r);
    r.routing = EP_ROUTING_TOPK;
    r.topk_idx = (const int64_t*)(uintptr_t)0x1000;
    r.num_tokens = 16;
    r.num_topk = 2;
    r.num_experts = 8;
    r.num_ranks = 2;
    size_t ws = ep_workspace_bytes(&r);
    CHECK(ws >= 256 && ws % 256 == 0, "workspace bytes");
    r.num_ranks = 3; /* 8 experts do not split into 3 ranks */
    CHECK(ep_workspace_bytes(&r) == 0, "workspace bytes rejects E % R");
    ep_layout_t l;
    memset(&l, 0, sizeof l);
    CHECK(ep_get_layout(&r, &l, NULL) == EP_ERR_INVALID_ARG, "layout rejects bad routing");
    r.num_ranks = 2;
    CHECK(ep_get_layout(&r, &l, NULL) == EP_ERR_WORKSPACE, "layout rejects a missing workspace");
    printf("host ok\n");
    return 0;
}

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static void* peer_buffer(size_t bytes)
{
    void* p = NULL;
    unsigned char handle[EP_IPC_HANDLE_BYTES];
    CHECK(ep_peer_alloc(bytes, &p, handle) == EP_OK && p != NULL, "peer alloc");
    CHECK(cudaMemset(p, 0xFF, bytes) == 0, "peer buffer fill");
    return p;
}

static void* device_table(void* const* host, int n)
{
    void* d = NULL;
    CHECK(cudaMalloc(&d, n * sizeof(void*)) == 0 && cudaMemcpy(d, host, n * sizeof(void*), H2D) == 0, "table");
    return d;
}

/* The peer path with its two ranks in this process: both ranks hold the
 * routing of gpu_mode (tokens 0..3 go to ranks {0,1}, {0}, {0,1}, {1}), so
 * every rank receives 3 rows from each source, source 0's first.  The
 * partial rows are the received rows themselves, so out[t] = (number of
 * ranks of t) * (t + 1): 2, 2, 6, 4. */
static void peer_mode(const void* d_x, const ep_routing_desc_t* r, const ep_layout_t* l, int T, int H, int K)
{
    enum { R = 2, CAP = 6 };
    int32_t *d_roff, *d_rrow;
    CHECK(cudaMalloc((void**)&d_roff, (R + 1) * 4) == 0 && cudaMalloc((void**)&d_rrow, T * R * 4) == 0, "cudaMalloc");
    ep_rank_layout_t rl = {d_roff, d_rrow};
    CHECK(ep_get_rank_layout(r, l, &rl, NULL) == EP_OK, "rank layout");
    void *rx[R], *y[R], *ridx[R], *rsrc[R], *cnt[R];
    for (int j = 0; j < R; ++j) {
        rx[j] = peer_buffer(CAP * H * 2);
        y[j] = peer_buffer(CAP * H * 2);
        ridx[j] = peer_buffer(CAP * K * 8);
        rsrc[j] = peer_buffer(CAP * 4);
        cnt[j] = peer_buffer(R * R * 4);
    }
    ep_peers_t p[R];
    for (int me = 0; me < R; ++me) {
        memset(&p[me], 0, sizeof p[me]);
        p[me].num_ranks = R;
        p[me].rank = me;
        p[me].capacity = CAP;
        p[me].recv_x = (void* const*)device_table(rx, R);
        p[me].recv_topk_idx = (int64_t* const*)device_table(ridx, R);
        p[me].recv_src = (int32_t* const*)device_table(rsrc, R);
        p[me].y = (const void* const*)device_table(y, R);
        p[me].rank_counts = (int32_t* const*)device_table(cnt, R);
    }
    for (int me = 0; me < R; ++me)
        CHECK(ep_peer_publish_counts(r, l, &p[me], NULL) == EP_OK, "publish counts");
    for (int me = 0; me < R; ++me)
        CHECK(ep_dispatch_peers(d_x, H, r, l, &rl, NULL, &p[me], NULL) == EP_OK, "dispatch peers");
    const float want_row[R][CAP] = {{1, 2, 3, 1, 2, 3}, {1, 3, 4, 1, 3, 4}};
    const int32_t want_src[R][CAP] = {{0, 1, 2, 0, 1, 2}, {0, 2, 3, 0, 2, 3}};
    for (int j = 0; j < R; ++j) {
        uint16_t rows[CAP * 8];
        int32_t src[CAP], counts[R * R];
        int64_t entries[2];
        CHECK(cudaMemcpy(rows, rx[j], sizeof rows, D2H) == 0 && cudaMemcpy(src, rsrc[j], sizeof src, D2H) == 0 &&
                  cudaMemcpy(counts, cnt[j], sizeof counts, D2H) == 0 &&
                  cudaMemcpy(entries, ridx[j], sizeof entries, D2H) == 0,
              "copy peer buffers");
        for (int i = 0; i < R * R; ++i)
            CHECK(counts[i] == 3, "every rank holds every rank's counts");
        for (int row = 0; row < CAP; ++row) {
            CHECK(bf16_to_f32(rows[row * H]) == want_row[j][row], "received row");
            CHECK(src[row] == want_src[j][row], "received source token");
        }
        /* token 0 (experts 0 and 3): rank 0 sees (0, -1), rank 1 sees (-1, 1) */
        CHECK(entries[0] == (j == 0 ? 0 : -1) && entries[1] == (j == 0 ? -1 : 1), "received top-k entries");
        CHECK(cudaMemcpy(y[j], rx[j], CAP * H * 2, cudaMemcpyDeviceToDevice) == 0, "partial rows");
    }
    const float want_out[4] = {2.0f, 2.0f, 6.0f, 4.0f};
    float* d_out;
    CHECK(cudaMalloc((void**)&d_out, T * H * 4) == 0, "cudaMalloc");
    for (int me = 0; me < R; ++me) {
        float out[4 * 8];
        CHECK(ep_combine_peers(H, r, l, &rl, &p[me], d_out, EP_FP32, NULL) == EP_OK, "combine peers");
        CHECK(cudaMemcpy(out, d_out, sizeof out, D2H) == 0, "copy out");
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h)
                CHECK(out[t * H + h] == want_out[t], "peer combined value");
    }
    uint32_t flags = 1;
    CHECK(ep_get_device_error(l, &flags, 1, NULL) == EP_OK && flags == 0, "device error word after the peer path");
    for (int me = 0; me < R; ++me) {
        cudaFree((void*)p[me].recv_x), cudaFree((void*)p[me].recv_topk_idx), cudaFree((void*)p[me].recv_src);
        cudaFree((void*)p[me].y), cudaFree((void*)p[me].rank_counts);
    }
    for (int j = 0; j < R; ++j)
        CHECK(ep_peer_free(rx[j]) == EP_OK && ep_peer_free(y[j]) == EP_OK && ep_peer_free(ridx[j]) == EP_OK &&
                  ep_peer_free(rsrc[j]) == EP_OK && ep_peer_free(cnt[j]) == EP_OK,
              "peer free");
    cudaFree(d_out), cudaFree(d_roff), cudaFree(d_rrow);
}

static int gpu_mode(void)
{
    /* 4 tokens, hidden 8, 4 experts in 2 ranks, top-2; x[t][h] = t + 1 */
    enum { T = 4, H = 8, E = 4, R = 2, K = 2 };
    const int64_t idx[T * K] = {0, 3, 1, -1, 3, 0, 2, 2};
    const float w[T * K] = {0.25f, 0.75f, 1.0f, 0.0f, 0.5f, 0.5f, 2.0f, 3.0f};
    uint16_t x[T * H];
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            float f = (float)(t + 1);
            uint32_t u;
            memcpy(&u, &f, 4);
            x[t * H + h] = (uint16_t)(u >> 16); /* small integers are exact in bf16 */
        }
    void *d_idx, *d_w, *d_x, *d_recv, *d_out, *d_ws;
    int32_t *d_cnt, *d_off, *d_rcnt, *d_slot;
    uint8_t* d_inr;
    ep_routing_desc_t r;
    memset(&r, 0, sizeof r);
    r.routing = EP_ROUTING_TOPK;
    r.num_tokens = T;
    r.num_topk = K;
    r.num_experts = E;
    r.num_ranks = R;
    CHECK(cudaMalloc(&d_idx, sizeof idx) == 0 && cudaMalloc(&d_w, sizeof w) == 0 && cudaMalloc(&d_x, sizeof x) == 0,
          "cudaMalloc");
    r.topk_idx = (const int64_t*)d_idx;
    size_t ws = ep_workspace_bytes(&r);
    CHECK(ws >= 256, "workspace bytes");
    CHECK(cudaMalloc(&d_recv, T * K * H * 2) == 0 && cudaMalloc(&d_out, T * H * 4) == 0 && cudaMalloc(&d_ws, ws) == 0,
          "cudaMalloc");
    CHECK(cudaMalloc((void**)&d_cnt, E * 4) == 0 && cudaMalloc((void**)&d_off, (E + 1) * 4) == 0 &&
              cudaMalloc((void**)&d_rcnt, R * 4) == 0 && cudaMalloc((void**)&d_slot, T * K * 4) == 0 &&
              cudaMalloc((void**)&d_inr, T * R) == 0,
          "cudaMalloc");
    CHECK(cudaMemcpy(d_idx, idx, sizeof idx, H2D) == 0 && cudaMemcpy(d_w, w, sizeof w, H2D) == 0 &&
              cudaMemcpy(d_x, x, sizeof x, H2D) == 0,
          "copy in");
    CHECK(ep_workspace_init(d_ws, ws, NULL) == EP_OK, "workspace init");
    ep_layout_t l;
    memset(&l, 0, sizeof l);
    l.num_tokens_per_expert = d_cnt;
    l.expert_offsets = d_off;
    l.num_tokens_per_rank = d_rcnt;
    l.is_token_in_rank = d_inr;
    l.slot = d_slot;
    l.workspace = d_ws;
    l.workspace_bytes = ws;
    CHECK(ep_get_layout(&r, &l, NULL) == EP_OK, "layout");
    /* the same layout again, reporting the routed-pair count to the host */
    int32_t num_valid = -1;
    l.num_valid_host = &num_valid;
    CHECK(ep_get_layout(&r, &l, NULL) == EP_OK, "layout with num_valid_host");
    CHECK(num_valid == 7, "num_valid_host holds the routed pairs");
    l.num_valid_host = NULL;
    CHECK(ep_dispatch(d_x, H, &r, &l, EP_LAYOUT_COMPACT, 0, T * K, EP_BF16, NULL, d_recv, NULL, NULL, NULL, NULL) ==
              EP_OK,
          "dispatch");
    CHECK(ep_combine(d_recv, H, T * K, &r, &l, EP_LAYOUT_COMPACT, 0, (const float*)d_w, d_out, EP_FP32, NULL) == EP_OK,
          "combine");
    uint32_t flags = 1;
    CHECK(ep_get_device_error(&l, &flags, 1, NULL) == EP_OK && flags == 0, "device error word");
    int32_t cnt[E], off[E + 1], slot[T * K];
    float out[T * H];
    uint16_t recv[T * K * H];
    CHECK(cudaMemcpy(cnt, d_cnt, sizeof cnt, D2H) == 0 && cudaMemcpy(off, d_off, sizeof off, D2H) == 0 &&
              cudaMemcpy(slot, d_slot, sizeof slot, D2H) == 0 && cudaMemcpy(out, d_out, sizeof out, D2H) == 0 &&
              cudaMemcpy(recv, d_recv, sizeof recv, D2H) == 0,
          "copy out");
    /* expert 0: (0,0), (2,1); expert 1: (1,0); expert 2: (3,0), (3,1); expert 3: (0,1), (2,0) */
    const int32_t want_cnt[E] = {2, 1, 2, 2}, want_off[E + 1] = {0, 2, 3, 5, 7};
    const int32_t want_slot[T * K] = {0, 0, 0, -1, 1, 1, 0, 1};
    for (int e = 0; e < E; ++e)
        CHECK(cnt[e] == want_cnt[e] && off[e] == want_off[e], "counts / offsets");
    CHECK(off[E] == 7, "total");
    for (int i = 0; i < T * K; ++i)
        CHECK(slot[i] == want_slot[i], "slots");
    /* row 3 (expert 2, slot 0) holds token 3 */
    CHECK(bf16_to_f32(recv[3 * H]) == 4.0f, "dispatched row");
    /* out[t] = (sum of valid weights) * (t + 1): 1, 2, 3, 20 (token 3: 2*4 + 3*4) */
    const float want_out[T] = {1.0f, 2.0f, 3.0f, 20.0f};
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h)
            CHECK(out[t * H + h] == want_out[t], "combined value");
    peer_mode(d_x, &r, &l, T, H, K);
    cudaDeviceSynchronize();
    cudaFree(d_idx), cudaFree(d_w), cudaFree(d_x), cudaFree(d_recv), cudaFree(d_out), cudaFree(d_ws);
    cudaFree(d_cnt), cudaFree(d_off), cudaFree(d_rcnt), cudaFree(d_slot), cudaFree(d_inr);
    printf("gpu ok\n");
    return 0;
}

int main(int argc, char** argv)
{
    if (argc > 1 && strcmp(argv[1], "gpu") == 0)
        return gpu_mode();
    return host_mode();
}
