// Host-side internals of libep: the buffer struct and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"

struct ep_buffer {
    ep_config_t cfg;
    int64_t n_max;   // R * T_max tokens
    int64_t m_max;   // R * T_max * K receive rows
    int64_t nc_max;  // chunk capacity of the layout scratch
    int device;
    int sm_count;
    int last_T;      // T of the last ep_get_layout (-1 = none)

    // layout arrays (device)
    int32_t* topk_idx;
    float* topk_w;
    uint8_t* is_token_in_rank;
    int32_t* num_tokens_per_rank;
    int32_t* cnt;
    int32_t* num_tokens_per_expert;
    int32_t* expert_off;
    int32_t* rank_off;
    int32_t* src_off;
    int32_t* dst_row;
    // layout scratch (device): barrier words, per-chunk counts and prefixes
    int32_t* scratch;
    // deduplicated receive (EP_FLAG_DEDUP; device)
    int64_t d_max;  // R * T_max * min(R, K) rows
    int32_t* tok_row;       // [N_max, R]
    int32_t* rank_row_off;  // [R + 1]
    int32_t* rank_src_off;  // [R, R]
    void* dd_x;             // [d_max, H] bf16 or e4m3
    float* dd_scale;        // [d_max, H/128] (FP8)
    int32_t* dd_src;        // [d_max]
    int32_t* dd_topk_idx;   // [d_max, K]
    float* dd_topk_w;       // [d_max, K]
    uint16_t* partial;      // [d_max, H] bf16
    // one rank per GPU (EP_FLAG_SHARD; device unless stated)
    int32_t* cnt_all;     // [R, E]: every rank's count row, filled by the caller's all-gather
    uint8_t* dst_rank;    // [T_max, K]: destination rank of each slot
    int32_t* recv_count;  // [E/R]: receive rows of each of this rank's experts
    int32_t* recv_off;    // [E/R + 1]: their exclusive prefix; recv_off[E/R] = rows received
    int shard_rank;       // host: rank of the last ep_shard_layout (-1 = none)
    bool placed;          // host: ep_shard_place ran after the last ep_shard_layout
    uint32_t* err;  // device error word
    // receive buffers (device)
    void* recv_x;
    float* recv_scale;
    int32_t* recv_src;
    float* recv_w;
};

namespace ep {

// Sets the message ep_last_error_message() returns on this host thread.
void set_last_error(const char* msg);

// Layout grid cap (CTAs = chunks) and the control words at the head of the
// layout scratch (two barrier counters, zero between launches).
constexpr int kMaxLayoutCtas = 1024;
// Ranks a peer-pointer table holds (the num_ranks limit).
constexpr int kMaxPeers = 32;
constexpr int kLayoutControlInts = 64;

struct LayoutArgs {
    int T;
    const float* logits;
    const int32_t* in_idx;
    const float* in_w;
    int route;
    uint64_t mask_seed;
    uint64_t mask_threshold;  // in [0, 2^32]
    int64_t m_max;            // rows the receive side holds (bound check)
    int low_latency;          // fixed (expert, source rank) regions of T_max rows
    int T_max;                // region size in low-latency mode
    int S = 0;                        // source ranks routed (0 = all R); 1 = one rank's own tokens
    int64_t g_base = 0;               // global id of the first token (slot-mask hash)
    int32_t* tok_row = nullptr;       // dedup outputs (NULL: not wanted)
    int32_t* rank_row_off = nullptr;
    int32_t* rank_src_off = nullptr;
};

// int32 entries of layout scratch for a grid of at most max_ctas CTAs:
// control words, per-chunk counts [E+R][max_ctas], column totals [E+R].
int64_t layout_scratch_ints(const ep_config_t& c, int max_ctas);

// The layout kernel on caller-given outputs and scratch
// (layout_scratch_ints(c, max_ctas) ints whose control words are zero).
cudaError_t launch_layout_raw(const ep_config_t& c, const LayoutArgs& a, const ep_layout_t& out,
                              int32_t* scratch, int max_ctas, uint32_t* err, cudaStream_t stream);

cudaError_t launch_layout(const ep_buffer& b, const LayoutArgs& a, cudaStream_t stream);

// Runs the layout's grid barrier with an unreachable target on 2 CTAs
// (words: 4 device uint32; [2] receives the error bits).
cudaError_t launch_barrier_timeout_selftest(uint32_t* words, unsigned long long limit_ns, cudaStream_t stream);
// The combine pipeline's mbarrier wait on a phase that never completes; sets
// *gave_up = 1 and EP_DEVERR_TIMEOUT in *err when the wait ends unmet.
cudaError_t launch_mbarrier_timeout_selftest(uint32_t* err, uint32_t* gave_up, unsigned long long limit_ns,
                                             cudaStream_t stream);
cudaError_t launch_dispatch(const ep_buffer& b, int T, const void* x, cudaStream_t stream);
cudaError_t launch_dispatch_dedup(const ep_buffer& b, int T, const void* x, cudaStream_t stream);
cudaError_t launch_permute(const ep_buffer& b, int T, cudaStream_t stream);
cudaError_t launch_local_reduce(const ep_buffer& b, int T, const void* y, const float* y_scale, cudaStream_t stream);
cudaError_t launch_combine_dedup(const ep_buffer& b, int T, void* out, cudaStream_t stream);
cudaError_t launch_combine(const ep_buffer& b, int T, const void* y, const float* y_scale, void* out,
                           cudaStream_t stream);

// One rank per GPU (EP_FLAG_SHARD): placement from the gathered count rows,
// then dispatch into / combine from every rank's arrays through tables of
// num_ranks device pointers.
cudaError_t launch_shard_place(const ep_buffer& b, int rank, int T, cudaStream_t stream);
cudaError_t launch_shard_dispatch(const ep_buffer& b, int rank, int T, const void* x, void* const* peer_x,
                                  float* const* peer_scale, int32_t* const* peer_src, float* const* peer_w,
                                  cudaStream_t stream);
cudaError_t launch_shard_combine(const ep_buffer& b, int T, const void* const* peer_y,
                                 const float* const* peer_scale, void* out, cudaStream_t stream);

}  // namespace ep
