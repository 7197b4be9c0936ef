// Placement for one rank per GPU (sm_100a).
//
// In a one-process-per-GPU deployment each rank routes only its own T tokens
// ("DeepEP：年度总结中的计算通信重叠摘记", §节点内通信: the intranode kernels
// exchange the counts first, then every rank writes its tokens straight into
// the receivers' buffers). The layout kernel, run over the rank's own tokens,
// leaves each slot at its rank-local row: the rank's own exclusive expert
// offset plus the slot's position among the rank's earlier slots of that
// expert. Once the caller has all-gathered the R count rows into cnt_all,
// this kernel moves every slot to its row on the destination rank d = e / L:
//
//   row = (expert_off[e] - expert_off[d*L])   expert e's block on rank d
//       + src_off[e][s]                        earlier source ranks' rows of e
//       + (local row - local expert_off[e])    position within rank s's rows of e
//
// where expert_off and src_off are the single-buffer layout's exclusive sums
// over every rank's counts. Rank d's receive rows are therefore exactly rows
// [rank_off[d], rank_off[d+1]) of the single-buffer layout, shifted to start
// at 0.
//
// Every CTA derives the per-expert shift from cnt_all (R*E int32 from L2),
// then maps a grid-stride range of the rank's T*K slots. CTA 0 also writes
// the rank's own receive counts: rows per local expert and their prefix.
// cnt_all is the caller's data: a negative count, or a total above the
// receive capacity, sets EP_DEVERR_ROW_BOUNDS and leaves every slot at -1.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace ep {
namespace {

constexpr int kPlaceThreads = 256;

struct PlaceParams {
    int R, E, L, rank;
    int64_t slots;              // T * K
    const int32_t* cnt_all;     // [R, E]
    const int32_t* eoff_local;  // [E + 1]: the rank-local exclusive expert offsets
    const int32_t* topk_idx;    // [T, K]
    int32_t* dst_row;           // [T, K]: rank-local rows in, destination rows out
    uint8_t* dst_rank;          // [T, K]
    int32_t* recv_count;        // [L]
    int32_t* recv_off;          // [L + 1]
    int64_t m_max;
    uint32_t* err;
};

__global__ void __launch_bounds__(kPlaceThreads) shard_place_kernel(PlaceParams p) {
    extern __shared__ int sm[];
    int* col = sm;             // [E]: rows of expert e over all source ranks
    int* pre = col + p.E;      // [E]: rows of e from ranks before this one
    int* eo = pre + p.E;       // [E + 1]: exclusive prefix of col
    int* shift = eo + p.E + 1; // [E]
    __shared__ int warp_tot[33];
    __shared__ unsigned long long s_total;
    __shared__ int s_bad;
    if (threadIdx.x == 0) {
        s_total = 0ull;
        s_bad = 0;
    }
    __syncthreads();
    // cnt_all comes from the caller's exchange: its total must fit the
    // receive buffer (so the int32 prefix sums below cannot overflow)
    unsigned long long mine = 0ull;
    for (int e = threadIdx.x; e < p.E; e += kPlaceThreads) {
        int v[kMaxPeers];
#pragma unroll
        for (int s = 0; s < kMaxPeers; ++s)  // all loads in flight at once
            v[s] = (s < p.R) ? __ldg(p.cnt_all + (int64_t)s * p.E + e) : 0;
        long long tot = 0, before = 0;
        bool neg = false;
#pragma unroll
        for (int s = 0; s < kMaxPeers; ++s) {
            neg = neg || v[s] < 0;
            if (s < p.rank) before += v[s];
            tot += v[s];
        }
        if (neg) s_bad = 1;
        mine += (unsigned long long)(tot < 0 ? 0 : tot);
        col[e] = (int)min(tot, (long long)p.m_max);
        pre[e] = (int)min(before, (long long)p.m_max);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(FULL, mine, off);
    if ((threadIdx.x & 31) == 0) atomicAdd(&s_total, mine);  // one shared atomic per warp
    __syncthreads();
    const bool bad = s_bad || s_total > (unsigned long long)p.m_max;
    if (bad) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_error(p.err, EP_DEVERR_ROW_BOUNDS);
        if (blockIdx.x == 0) {
            for (int j = threadIdx.x; j < p.L; j += kPlaceThreads) p.recv_count[j] = 0;
            for (int j = threadIdx.x; j <= p.L; j += kPlaceThreads) p.recv_off[j] = 0;
        }
        for (int64_t i = (int64_t)blockIdx.x * kPlaceThreads + threadIdx.x; i < p.slots;
             i += (int64_t)gridDim.x * kPlaceThreads) {
            p.dst_row[i] = -1;
            p.dst_rank[i] = 0;
        }
        return;
    }
    block_exclusive_scan(col, 1, p.E, eo, warp_tot);
    for (int e = threadIdx.x; e < p.E; e += kPlaceThreads)
        shift[e] = (eo[e] - eo[(e / p.L) * p.L]) + pre[e] - __ldg(p.eoff_local + e);
    if (blockIdx.x == 0) {
        const int e0 = p.rank * p.L;
        for (int j = threadIdx.x; j < p.L; j += kPlaceThreads) {
            p.recv_count[j] = col[e0 + j];
            p.recv_off[j] = eo[e0 + j] - eo[e0];
        }
        if (threadIdx.x == 0) p.recv_off[p.L] = eo[e0 + p.L] - eo[e0];
    }
    __syncthreads();
    for (int64_t i = (int64_t)blockIdx.x * kPlaceThreads + threadIdx.x; i < p.slots;
         i += (int64_t)gridDim.x * kPlaceThreads) {
        const int e = p.topk_idx[i];
        int32_t row = -1;
        int d = 0;
        if (e >= 0 && e < p.E) {
            const int64_t r = (int64_t)p.dst_row[i] + shift[e];
            d = e / p.L;
            if (r >= 0 && r < p.m_max) row = (int32_t)r;
            else set_error(p.err, EP_DEVERR_ROW_BOUNDS);
        }
        p.dst_row[i] = row;
        p.dst_rank[i] = (uint8_t)d;
    }
}

}  // namespace

cudaError_t launch_shard_place(const ep_buffer& b, int rank, int T, cudaStream_t st) {
    const ep_config_t& c = b.cfg;
    PlaceParams p{};
    p.R = c.num_ranks;
    p.E = c.num_experts;
    p.L = c.num_experts / c.num_ranks;
    p.rank = rank;
    p.slots = (int64_t)T * c.topk;
    p.cnt_all = b.cnt_all;
    p.eoff_local = b.expert_off;
    p.topk_idx = b.topk_idx;
    p.dst_row = b.dst_row;
    p.dst_rank = b.dst_rank;
    p.recv_count = b.recv_count;
    p.recv_off = b.recv_off;
    p.m_max = b.m_max;
    p.err = b.err;
    int64_t grid = (p.slots + kPlaceThreads - 1) / kPlaceThreads;
    if (grid > 2 * b.sm_count) grid = 2 * b.sm_count;
    if (grid < 1) grid = 1;  // CTA 0 still writes the receive counts
    const size_t smem = sizeof(int) * (4 * (size_t)p.E + 1);
    shard_place_kernel<<<(unsigned)grid, kPlaceThreads, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
