// Routing + layout (sm_100a). Top-K is fused with the layout that the
// dispatch needs: "DeepEP：年度总结中的计算通信重叠摘记", §节点内通信, fuses
// Top-K with the sparse communication and builds is_token_in_rank.
//
// Three stream-ordered launches, with no host sync in between:
//   A  route_count: one warp per token. It selects the top K (optionally
//      group-limited, §计算-通信重叠), applies the slot mask and writes
//      topk_idx / topk_w / is_token_in_rank. It also builds per-chunk expert
//      and rank histograms in shared memory.
//   B  chunk_scan: an exclusive scan over chunks for every expert and rank
//      column, plus the prefix at each rank's first chunk.
//   C  assign_rows: the exclusive scan over experts (expert_off). Then each
//      chunk's slots, in (token, slot) order, get consecutive rows inside
//      their expert's block via warp match/popc. Block 0 writes the small
//      global arrays.
// A chunk is a run of consecutive tokens of one source rank. Chunks are in
// global token order, so scanning chunks in order places rows in (expert,
// source rank, token, slot) order.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ep {
namespace {

constexpr int kRouteWarps = 8;  // warps (tokens in flight) per route_count block
constexpr int kAssignThreads = 256;

struct LayoutParams {
    int R, T, E, K, L, G, KG;
    int ch, ncpr, nc, J;  // chunk tokens, chunks per rank, chunks, columns (E + R)
    int route;
    int vec_logits;  // logits rows are 16-byte aligned and E % 4 == 0
    const float* logits;
    const int32_t* in_idx;
    const float* in_w;
    uint64_t mask_seed;
    uint64_t mask_thr;
    int32_t* topk_idx;
    float* topk_w;
    uint8_t* itr;
    int32_t* chunk;
    int32_t* pref;
    int32_t *ntpr, *cnt, *ntpe, *expert_off, *rank_off, *src_off, *dst_row;
    int64_t m_max;
    uint32_t* err;
};

__device__ __forceinline__ double sigmoid_d(double x) { return 1.0 / (1.0 + exp(-x)); }

// Warp-wide top-2 of one value per lane (NEG = no value), across lanes that
// differ in the bits of `span` (a power of two): butterfly over offsets span/2..1.
__device__ __forceinline__ void top2_merge(uint32_t& a, uint32_t& b, int span) {
    for (int off = span >> 1; off > 0; off >>= 1) {
        uint32_t oa = __shfl_xor_sync(FULL, a, off);
        uint32_t ob = __shfl_xor_sync(FULL, b, off);
        // merge two sorted pairs (a >= b, oa >= ob) into the top two
        uint32_t hi = max(a, oa);
        uint32_t lo = max(min(a, oa), max(b, ob));
        a = hi;
        b = lo;
    }
}

// Routes token g with one warp. Lane k < K ends up holding slot k's expert id
// (-1 = masked) and weight.
template <int EPL>
__device__ __forceinline__ void route_token(const LayoutParams& p, int64_t g, int lane, int& my_e, float& my_w) {
    my_e = -1;
    my_w = 0.0f;
    if (p.logits == nullptr) {
        // caller-supplied top-k
        if (lane < p.K) {
            int e = p.in_idx[g * p.K + lane];
            float w = p.in_w[g * p.K + lane];
            if (e < -1 || e >= p.E) {
                set_error(p.err, EP_DEVERR_EXPERT_ID);
                e = -1;
            }
            my_e = e;
            my_w = w;
        }
    } else {
        const float* row = p.logits + g * p.E;
        float v[EPL];
        uint32_t key[EPL];
        const int e0 = lane * EPL;
        if (EPL >= 4 && p.vec_logits) {
#pragma unroll
            for (int j = 0; j < EPL; j += 4) {
                if (e0 + j < p.E) {
                    float4 q = *reinterpret_cast<const float4*>(row + e0 + j);
                    v[j] = q.x;
                    v[j + 1] = q.y;
                    v[j + 2] = q.z;
                    v[j + 3] = q.w;
                } else {
                    v[j] = v[j + 1] = v[j + 2] = v[j + 3] = 0.0f;
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < EPL; ++j) v[j] = (e0 + j < p.E) ? row[e0 + j] : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < EPL; ++j) key[j] = (e0 + j < p.E) ? order_key(v[j]) : 0u;

        if (p.route == EP_ROUTE_GROUP_SIGMOID && p.G > 1) {
            // group score = sigmoid of the group's two largest logits, summed in fp64
            const int gs = p.E / p.G;
            double score = -1.0;  // valid on lane g for g < G
            const int lpg = gs / EPL;
            if (gs % EPL == 0 && lpg <= 32 && (lpg & (lpg - 1)) == 0) {
                // each group spans lpg whole lanes
                uint32_t a = 0, b = 0;
#pragma unroll
                for (int j = 0; j < EPL; ++j) {
                    uint32_t k = key[j];
                    if (k > a) {
                        b = a;
                        a = k;
                    } else if (k > b) {
                        b = k;
                    }
                }
                top2_merge(a, b, lpg);
                double s = sigmoid_d((double)key_value(a)) + sigmoid_d((double)key_value(b));
                // group g's score sits on lane g*lpg; move it to lane g
                int src = (lane < p.G) ? lane * lpg : 0;
                double sg = __shfl_sync(FULL, s, src);
                if (lane < p.G) score = sg;
            } else {
                // generic: one warp-wide top-2 per group
                for (int grp = 0; grp < p.G; ++grp) {
                    uint32_t a = 0, b = 0;
#pragma unroll
                    for (int j = 0; j < EPL; ++j) {
                        int e = e0 + j;
                        uint32_t k = (e < p.E && e / gs == grp) ? key[j] : 0u;
                        if (k > a) {
                            b = a;
                            a = k;
                        } else if (k > b) {
                            b = k;
                        }
                    }
                    top2_merge(a, b, 32);
                    if (lane == grp)
                        score = sigmoid_d((double)key_value(a)) + sigmoid_d((double)key_value(b));
                }
            }
            // keep the KG best groups: rank = groups strictly better (ties: lower id)
            int rank = 0;
            for (int h = 0; h < p.G; ++h) {
                double sh = __shfl_sync(FULL, score, h);
                if (lane < p.G && (sh > score || (sh == score && h < lane))) ++rank;
            }
            const uint32_t kept = __ballot_sync(FULL, lane < p.G && rank < p.KG);
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                int e = e0 + j;
                if (e < p.E && !((kept >> (e / gs)) & 1u)) key[j] = 0u;
            }
        }

        // top-K: K rounds of warp argmax on (value desc, expert id asc)
        uint32_t top_key = 0;
        for (int k = 0; k < p.K; ++k) {
            uint32_t lk = 0;
            int lj = 0;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                if (key[j] > lk) {  // strict: equal keys keep the lower id
                    lk = key[j];
                    lj = j;
                }
            }
            const uint32_t wk = __reduce_max_sync(FULL, lk);
            const uint32_t cand = (lk == wk && lk != 0u) ? (0xffffffffu - (uint32_t)(e0 + lj)) : 0u;
            const uint32_t wc = __reduce_max_sync(FULL, cand);
            const int e = (int)(0xffffffffu - wc);
            if (k == 0) top_key = wk;
            if (e0 <= e && e < e0 + EPL) {
#pragma unroll
                for (int j = 0; j < EPL; ++j)
                    if (e0 + j == e) key[j] = 0u;
            }
            if (lane == k) {
                my_e = (wk != 0u) ? e : -1;
                my_w = key_value(wk);  // the logit, for the weight below
            }
        }

        // weights, fp64
        double wt = 0.0;
        if (p.route == EP_ROUTE_GROUP_SIGMOID) {
            double s = (lane < p.K && my_e >= 0) ? sigmoid_d((double)my_w) : 0.0;
            double sum = 0.0;
            for (int k = 0; k < p.K; ++k) sum += __shfl_sync(FULL, s, k);
            wt = s / sum;
        } else {
            const double mx = (double)key_value(top_key);
            double z = 0.0;
#pragma unroll
            for (int j = 0; j < EPL; ++j)
                if (e0 + j < p.E) z += exp((double)v[j] - mx);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(FULL, z, off);
            double pk = (lane < p.K && my_e >= 0) ? exp((double)my_w - mx) / z : 0.0;
            if (p.route == EP_ROUTE_SOFTMAX_RENORM) {
                double sum = 0.0;
                for (int k = 0; k < p.K; ++k) sum += __shfl_sync(FULL, pk, k);
                wt = pk / sum;
            } else {
                wt = pk;
            }
        }
        my_w = (lane < p.K) ? (float)wt : 0.0f;
    }
    // slot mask
    if (lane < p.K && p.mask_thr != 0ull) {
        uint64_t h = splitmix64(p.mask_seed ^ (uint64_t)(g * p.K + lane));
        if ((h >> 32) < p.mask_thr) {
            my_e = -1;
            my_w = 0.0f;
        }
    }
}

template <int EPL>
__global__ void __launch_bounds__(kRouteWarps * 32) route_count_kernel(LayoutParams p) {
    extern __shared__ int hist[];  // [J]
    const int c = blockIdx.x;
    const int s = c / p.ncpr;
    const int t0 = (c % p.ncpr) * p.ch;
    const int t1 = min(p.T, t0 + p.ch);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    for (int j = threadIdx.x; j < p.J; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    for (int t = t0 + warp; t < t1; t += kRouteWarps) {
        const int64_t g = (int64_t)s * p.T + t;
        int e;
        float w;
        route_token<EPL>(p, g, lane, e, w);
        if (lane < p.K) {
            p.topk_idx[g * p.K + lane] = e;
            p.topk_w[g * p.K + lane] = w;
            if (e >= 0) atomicAdd(&hist[e], 1);
        }
        const uint32_t ranks = __reduce_or_sync(FULL, (lane < p.K && e >= 0) ? (1u << (e / p.L)) : 0u);
        if (lane < p.R) {
            const uint32_t in = (ranks >> lane) & 1u;
            p.itr[g * p.R + lane] = (uint8_t)in;
            if (in) atomicAdd(&hist[p.E + lane], 1);
        }
    }
    __syncthreads();
    int32_t* out = p.chunk + (int64_t)c * p.J;
    for (int j = threadIdx.x; j < p.J; j += blockDim.x) out[j] = hist[j];
}

// Block (32 x 32): x = column within a 32-column tile, y = segment of chunks.
__global__ void __launch_bounds__(1024) chunk_scan_kernel(LayoutParams p) {
    __shared__ int part[32][33];
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int col = blockIdx.x * 32 + tx;
    const int per = (p.nc + 31) / 32;
    const int c0 = min(p.nc, ty * per);
    const int c1 = min(p.nc, c0 + per);
    int sum = 0;
    if (col < p.J) {
        for (int c = c0; c < c1; ++c) sum += p.chunk[(int64_t)c * p.J + col];
    }
    part[ty][tx] = sum;
    __syncthreads();
    {
        // warp ty scans column ty over the 32 segments
        const int lane = tx;
        const int v = part[lane][ty];
        int incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int o = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += o;
        }
        __syncthreads();
        part[lane][ty] = incl - v;  // exclusive offset of segment `lane`
        const int c2 = blockIdx.x * 32 + ty;
        if (lane == 31 && c2 < p.J) p.pref[(int64_t)c2 * (p.R + 1) + p.R] = incl;  // column total
    }
    __syncthreads();
    if (col < p.J) {
        int run = part[ty][tx];
        for (int c = c0; c < c1; ++c) {
            const int64_t i = (int64_t)c * p.J + col;
            const int x = p.chunk[i];
            p.chunk[i] = run;
            if (c % p.ncpr == 0) p.pref[(int64_t)col * (p.R + 1) + c / p.ncpr] = run;
            run += x;
        }
        if (p.nc == 0 && ty == 0)
            for (int r = 0; r < p.R; ++r) p.pref[(int64_t)col * (p.R + 1) + r] = 0;
    }
}

// Exclusive scan of n <= 4 * blockDim.x values from `in` into out[0..n],
// with out[n] = total. All threads of the block must call it.
__device__ void block_exclusive_scan(const int32_t* in, int stride, int n, int* out, int* warp_tot) {
    const int t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5, nw = blockDim.x >> 5;
    int v[4];
    int local = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = 4 * t + i;
        v[i] = (j < n) ? in[(int64_t)j * stride] : 0;
        local += v[i];
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int o = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int wv = (lane < nw) ? warp_tot[lane] : 0;
        int wi = wv;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int o = __shfl_up_sync(FULL, wi, off);
            if (lane >= off) wi += o;
        }
        if (lane < nw) warp_tot[lane] = wi - wv;
        if (lane == nw - 1) warp_tot[32] = wi;
    }
    __syncthreads();
    int run = warp_tot[warp] + incl - local;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = 4 * t + i;
        if (j < n) out[j] = run;
        run += v[i];
    }
    if (t == 0) out[n] = warp_tot[32];
    __syncthreads();
}

__global__ void __launch_bounds__(kAssignThreads) assign_rows_kernel(LayoutParams p) {
    extern __shared__ int sm[];
    int* eoff = sm;                 // [E + 1]
    int* base = sm + p.E + 1;       // [E]
    __shared__ int warp_tot[33];
    const int R1 = p.R + 1;
    // expert totals are the column totals of the first E columns
    block_exclusive_scan(p.pref + p.R, R1, p.E, eoff, warp_tot);

    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e <= p.E; e += blockDim.x) p.expert_off[e] = eoff[e];
        for (int r = threadIdx.x; r <= p.R; r += blockDim.x) p.rank_off[r] = eoff[r * p.L];
        for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
            const int32_t* pe = p.pref + (int64_t)e * R1;
            p.ntpe[e] = pe[p.R];
            for (int s = 0; s < p.R; ++s) {
                p.src_off[(int64_t)e * p.R + s] = pe[s];
                p.cnt[(int64_t)s * p.E + e] = pe[s + 1] - pe[s];
            }
        }
        for (int i = threadIdx.x; i < p.R * p.R; i += blockDim.x) {
            const int s = i / p.R, r = i % p.R;
            const int32_t* pr = p.pref + (int64_t)(p.E + r) * R1;
            p.ntpr[i] = pr[s + 1] - pr[s];
        }
    }
    if (p.nc == 0) return;

    const int c = blockIdx.x;
    const int s = c / p.ncpr;
    const int t0 = (c % p.ncpr) * p.ch;
    const int t1 = min(p.T, t0 + p.ch);
    const int32_t* cpre = p.chunk + (int64_t)c * p.J;
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) base[e] = eoff[e] + cpre[e];
    __syncthreads();
    if (threadIdx.x >= 32) return;

    const int lane = threadIdx.x;
    const unsigned lt = (1u << lane) - 1u;
    const int64_t slot0 = ((int64_t)s * p.T + t0) * p.K;
    const int nslots = (t1 - t0) * p.K;
    for (int i0 = 0; i0 < nslots; i0 += 32) {
        const int j = i0 + lane;
        const bool active = j < nslots;
        const int e = active ? p.topk_idx[slot0 + j] : -1;
        const bool valid = e >= 0;
        const unsigned peers = __match_any_sync(FULL, valid ? e : -1);
        if (active) {
            int32_t row = -1;
            if (valid) {
                const int64_t r = (int64_t)base[e] + __popc(peers & lt);
                if (r < p.m_max) {
                    row = (int32_t)r;
                } else {
                    set_error(p.err, EP_DEVERR_ROW_BOUNDS);
                }
            }
            p.dst_row[slot0 + j] = row;
        }
        __syncwarp();
        if (valid && (peers >> lane) == 1u) base[e] += __popc(peers);  // highest lane of the group
        __syncwarp();
    }
}

template <int EPL>
cudaError_t launch_route(const LayoutParams& p, cudaStream_t st) {
    const size_t smem = sizeof(int) * p.J;
    route_count_kernel<EPL><<<p.nc, kRouteWarps * 32, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

int layout_chunk_tokens(int64_t n_tokens) {
    int ch = 32;
    while ((n_tokens + ch - 1) / ch > 1024) ch *= 2;
    return ch;
}

cudaError_t launch_layout(const ep_buffer& b, const LayoutArgs& a, cudaStream_t st) {
    const ep_config_t& c = b.cfg;
    LayoutParams p{};
    p.R = c.num_ranks;
    p.T = a.T;
    p.E = c.num_experts;
    p.K = c.topk;
    p.L = c.num_experts / c.num_ranks;
    p.G = c.num_groups;
    p.KG = c.topk_groups;
    p.ch = layout_chunk_tokens((int64_t)p.R * p.T);
    p.ncpr = (p.T + p.ch - 1) / p.ch;
    p.nc = p.R * p.ncpr;
    p.J = p.E + p.R;
    p.route = a.route;
    p.logits = a.logits;
    p.vec_logits = (a.logits != nullptr && (p.E % 4 == 0) && ((uintptr_t)a.logits % 16 == 0)) ? 1 : 0;
    p.in_idx = a.in_idx;
    p.in_w = a.in_w;
    p.mask_seed = a.mask_seed;
    p.mask_thr = a.mask_threshold;
    p.topk_idx = b.topk_idx;
    p.topk_w = b.topk_w;
    p.itr = b.is_token_in_rank;
    p.chunk = b.chunk;
    p.pref = b.pref;
    p.ntpr = b.num_tokens_per_rank;
    p.cnt = b.cnt;
    p.ntpe = b.num_tokens_per_expert;
    p.expert_off = b.expert_off;
    p.rank_off = b.rank_off;
    p.src_off = b.src_off;
    p.dst_row = b.dst_row;
    p.m_max = b.m_max;
    p.err = b.err;

    cudaError_t e = cudaSuccess;
    if (p.nc > 0) {
        const int epl = (p.E + 31) / 32;
        if (epl <= 1) e = launch_route<1>(p, st);
        else if (epl <= 2) e = launch_route<2>(p, st);
        else if (epl <= 4) e = launch_route<4>(p, st);
        else if (epl <= 8) e = launch_route<8>(p, st);
        else if (epl <= 16) e = launch_route<16>(p, st);
        else e = launch_route<32>(p, st);
        if (e != cudaSuccess) return e;
    }
    chunk_scan_kernel<<<(p.J + 31) / 32, dim3(32, 32), 0, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t smem = sizeof(int) * (2 * p.E + 1);
    assign_rows_kernel<<<p.nc > 0 ? p.nc : 1, kAssignThreads, smem, st>>>(p);
    return cudaGetLastError();
}

int64_t layout_scratch_ints(const ep_config_t& c, int T) {
    const int ch = layout_chunk_tokens((int64_t)c.num_ranks * T);
    const int64_t nc = (int64_t)c.num_ranks * ((T + ch - 1) / ch);
    const int64_t J = (int64_t)c.num_experts + c.num_ranks;
    return nc * J + J * (c.num_ranks + 1);
}

cudaError_t launch_layout_raw(const ep_config_t& c, const LayoutArgs& a, const ep_layout_t& out,
                              int32_t* scratch, uint32_t* err, cudaStream_t st) {
    LayoutParams p{};
    p.R = c.num_ranks;
    p.T = a.T;
    p.E = c.num_experts;
    p.K = c.topk;
    p.L = c.num_experts / c.num_ranks;
    p.G = c.num_groups;
    p.KG = c.topk_groups;
    p.ch = layout_chunk_tokens((int64_t)p.R * p.T);
    p.ncpr = (p.T + p.ch - 1) / p.ch;
    p.nc = p.R * p.ncpr;
    p.J = p.E + p.R;
    p.route = a.route;
    p.logits = a.logits;
    p.vec_logits = (a.logits != nullptr && (p.E % 4 == 0) && ((uintptr_t)a.logits % 16 == 0)) ? 1 : 0;
    p.in_idx = a.in_idx;
    p.in_w = a.in_w;
    p.mask_seed = a.mask_seed;
    p.mask_thr = a.mask_threshold;
    p.topk_idx = out.topk_idx;
    p.topk_w = out.topk_w;
    p.itr = out.is_token_in_rank;
    p.chunk = scratch;
    p.pref = scratch + (int64_t)p.nc * p.J;
    p.ntpr = out.num_tokens_per_rank;
    p.cnt = out.cnt_src_expert;
    p.ntpe = out.num_tokens_per_expert;
    p.expert_off = out.expert_off;
    p.rank_off = out.rank_off;
    p.src_off = out.src_off;
    p.dst_row = out.dst_row;
    p.m_max = (int64_t)p.R * p.T * p.K;  // no receive buffer: rows of this call only
    p.err = err;

    cudaError_t e = cudaSuccess;
    if (p.nc > 0) {
        const int epl = (p.E + 31) / 32;
        if (epl <= 1) e = launch_route<1>(p, st);
        else if (epl <= 2) e = launch_route<2>(p, st);
        else if (epl <= 4) e = launch_route<4>(p, st);
        else if (epl <= 8) e = launch_route<8>(p, st);
        else if (epl <= 16) e = launch_route<16>(p, st);
        else e = launch_route<32>(p, st);
        if (e != cudaSuccess) return e;
    }
    chunk_scan_kernel<<<(p.J + 31) / 32, dim3(32, 32), 0, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t smem = sizeof(int) * (2 * p.E + 1);
    assign_rows_kernel<<<p.nc > 0 ? p.nc : 1, kAssignThreads, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
