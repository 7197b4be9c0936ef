// Routing + layout (sm_100a). Top-K is fused with the layout that the
// dispatch needs: "DeepEP：年度总结中的计算通信重叠摘记", §节点内通信, fuses
// Top-K with the sparse communication and builds is_token_in_rank.
//
// One persistent cooperative kernel. The grid is one resident wave, and every
// CTA owns one chunk: a run of consecutive tokens of one source rank, so
// chunks are in global token order. Phases, separated by bounded grid barriers:
//   1  route: one warp per token. Top-K (optionally group-limited,
//      §计算-通信重叠), the slot mask, and the topk_idx / topk_w /
//      is_token_in_rank writes. Each warp takes a contiguous run of its
//      chunk's tokens and counts its slots per expert and its tokens per
//      destination rank in shared memory. The chunk's totals go to global
//      scratch.
//   2  scan: one CTA per expert/rank column. A block scan over the chunks
//      gives each chunk's exclusive prefix and the column total. Reading it
//      at each rank's first chunk gives src_off and cnt (expert columns) or
//      num_tokens_per_rank (rank columns).
//   3  place: every CTA scans the expert totals into expert_off. Its warps
//      then turn their kept histograms into per-warp row bases and rank their
//      own slots in (token, slot) order with match_any/popc, writing dst_row.
// Receive rows come out ordered by (expert, source rank, token, slot).
//
// Routing arithmetic:
//  - Expert ranking compares the logits exactly (order-preserving 32-bit
//    keys; equal values go to the lower expert id).
//  - Group scores (sum of the two largest sigmoids) run in fp32, with a
//    bound on their error. If the gap between the last kept and the first
//    dropped group is under 4e-6, well above that bound, the warp recomputes
//    the scores in fp64, the precision the decision is defined in. The kept
//    groups therefore always equal the fp64 ones.
//  - Weights are computed in fp64 and rounded once to fp32.
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace ep {
namespace {

constexpr int kWarps = 8;  // warps per CTA
constexpr int kPrePlace = 2;  // placement rounds (32 slots each) whose experts are loaded ahead
constexpr int kThreads = kWarps * 32;

struct LayoutParams {
    int R, T, E, K, L, G, KG, J;  // J = E + R histogram columns
    int S;                        // source ranks whose tokens this launch routes: R, or 1 (one rank's own)
    int64_t g_base;               // global id of local token 0 (the slot mask hashes global ids)
    uint32_t l_magic;             // e / L == __umulhi(e, l_magic) for 0 <= e < 2^16
    int nb;                       // CTAs (one resident wave)
    int ncpr, nc;                 // chunks per rank, chunks (nc <= nb)
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
    int32_t* chunk;  // [J][nc]: chunk counts, then their exclusive prefix over chunks
    int32_t* tot;    // [J]: column totals
    int32_t *ntpr, *cnt, *ntpe, *expert_off, *rank_off, *src_off, *dst_row;
    int64_t m_max;
    int ll;     // low-latency layout: row = (e*R + s)*T_max + j
    int T_max;  // region size (low-latency layout)
    int dedup;  // also place one row per (token, destination rank)
    int32_t *tok_row, *rank_row_off, *rank_src_off;  // dedup outputs
    uint32_t* err;
    uint32_t* bar;  // [2]: barrier arrivals, finished CTAs; both 0 between launches
};

__device__ __forceinline__ double sigmoid_d(double x) { return 1.0 / (1.0 + exp(-x)); }
// fp32 sigmoid from the fast intrinsics, whose published maximum errors are
// 2 + floor(|1.173 x|) ulp for __expf(x) and 2 ulp for __fdividef(x, y) with
// 2^-126 <= |y| <= 2^126 (0 above, where the true value is below 2^-126).
// With e = __expf(-x) off by |d| <= (2 + 1.2|x|) 2^-23 relative, the add and
// the divide by 2^-24 and 2^-22 relative:
//   |s - sigmoid(x)| <= s(1-s)|d| + s(2^-24 + 2^-22) <= (0.63 + 0.5 + 2) 2^-23 < 3.8e-7,
// as s(1-s)(2 + 1.2|x|) <= 0.63 for every x.
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded grid-wide barrier (the grid is co-resident: cooperative launch).
// The CTA barrier orders every thread's writes before thread 0, whose
// release-add publishes them (cumulatively) at GPU scope; the acquire loads
// of the spin order the CTA's later reads after every other CTA's arrival.
__device__ void grid_barrier(uint32_t* arrive, uint32_t target, uint32_t* err,
                             unsigned long long limit_ns = kWaitLimitNs) {
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(arrive) : "memory");
        const unsigned long long t0 = globaltimer_ns();
        while (ld_acquire(arrive) < target) {
            if (globaltimer_ns() - t0 > limit_ns) {
                set_error(err, EP_DEVERR_TIMEOUT);
                break;
            }
            __nanosleep(32);
        }
    }
    __syncthreads();
}

// Top-2 of one pair per lane across lanes that differ in the bits of `span`
// (a power of two): butterfly over offsets span/2..1.
__device__ __forceinline__ void top2_merge(uint32_t& a, uint32_t& b, int span) {
    for (int off = span >> 1; off > 0; off >>= 1) {
        const uint32_t oa = __shfl_xor_sync(FULL, a, off);
        const uint32_t ob = __shfl_xor_sync(FULL, b, off);
        const uint32_t hi = max(a, oa);
        const uint32_t lo = max(min(a, oa), max(b, ob));
        a = hi;
        b = lo;
    }
}

// This lane's three best candidates by (key desc, position asc), skipping
// taken positions and zero keys. Returns key 0 where there is none.
template <int EPL>
__device__ __forceinline__ void top3_of(const uint32_t (&key)[EPL], uint32_t taken, uint32_t& a, int& pa,
                                        uint32_t& b, int& pb, uint32_t& c, int& pc) {
    a = b = c = 0u;
    pa = pb = pc = 0;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
        const uint32_t k = ((taken >> j) & 1u) ? 0u : key[j];
        if (k > a) {  // strict: an equal key later in the list stays behind
            c = b;
            pc = pb;
            b = a;
            pb = pa;
            a = k;
            pa = j;
        } else if (k > b) {
            c = b;
            pc = pb;
            b = k;
            pb = j;
        } else if (k > c) {
            c = k;
            pc = j;
        }
    }
}

// Group scores and the kept-group mask (bit g set = group g kept).
template <int EPL>
__device__ __forceinline__ uint32_t kept_groups(const LayoutParams& p, const uint32_t (&key)[EPL], uint32_t a,
                                                uint32_t b, int lane) {
    const int gs = p.E / p.G;
    const int e0 = lane * EPL;
    const int lpg = gs / EPL;
    int rank = 0;
    if (gs % EPL == 0 && lpg <= 32 && (lpg & (lpg - 1)) == 0) {
        // each group spans lpg whole lanes: the lanes' top-2, then a butterfly
        top2_merge(a, b, lpg);
        // group g's fp32 score sits on lane g * lpg. A group's rank is the
        // number of groups ahead of it: higher score, or equal score and lower
        // id. Kept = rank < KG.
        // group score: lane pairs (2i, 2i+1) inside a group take one sigmoid
        // each, of a and of b, and add them (either order: the sum is exact)
        float s32;
        if (lpg >= 2) {
            const float sg1 = sigmoid_f(key_value((lane & 1) ? b : a));
            s32 = sg1 + __shfl_xor_sync(FULL, sg1, 1);
        } else {
            s32 = sigmoid_f(key_value(a)) + sigmoid_f(key_value(b));
        }
        float sg;   // score of group gq
        int gq, rk;  // rank of group gq, on the lanes that report it
        bool lead;  // this lane reports group gq
        if (p.G <= 8) {
            // all pairs at once: lane = 4*gq + q compares group gq with groups 2q, 2q+1
            gq = lane >> 2;
            const int q = lane & 3, h0 = 2 * q, h1 = 2 * q + 1;
            sg = __shfl_sync(FULL, s32, (gq < p.G ? gq : 0) * lpg);
            const float s0 = __shfl_sync(FULL, s32, (h0 < p.G ? h0 : 0) * lpg);
            const float s1 = __shfl_sync(FULL, s32, (h1 < p.G ? h1 : 0) * lpg);
            rk = (h0 < p.G && (s0 > sg || (s0 == sg && h0 < gq))) + (h1 < p.G && (s1 > sg || (s1 == sg && h1 < gq)));
            rk += __shfl_xor_sync(FULL, rk, 1);
            rk += __shfl_xor_sync(FULL, rk, 2);
            lead = q == 0 && gq < p.G;
        } else {
            // lane g ranks group g against every group (independent shuffles)
            gq = lane;
            sg = __shfl_sync(FULL, s32, (lane < p.G ? lane : 0) * lpg);
            rk = 0;
            for (int h = 0; h < p.G; ++h) {
                const float sh = __shfl_sync(FULL, sg, h);
                rk += (sh > sg || (sh == sg && h < lane)) ? 1 : 0;
            }
            lead = lane < p.G;
        }
        const uint32_t kept = __reduce_or_sync(FULL, (lead && rk < p.KG) ? 1u << gq : 0u);  // gq < G <= 32
        bool certain = true;
        if (p.KG < p.G) {
            // A score (two sigmoids < 3.8e-7 each, then an add rounding
            // < 1.2e-7) errs by < 9e-7, a gap between two by < 1.8e-6. A gap
            // over 4e-6 decides as fp64 would.
            const uint32_t m_last = __ballot_sync(FULL, lead && rk == p.KG - 1);
            const uint32_t m_next = __ballot_sync(FULL, lead && rk == p.KG);
            const float s_last = __shfl_sync(FULL, sg, __ffs(m_last) - 1);
            const float s_next = __shfl_sync(FULL, sg, __ffs(m_next) - 1);
            certain = (s_last - s_next) > 4e-6f;
        }
        if (certain) return kept;
        // warp-uniform: decide in fp64
        const int src = (lane < p.G) ? lane * lpg : 0;
        const double s64 = sigmoid_d((double)key_value(a)) + sigmoid_d((double)key_value(b));
        const double sd = __shfl_sync(FULL, s64, src);
        for (int h = 0; h < p.G; ++h) {
            const double sh = __shfl_sync(FULL, sd, h);
            if (lane < p.G && (sh > sd || (sh == sd && h < lane))) ++rank;
        }
    } else {
        // generic layout of groups over lanes: one warp-wide top-2 per group, fp64
        double score = -1.0;
        for (int grp = 0; grp < p.G; ++grp) {
            uint32_t a = 0, b = 0;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                const int e = e0 + j;
                const uint32_t k = (e < p.E && e / gs == grp) ? key[j] : 0u;
                if (k > a) {
                    b = a;
                    a = k;
                } else if (k > b) {
                    b = k;
                }
            }
            top2_merge(a, b, 32);
            if (lane == grp) score = sigmoid_d((double)key_value(a)) + sigmoid_d((double)key_value(b));
        }
        for (int h = 0; h < p.G; ++h) {
            const double sh = __shfl_sync(FULL, score, h);
            if (lane < p.G && (sh > score || (sh == score && h < lane))) ++rank;
        }
    }
    return __ballot_sync(FULL, lane < p.G && rank < p.KG);
}

// This lane's EPL logits of token g (experts lane*EPL ..); zeros past E.
template <int EPL>
__device__ __forceinline__ void load_logits(const LayoutParams& p, int64_t g, int lane, float (&v)[EPL]) {
    const float* row = p.logits + g * p.E;
    const int e0 = lane * EPL;
    if (EPL >= 4 && p.vec_logits) {
#pragma unroll
        for (int j = 0; j < EPL; j += 4) {
            if (e0 + j < p.E) {
                const float4 q = __ldcs(reinterpret_cast<const float4*>(row + e0 + j));
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
        for (int j = 0; j < EPL; ++j) v[j] = (e0 + j < p.E) ? __ldcs(row + e0 + j) : 0.0f;
    }
}

// Per-warp staging of a group of B = 32 / K tokens: slot k of the group's
// token j sits at index j*K + k, so the group's per-slot work (weights, mask,
// writes, counts) runs once over all 32 lanes instead of once per token on K
// lanes.
struct WarpStage {
    int32_t e[32];     // expert of each slot (-1: none)
    uint32_t key[32];  // order key of the slot's logit
    double z[32];      // per token: sum over all experts of exp(l - max) (plain softmax)
    double s[32];      // per slot: unnormalised weight
    uint32_t rb[32];   // per slot: bit of its destination rank
};

// Selects token g's top-K with one warp from its logits vin (load_logits) and
// stages slot k (expert, key) at st.e / st.key[j*K + k]. Ranking: logit
// descending, then expert id ascending.
template <int EPL>
__device__ __forceinline__ void select_token(const LayoutParams& p, int lane, const float (&vin)[EPL], int j,
                                             WarpStage& st) {
    uint32_t key[EPL];
    const int e0 = lane * EPL;
#pragma unroll
    for (int i = 0; i < EPL; ++i) key[i] = (e0 + i < p.E) ? order_key(vin[i]) : 0u;

    // this lane's three best candidates; a lane rescans its list only when
    // all three have been taken
    uint32_t a, b, c, taken = 0u;
    int pa, pb, pc;
    top3_of<EPL>(key, 0u, a, pa, b, pb, c, pc);

    if (p.route == EP_ROUTE_GROUP_SIGMOID && p.G > 1) {
        const uint32_t kept = kept_groups<EPL>(p, key, a, b, lane);
        const int gs = p.E / p.G;
        if (gs % EPL == 0) {
            // all of this lane's experts sit in group e0 / gs
            if (!((kept >> (e0 / gs)) & 1u)) a = b = c = 0u;
        } else {
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int e = e0 + i;
                if (e < p.E && !((kept >> (e / gs)) & 1u)) key[i] = 0u;
            }
            top3_of<EPL>(key, 0u, a, pa, b, pb, c, pc);
        }
    }

    // top-K: K rounds of warp max. Equal keys go to the lowest lane, which
    // holds the lowest expert ids; within a lane top3_of keeps id order. The
    // winner is the lane holding the maximum with no lower lane holding it.
    // Slot 0's key is the token's largest logit (the softmax max).
    const int base = j * p.K;
    const unsigned below = (1u << lane) - 1u;
    for (int k = 0; k < p.K; ++k) {
        const uint32_t wk = __reduce_max_sync(FULL, a);
        const unsigned tie = __ballot_sync(FULL, a == wk);
        if (a == wk && (tie & below) == 0u) {
            st.e[base + k] = (wk != 0u) ? e0 + pa : -1;
            st.key[base + k] = wk;
            if (wk != 0u) {  // pop this lane's head
                taken |= 1u << pa;
                a = b;
                pa = pb;
                b = c;
                pb = pc;
                c = 0u;
                if (a == 0u) top3_of<EPL>(key, taken, a, pa, b, pb, c, pc);
            }
        }
    }

    if (p.route == EP_ROUTE_SOFTMAX) {
        // the normaliser of the plain softmax: every expert, fp64
        __syncwarp();
        const double mx = (double)key_value(st.key[base]);
        double z = 0.0;
#pragma unroll
        for (int i = 0; i < EPL; ++i)  // softmax routes never zero keys: key i is logit i
            if (key[i] != 0u) z += exp((double)key_value(key[i]) - mx);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(FULL, z, off);
        if (lane == 0) st.z[j] = z;
    }
}

// Finishes the staged group: tokens g0 .. g0+nt-1 (global index g0 within
// this launch), lane = j*K + k. Weights in fp64, rounded once to fp32:
//  - group sigmoid: w_k = s_k / sum_k s_k, s = sigmoid(logit);
//  - softmax: w_k = exp(l_k - max) / z;
//  - renormalised softmax: w_k = p_k / sum_k p_k = exp(l_k - max) / sum_k exp(l_k - max)
//    (z cancels).
// The sums run over the token's slots in ascending k. Then the slot mask,
// the topk_idx / topk_w writes (coalesced over the group), the per-warp
// expert counts, is_token_in_rank and the per-warp rank counts.
__device__ __forceinline__ void finish_group(const LayoutParams& p, int lane, int64_t g0, int nt, WarpStage& st,
                                             int* my_hist) {
    const int K = p.K;
    const int jj = lane / K, k = lane - jj * K;
    const bool act = jj < nt;
    const int64_t g = g0 + jj;
    int e = -1;
    float w = 0.0f;
    if (p.logits == nullptr) {
        // caller-supplied top-k
        if (act) {
            e = p.in_idx[g * K + k];
            w = p.in_w[g * K + k];
            if (e < -1 || e >= p.E) {
                set_error(p.err, EP_DEVERR_EXPERT_ID);
                e = -1;
            }
        }
    } else {
        __syncwarp();
        e = act ? st.e[lane] : -1;
        double sv = 0.0;
        if (e >= 0) {
            const double l = (double)key_value(st.key[lane]);
            sv = (p.route == EP_ROUTE_GROUP_SIGMOID) ? sigmoid_d(l) : exp(l - (double)key_value(st.key[jj * K]));
        }
        st.s[lane] = sv;
        __syncwarp();
        double den = 0.0;
        if (p.route == EP_ROUTE_SOFTMAX) {
            den = act ? st.z[jj] : 1.0;
        } else if (act) {
            for (int q = 0; q < K; ++q) den += st.s[jj * K + q];
        }
        w = (e >= 0) ? (float)(sv / den) : 0.0f;
    }
    // slot mask
    if (act && p.mask_thr != 0ull) {
        const uint64_t h = splitmix64(p.mask_seed ^ (uint64_t)((p.g_base + g) * K + k));
        if ((h >> 32) < p.mask_thr) {
            e = -1;
            w = 0.0f;
        }
    }
    if (act) {
        p.topk_idx[g * K + k] = e;
        p.topk_w[g * K + k] = w;
        if (e >= 0) atomicAdd(&my_hist[e], 1);
    }
    st.rb[lane] = (e >= 0) ? (1u << (p.L == 1 ? (uint32_t)e : __umulhi((uint32_t)e, p.l_magic))) : 0u;
    __syncwarp();
    for (int i = lane; i < nt * p.R; i += 32) {
        const int tj = i / p.R, r = i - tj * p.R;
        uint32_t bits = 0u;
        for (int q = 0; q < K; ++q) bits |= st.rb[tj * K + q];
        const uint32_t in = (bits >> r) & 1u;
        p.itr[(g0 + tj) * p.R + r] = (uint8_t)in;
        if (in) atomicAdd(&my_hist[p.E + r], 1);
    }
    __syncwarp();  // the stage is refilled by the next group
}

// Outputs of column `col` for source rank r, whose chunks' exclusive prefix
// starts at a and ends at b: src_off and cnt (expert columns), or
// num_tokens_per_rank and the dedup rank offsets (rank columns).
__device__ __forceinline__ void column_outputs(const LayoutParams& p, int col, int r, int a, int b) {
    if (col < p.E) {
        p.src_off[(int64_t)col * p.S + r] = a;
        p.cnt[(int64_t)r * p.E + col] = b - a;
    } else {
        p.ntpr[(int64_t)r * p.R + (col - p.E)] = b - a;
        if (p.dedup) p.rank_src_off[(int64_t)(col - p.E) * p.S + r] = a;
    }
}

template <int EPL>
__global__ void __launch_bounds__(kThreads, EPL >= 16 ? 2 : 4) layout_kernel(LayoutParams p) {
    extern __shared__ int sm[];
    int* hist = sm;                      // [kWarps][J]: per-warp counts, later per-warp row bases
    int* eoff = sm + kWarps * p.J;       // [max(E, nc) + 1]: scan output
    __shared__ int warp_tot[33];
    __shared__ WarpStage stage[kWarps];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int c = blockIdx.x;
    const bool has_chunk = c < p.nc;
    int s = 0, t0 = 0, t1 = 0, w0 = 0, w1 = 0;
    if (has_chunk) {
        s = c / p.ncpr;
        const int j = c % p.ncpr;
        t0 = (int)((int64_t)j * p.T / p.ncpr);
        t1 = (int)((int64_t)(j + 1) * p.T / p.ncpr);
        const int n = t1 - t0;
        w0 = t0 + warp * n / kWarps;
        w1 = t0 + (warp + 1) * n / kWarps;
    }

    // ---- phase 1: route; per-warp expert and rank histograms. The warp
    // selects B = 32 / K tokens one at a time, then finishes them together.
    for (int i = threadIdx.x; i < kWarps * p.J; i += kThreads) hist[i] = 0;
    __syncthreads();
    int* my_hist = hist + warp * p.J;
    WarpStage& st = stage[warp];
    const int B = 32 / p.K;
    float vnext[EPL];
    if (p.logits != nullptr && w0 < w1) load_logits<EPL>(p, (int64_t)s * p.T + w0, lane, vnext);
    for (int t0g = w0; t0g < w1; t0g += B) {
        const int nt = min(B, w1 - t0g);
        const int64_t g0 = (int64_t)s * p.T + t0g;
        if (p.logits != nullptr) {
            for (int j = 0; j < nt; ++j) {
                const int t = t0g + j;
                float vcur[EPL];
#pragma unroll
                for (int i = 0; i < EPL; ++i) vcur[i] = vnext[i];
                if (t + 1 < w1) load_logits<EPL>(p, g0 + j + 1, lane, vnext);  // prefetch
                select_token<EPL>(p, lane, vcur, j, st);
            }
        }
        finish_group(p, lane, g0, nt, st, my_hist);
    }
    __syncthreads();
    if (has_chunk) {
        for (int j = threadIdx.x; j < p.J; j += kThreads) {
            int sum = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) sum += hist[w * p.J + j];
            p.chunk[(int64_t)j * p.nc + c] = sum;
        }
    }
    grid_barrier(p.bar, (uint32_t)p.nb, p.err);

    // ---- phase 2: per-column exclusive scan over chunks. Few chunks: one
    // warp per column (4 chunks per lane). Otherwise one CTA per column.
    if (p.nc <= 4 * 32) {
        for (int col = blockIdx.x * kWarps + warp; col < p.J; col += p.nb * kWarps) {
            int32_t* colp = p.chunk + (int64_t)col * p.nc;
            int v[4];
            int local = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j = 4 * lane + i;
                v[i] = (j < p.nc) ? colp[j] : 0;
                local += v[i];
            }
            int incl = local;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(FULL, incl, off);
                if (lane >= off) incl += o;
            }
            const int total = __shfl_sync(FULL, incl, 31);
            int run = incl - local;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j = 4 * lane + i;
                if (j < p.nc) colp[j] = run;
                run += v[i];
            }
            __syncwarp();  // the prefixes written above are read back by other lanes
            if (lane < p.S) {
                const int r = lane;  // source rank; S * ncpr = nc
                const int a = (p.nc > 0) ? colp[r * p.ncpr] : 0;
                const int b = (p.nc > 0 && r + 1 < p.S) ? colp[(r + 1) * p.ncpr] : total;
                column_outputs(p, col, r, a, b);
            }
            if (lane == 0) {
                p.tot[col] = total;
                if (col < p.E) p.ntpe[col] = total;
            }
            __syncwarp();
        }
    } else {
        for (int col = blockIdx.x; col < p.J; col += p.nb) {
            int32_t* colp = p.chunk + (int64_t)col * p.nc;
            block_exclusive_scan(colp, 1, p.nc, eoff, warp_tot);  // eoff: scratch here, [nc + 1]
            for (int cc = threadIdx.x; cc < p.nc; cc += kThreads) colp[cc] = eoff[cc];
            // prefix at each rank's first chunk; eoff[nc] is the column total
            if (threadIdx.x < p.S) {
                const int r = threadIdx.x;  // source rank
                column_outputs(p, col, r, eoff[r * p.ncpr], eoff[(r + 1) * p.ncpr]);
            }
            if (threadIdx.x == 0) {
                const int total = eoff[p.nc];
                p.tot[col] = total;
                if (col < p.E) p.ntpe[col] = total;
            }
            __syncthreads();
        }
    }
    grid_barrier(p.bar, 2u * (uint32_t)p.nb, p.err);

    // ---- phase 3: expert offsets, per-warp bases, row placement. The warp's
    // first kPrePlace * 32 slot experts and this thread's chunk prefix are
    // loaded before the scan, so their latency overlaps it.
    const unsigned lt = (1u << lane) - 1u;
    const int64_t slot0 = ((int64_t)s * p.T + w0) * p.K;
    const int nslots = has_chunk ? (w1 - w0) * p.K : 0;
    int pre_e[kPrePlace];
#pragma unroll
    for (int q = 0; q < kPrePlace; ++q) {
        const int j = q * 32 + lane;
        pre_e[q] = (j < nslots) ? p.topk_idx[slot0 + j] : -1;
    }
    const int pre_chunk = (has_chunk && (int)threadIdx.x < p.E) ? p.chunk[(int64_t)threadIdx.x * p.nc + c] : 0;
    block_exclusive_scan(p.tot, 1, p.E, eoff, warp_tot);
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e <= p.E; e += kThreads) p.expert_off[e] = eoff[e];
        for (int r = threadIdx.x; r <= p.R; r += kThreads) p.rank_off[r] = eoff[r * p.L];
    }
    __shared__ int s_rr[33];  // dedup: rows per destination rank, exclusive prefix
    if (p.dedup) {
        if (warp == 0) {
            const int v = (lane < p.R) ? p.tot[p.E + lane] : 0;
            int incl = v;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(FULL, incl, off);
                if (lane >= off) incl += o;
            }
            if (lane < p.R) s_rr[lane] = incl - v;
            if (lane == p.R - 1) s_rr[p.R] = incl;
        }
        __syncthreads();
        if (blockIdx.x == 0)
            for (int r = threadIdx.x; r <= p.R; r += kThreads) p.rank_row_off[r] = s_rr[r];
    }
    if (has_chunk) {
        if (p.dedup) {
            for (int r = threadIdx.x; r < p.R; r += kThreads) {
                const int j = p.E + r;
                int run = s_rr[r] + p.chunk[(int64_t)j * p.nc + c];
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    const int x = hist[w * p.J + j];
                    hist[w * p.J + j] = run;
                    run += x;
                }
            }
        }
        for (int e = threadIdx.x; e < p.E; e += kThreads) {
            // standard: expert block + chunk prefix. Low-latency: fixed region of
            // (e, s) + this rank's part of the chunk prefix
            const int cpre = (e == (int)threadIdx.x) ? pre_chunk : p.chunk[(int64_t)e * p.nc + c];
            int run = p.ll ? (int)(((int64_t)e * p.R + s) * p.T_max) + cpre - p.src_off[(int64_t)e * p.R + s]
                           : eoff[e] + cpre;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const int x = hist[w * p.J + e];
                hist[w * p.J + e] = run;
                run += x;
            }
        }
        __syncthreads();
        for (int i0 = 0; i0 < nslots; i0 += 32) {
            const int j = i0 + lane;
            const bool active = j < nslots;
            int e = -1;
#pragma unroll
            for (int q = 0; q < kPrePlace; ++q)
                if (i0 == q * 32) e = pre_e[q];
            if (i0 >= kPrePlace * 32) e = active ? p.topk_idx[slot0 + j] : -1;
            const bool valid = e >= 0;
            const unsigned peers = __match_any_sync(FULL, valid ? e : -1);
            if (active) {
                int32_t row = -1;
                if (valid) {
                    const int64_t r = (int64_t)my_hist[e] + __popc(peers & lt);
                    const bool in_region =
                        !p.ll || r - ((int64_t)e * p.R + s) * p.T_max < (int64_t)p.T_max;  // only duplicates overflow
                    if (r < p.m_max && in_region) row = (int32_t)r;
                    else set_error(p.err, EP_DEVERR_ROW_BOUNDS);
                }
                p.dst_row[slot0 + j] = row;
            }
            __syncwarp();
            if (valid && (peers >> lane) == 1u) my_hist[e] += __popc(peers);  // highest lane of the group
            __syncwarp();
        }
        if (p.dedup) {
            // one row per (token, destination rank), tokens in order: lane = token
            for (int t0w = w0; t0w < w1; t0w += 32) {
                const int t = t0w + lane;
                const bool active = t < w1;
                const int64_t g = (int64_t)s * p.T + t;
                for (int r = 0; r < p.R; ++r) {
                    const bool in = active && p.itr[g * p.R + r] != 0;
                    const unsigned bal = __ballot_sync(FULL, in);
                    if (active) p.tok_row[g * p.R + r] = in ? my_hist[p.E + r] + __popc(bal & lt) : -1;
                    __syncwarp();
                    if (lane == 0) my_hist[p.E + r] += __popc(bal);
                    __syncwarp();
                }
            }
        }
    }

    // The last CTA out resets the barrier words for the next launch. Every
    // CTA counts itself out after leaving the last grid barrier, so when the
    // count is full no CTA reads the words again in this launch; the end of
    // the kernel publishes the reset to the next one.
    if (threadIdx.x == 0 && atomicAdd(p.bar + 1, 1u) == (uint32_t)p.nb - 1u) {
        p.bar[0] = 0u;
        p.bar[1] = 0u;
    }
}

// Self-test of the bounded wait: the barrier target (one more arrival than the
// grid has) can never be met, so every CTA must give up after limit_ns and
// set EP_DEVERR_TIMEOUT.
__global__ void barrier_timeout_selftest_kernel(uint32_t* bar, uint32_t* err, unsigned long long limit_ns) {
    grid_barrier(bar, gridDim.x + 1u, err, limit_ns);
}

// Resident CTAs per SM for each kernel instantiation and shared-memory size
// (the occupancy query is a host-side cost worth skipping per call).
struct OccCache {
    std::mutex mu;
    const void* fn[32] = {};
    size_t smem[32] = {};
    int dev[32] = {};
    int per_sm[32] = {};
    int n = 0;
};
OccCache g_occ;

cudaError_t occupancy(const void* fn, size_t smem, int dev, int* per_sm) {
    std::lock_guard<std::mutex> lock(g_occ.mu);
    for (int i = 0; i < g_occ.n; ++i)
        if (g_occ.fn[i] == fn && g_occ.smem[i] == smem && g_occ.dev[i] == dev) {
            *per_sm = g_occ.per_sm[i];
            return cudaSuccess;
        }
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, fn, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (g_occ.n < 32) {
        g_occ.fn[g_occ.n] = fn;
        g_occ.smem[g_occ.n] = smem;
        g_occ.dev[g_occ.n] = dev;
        g_occ.per_sm[g_occ.n] = *per_sm;
        ++g_occ.n;
    }
    return cudaSuccess;
}

template <int EPL>
cudaError_t launch_epl(LayoutParams& p, int dev, int sm_count, int max_ctas, cudaStream_t st) {
    auto kern = layout_kernel<EPL>;
    const int scan_n = (p.E > max_ctas) ? p.E : max_ctas;
    const size_t smem = sizeof(int) * ((size_t)kWarps * p.J + scan_n + 1);
    if (smem > 48 * 1024) return cudaErrorInvalidConfiguration;
    int per_sm = 0;
    cudaError_t e = occupancy((const void*)kern, smem, dev, &per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int nb = per_sm * sm_count;
    if (nb > max_ctas) nb = max_ctas;
    // small batches: about one token per warp, so the grid barriers stay cheap
    const int64_t want = ((int64_t)p.S * p.T + kWarps - 1) / kWarps;
    if (want < nb) nb = (int)(want > p.S ? want : p.S);
    if (nb < p.S) return cudaErrorInvalidConfiguration;  // every source rank needs a chunk
    p.nb = nb;
    int ncpr = nb / p.S;
    if (ncpr > p.T) ncpr = p.T;
    p.ncpr = ncpr > 0 ? ncpr : 1;
    p.nc = (p.T > 0) ? p.S * ncpr : 0;
    void* args[] = {&p};
    e = cudaLaunchCooperativeKernel((const void*)kern, dim3(nb), dim3(kThreads), args, smem, st);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

int64_t layout_scratch_ints(const ep_config_t& c, int max_ctas) {
    const int64_t J = (int64_t)c.num_experts + c.num_ranks;
    return kLayoutControlInts + J * max_ctas + J;
}

cudaError_t launch_layout_raw(const ep_config_t& c, const LayoutArgs& a, const ep_layout_t& out,
                              int32_t* scratch, int max_ctas, uint32_t* err, cudaStream_t st) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    LayoutParams p{};
    p.R = c.num_ranks;
    p.T = a.T;
    p.E = c.num_experts;
    p.K = c.topk;
    p.L = c.num_experts / c.num_ranks;
    // ceil(2^32 / L): exact quotients for e < 2^16 since 2 <= L <= 1024 (L == 1 is e itself)
    p.l_magic = p.L > 1 ? (uint32_t)((((uint64_t)1 << 32) + (uint64_t)p.L - 1) / (uint64_t)p.L) : 0u;
    p.G = c.num_groups;
    p.KG = c.topk_groups;
    p.J = p.E + p.R;
    p.S = a.S > 0 ? a.S : p.R;
    p.g_base = a.g_base;
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
    p.ntpr = out.num_tokens_per_rank;
    p.cnt = out.cnt_src_expert;
    p.ntpe = out.num_tokens_per_expert;
    p.expert_off = out.expert_off;
    p.rank_off = out.rank_off;
    p.src_off = out.src_off;
    p.dst_row = out.dst_row;
    p.m_max = a.m_max;
    p.ll = a.low_latency;
    p.T_max = a.T_max;
    p.dedup = a.tok_row != nullptr;
    p.tok_row = a.tok_row;
    p.rank_row_off = a.rank_row_off;
    p.rank_src_off = a.rank_src_off;
    p.err = err;
    // scratch: [control][chunk J*max_ctas][tot J]
    p.bar = reinterpret_cast<uint32_t*>(scratch);
    p.chunk = scratch + kLayoutControlInts;
    p.tot = p.chunk + (int64_t)p.J * max_ctas;
    const int epl = (p.E + 31) / 32;
    if (epl <= 1) return launch_epl<1>(p, dev, sms, max_ctas, st);
    if (epl <= 2) return launch_epl<2>(p, dev, sms, max_ctas, st);
    if (epl <= 4) return launch_epl<4>(p, dev, sms, max_ctas, st);
    if (epl <= 8) return launch_epl<8>(p, dev, sms, max_ctas, st);
    if (epl <= 16) return launch_epl<16>(p, dev, sms, max_ctas, st);
    return launch_epl<32>(p, dev, sms, max_ctas, st);
}

cudaError_t launch_layout(const ep_buffer& b, const LayoutArgs& a, cudaStream_t st) {
    ep_layout_t out;
    out.topk_idx = b.topk_idx;
    out.topk_w = b.topk_w;
    out.is_token_in_rank = b.is_token_in_rank;
    out.num_tokens_per_rank = b.num_tokens_per_rank;
    out.cnt_src_expert = b.cnt;
    out.num_tokens_per_expert = b.num_tokens_per_expert;
    out.expert_off = b.expert_off;
    out.rank_off = b.rank_off;
    out.src_off = b.src_off;
    out.dst_row = b.dst_row;
    LayoutArgs aa = a;
    aa.m_max = b.m_max;
    aa.low_latency = (b.cfg.flags & EP_FLAG_LOW_LATENCY) ? 1 : 0;
    aa.T_max = b.cfg.max_tokens_per_rank;
    if (b.cfg.flags & EP_FLAG_DEDUP) {
        aa.tok_row = b.tok_row;
        aa.rank_row_off = b.rank_row_off;
        aa.rank_src_off = b.rank_src_off;
    }
    return launch_layout_raw(b.cfg, aa, out, b.scratch, kMaxLayoutCtas, b.err, st);
}

cudaError_t launch_barrier_timeout_selftest(uint32_t* words, unsigned long long limit_ns, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(words, 0, 4 * sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    uint32_t* bar = words;
    uint32_t* err = words + 2;
    void* args[] = {&bar, &err, &limit_ns};
    e = cudaLaunchCooperativeKernel((const void*)barrier_timeout_selftest_kernel, dim3(2), dim3(32), args, 0, st);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ep
