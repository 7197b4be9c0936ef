// Dispatch (sm_100a): scatter each token's hidden vector to the receive row
// of every unmasked slot. Only target experts get a copy
// ("DeepEP：年度总结中的计算通信重叠摘记", §节点内通信: is_token_in_rank, no
// full all-to-all). The optional FP8 cast sends 1 byte per element instead of
// 2 (same section) and adds one fp32 scale per 128 channels.
//
// One CTA per token; under a num_sms cap, at most num_sms CTAs of several
// token groups each, looping over tokens. The threads read the token's row
// once into registers with 256-bit loads, then write it to each of the K
// receive rows:
//  - bf16: 256-bit stores, 16 channels per thread;
//  - FP8: each thread reads 16 channels (32 B) and 8 threads reduce amax over
//    one 128-channel block with xor shuffles. It casts with
//    cvt.rn.satfinite.e4m3x2 and writes 16 B (128-bit store) per row, and
//    the block's first thread writes the fp32 scale.
// Each receive row is written as one contiguous 14 KB (bf16) or 7 KB (FP8)
// burst by one CTA, and consecutive tokens' rows of the same expert are
// adjacent. Measured on B200, register stores from 256-bit vectors beat
// bulk-copy (cp.async.bulk) stores from shared memory for this scatter:
// 6.4 vs 5.7 TB/s on the prefill shape. The barrier after the loads keeps a
// CTA's warps in step, so each 14 KB row leaves as one burst. Without it, each
// warp fetching the row indices itself, the warps drift apart, their rows
// interleave, and prefill dispatch slows from 682 to 708 us.
// Every row index is checked against the buffer (EP_DEVERR_ROW_BOUNDS).
//
// The same kernels serve one rank of a one-process-per-GPU deployment
// (PeerRecv): each slot's row then goes to the receive buffer of its
// destination rank, through a table of that rank's device pointers (peer
// memory over NVLink on a multi-GPU node).
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace ep {
namespace {

struct DispatchParams {
    int64_t N;
    int K, H;
    int64_t m_max;
    const uint8_t* x;  // bf16 [N, H]
    const int32_t* dst_row;
    const float* topk_w;
    const uint8_t* dst_rank;  // [N, K] destination rank of each slot (PeerRecv only)
    int num_peers;            // entries of the PeerRecv tables
    int64_t g_base;           // global id of local token 0 (recv_src)
    int ordered;              // write a token's rows in (destination rank, row) order
    int sub_threads;          // threads per token group: blockDim.x, or a part of it under a num_sms cap
    uint32_t* err;
};

// Receive arrays of the single-buffer layout: every row lives in this buffer.
struct LocalRecv {
    static constexpr bool kPeer = false;
    uint8_t* x;
    float* scale;
    int32_t* src;
    float* w;
    __device__ __forceinline__ uint8_t* x_of(int) const { return x; }
    __device__ __forceinline__ float* scale_of(int) const { return scale; }
    __device__ __forceinline__ int32_t* src_of(int) const { return src; }
    __device__ __forceinline__ float* w_of(int) const { return w; }
};

// Receive arrays of every destination rank (device pointers, peer-mapped
// where the rank is another GPU).
struct PeerRecv {
    static constexpr bool kPeer = true;
    uint8_t* x[kMaxPeers];
    float* scale[kMaxPeers];
    int32_t* src[kMaxPeers];
    float* w[kMaxPeers];
    __device__ __forceinline__ uint8_t* x_of(int d) const { return x[d]; }
    __device__ __forceinline__ float* scale_of(int d) const { return scale[d]; }
    __device__ __forceinline__ int32_t* src_of(int d) const { return src[d]; }
    __device__ __forceinline__ float* w_of(int d) const { return w[d]; }
};

constexpr int kMaxK = 32;
constexpr int kMaxSub = 8;  // token groups per CTA under a num_sms cap

// Token groups. Without a num_sms cap (G = false) a CTA is one group: one
// token at a time, __syncthreads. Under a cap (G = true) a CTA holds
// blockDim.x / p.sub_threads groups; group j of CTA b takes tokens
// b * groups + j, then strides by the grid's groups, and waits only for
// itself, on named barrier 1 + j.
template <bool G>
struct Group;
template <>
struct Group<false> {
    static constexpr int sub = 0, n = 1;
    int tid, threads;
    __device__ __forceinline__ explicit Group(int) : tid(threadIdx.x), threads(blockDim.x) {}
    __device__ __forceinline__ void sync() const { __syncthreads(); }
};
template <>
struct Group<true> {
    int sub, tid, n, threads;
    __device__ __forceinline__ explicit Group(int sub_threads)
        : sub(threadIdx.x / sub_threads),
          tid(threadIdx.x - sub * sub_threads),
          n(blockDim.x / sub_threads),
          threads(sub_threads) {}
    __device__ __forceinline__ void sync() const {
        asm volatile("bar.sync %0, %1;" ::"r"(1 + sub), "r"(threads) : "memory");
    }
};

// Loads the token's K receive rows (checked) and destination ranks, and
// writes recv_src / recv_w.
template <class Recv>
__device__ __forceinline__ void stage_rows(const DispatchParams& p, const Recv& rv, int64_t g, int32_t* s_row,
                                           int32_t* s_rank, int t) {
    if (t < p.K) {
        int32_t r = __ldg(p.dst_row + g * p.K + t);
        int d = 0;
        if constexpr (Recv::kPeer) {
            d = __ldg(p.dst_rank + g * p.K + t);
            if (r >= 0 && d >= p.num_peers) {
                set_error(p.err, EP_DEVERR_ROW_BOUNDS);
                r = -1;
            }
            s_rank[t] = d;
        }
        if (r >= p.m_max) {
            set_error(p.err, EP_DEVERR_ROW_BOUNDS);
            r = -1;
        }
        s_row[t] = r;
        if (r >= 0) {
            rv.src_of(d)[r] = (int32_t)(p.g_base + g);
            rv.w_of(d)[r] = __ldg(p.topk_w + g * p.K + t);
        }
    }
}

// The order in which the CTA writes the token's K rows: ascending
// (destination rank, row), masked rows last; s_ord[i] = the i-th slot. CTAs
// in flight hold consecutive tokens, whose rows for one expert are adjacent,
// so in this order their writes meet in fewer places at a time (measured on
// B200: prefill dispatch 687 -> 678 us). Threads t < K, after s_row / s_rank
// are visible. With many tokens in flight (a full grid, or a num_sms cap of
// at least half the SMs) the CTAs write in this order. Under a smaller cap
// each group loops over hundreds of tokens and pays the extra barrier on
// each, and slot order is faster.
template <class Recv>
__device__ __forceinline__ void order_rows(int K, const int32_t* s_row, const int32_t* s_rank, int32_t* s_ord, int t) {
    if (t < K) {
        auto key = [&](int q) -> uint64_t {
            const int32_t r = s_row[q];
            if (r < 0) return ~0ull;
            const uint64_t d = Recv::kPeer ? (uint64_t)(uint32_t)s_rank[q] : 0ull;
            return (d << 32) | (uint32_t)r;
        };
        const uint64_t me = key(t);
        int pos = 0;
        for (int q = 0; q < K; ++q) {
            const uint64_t o = key(q);
            pos += (o < me || (o == me && q < t)) ? 1 : 0;
        }
        s_ord[pos] = t;
    }
}

template <int VPT, class Recv, bool G>
__global__ void __launch_bounds__(G ? 1024 : 512) dispatch_bf16_kernel(DispatchParams p, Recv rv) {
    __shared__ int32_t s_row_all[G ? kMaxSub : 1][kMaxK];
    __shared__ int32_t s_rank_all[G ? kMaxSub : 1][Recv::kPeer ? kMaxK : 1];
    __shared__ int32_t s_ord_all[G ? kMaxSub : 1][kMaxK];
    const Group<G> grp(p.sub_threads);
    int32_t* s_row = s_row_all[grp.sub];
    int32_t* s_rank = s_rank_all[grp.sub];
    int32_t* s_ord = s_ord_all[grp.sub];
    const int nv = p.H / 16;  // 32-byte vectors per bf16 row
    const size_t rb = (size_t)p.H * 2;
    for (int64_t g = (int64_t)blockIdx.x * grp.n + grp.sub; g < p.N; g += (int64_t)gridDim.x * grp.n) {
        stage_rows(p, rv, g, s_row, s_rank, grp.tid);
        u32x8 v[VPT];
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int c = grp.tid + j * grp.threads;
            if (c < nv) v[j] = ld256_stream(p.x + g * rb + (size_t)c * 32);
        }
        grp.sync();
        if (p.ordered) {  // uniform over the grid
            order_rows<Recv>(p.K, s_row, s_rank, s_ord, grp.tid);
            grp.sync();
        }
        for (int i = 0; i < p.K; ++i) {
            const int k = p.ordered ? s_ord[i] : i;
            const int32_t r = s_row[k];
            if (r < 0) continue;
            uint8_t* dst = rv.x_of(Recv::kPeer ? s_rank[k] : 0) + (size_t)r * rb;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int c = grp.tid + j * grp.threads;
                if (c < nv) st256(dst + (size_t)c * 32, v[j]);
            }
        }
        grp.sync();  // s_row is rewritten by the next token
    }
    // Stores into peer memory reach the other GPUs before the kernel ends, so
    // a collective that follows it on the stream orders them for the readers.
    // The loop's last barrier orders every thread's stores of a group before
    // its thread 0, whose system-scope fence (cumulative) then covers the
    // group.
    if constexpr (Recv::kPeer) {
        if (grp.tid == 0) __threadfence_system();
    }
}

template <int VPT, class Recv, bool G>
__global__ void __launch_bounds__(G ? 1024 : 512) dispatch_fp8_kernel(DispatchParams p, Recv rv) {
    __shared__ int32_t s_row_all[G ? kMaxSub : 1][kMaxK];
    __shared__ int32_t s_rank_all[G ? kMaxSub : 1][Recv::kPeer ? kMaxK : 1];
    __shared__ int32_t s_ord_all[G ? kMaxSub : 1][kMaxK];
    const Group<G> grp(p.sub_threads);
    int32_t* s_row = s_row_all[grp.sub];
    int32_t* s_rank = s_rank_all[grp.sub];
    int32_t* s_ord = s_ord_all[grp.sub];
    const int nv = p.H / 16;  // 16-channel vectors per row: 32 B in, 16 B out
    const int nb = p.H / 128;
    const size_t rb_in = (size_t)p.H * 2;
    const int lane = threadIdx.x & 31;
    for (int64_t g = (int64_t)blockIdx.x * grp.n + grp.sub; g < p.N; g += (int64_t)gridDim.x * grp.n) {
        stage_rows(p, rv, g, s_row, s_rank, grp.tid);
        uint4 q[VPT];
        float sc[VPT];
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int c = grp.tid + j * grp.threads;
            const bool act = c < nv;  // uniform over each aligned group of 8 lanes
            u32x8 x = act ? ld256_stream(p.x + g * rb_in + (size_t)c * 32) : u32x8{};
            float f[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                f[2 * i] = bf16lo(x.v[i]);
                f[2 * i + 1] = bf16hi(x.v[i]);
            }
            float a = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(f[i]));
#pragma unroll
            for (int off = 4; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, off));
            const float amax = fmaxf(a, 1e-4f);
            const float inv = __fdiv_rn(448.0f, amax);
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                w[i] = pack_e4m3x2(__fmul_rn(f[4 * i], inv), __fmul_rn(f[4 * i + 1], inv)) |
                       (pack_e4m3x2(__fmul_rn(f[4 * i + 2], inv), __fmul_rn(f[4 * i + 3], inv)) << 16);
            q[j] = make_uint4(w[0], w[1], w[2], w[3]);
            sc[j] = __fdiv_rn(amax, 448.0f);
        }
        grp.sync();
        if (p.ordered) {  // uniform over the grid
            order_rows<Recv>(p.K, s_row, s_rank, s_ord, grp.tid);
            grp.sync();
        }
        for (int i = 0; i < p.K; ++i) {
            const int k = p.ordered ? s_ord[i] : i;
            const int32_t r = s_row[k];
            if (r < 0) continue;
            const int d = Recv::kPeer ? s_rank[k] : 0;
            uint8_t* dst = rv.x_of(d) + (size_t)r * p.H;
            float* scale = rv.scale_of(d);
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int c = grp.tid + j * grp.threads;
                if (c < nv) {
                    __stcs(reinterpret_cast<uint4*>(dst) + c, q[j]);
                    if ((lane & 7) == 0) scale[(size_t)r * nb + c / 8] = sc[j];
                }
            }
        }
        grp.sync();
    }
    if constexpr (Recv::kPeer) {  // as in dispatch_bf16_kernel
        if (grp.tid == 0) __threadfence_system();
    }
}

// One CTA per token (a grid-stride loop past 2^31 - 1 tokens).
template <class Recv>
cudaError_t launch_rows(void (*kernel)(DispatchParams, Recv), int threads, DispatchParams p, const Recv& rv,
                        cudaStream_t st) {
    p.sub_threads = threads;
    const unsigned grid = (unsigned)(p.N < 0x7fffffff ? p.N : 0x7fffffff);
    kernel<<<grid, threads, 0, st>>>(p, rv);
    return cudaGetLastError();
}

// Threads per CTA, a multiple of 32 and at most 512, and VPT 16-channel
// vectors per thread, for a target of `per` vectors per thread: one for bf16
// rows, two for FP8 rows (the cast gives each thread enough work to hide the
// load; measured on B200, FP8 dispatch 1569 -> 1522 us on the large shape,
// 174.5 -> 168.4 us on skewed; bf16 prefill is fastest at one).
void shape_of(int H, int per, int* threads, int* vpt) {
    const int nv = H / 16;
    int t = (nv + per - 1) / per;
    t = t < 512 ? t : 512;
    t = (t + 31) / 32 * 32;
    *threads = t;
    *vpt = (nv + t - 1) / t;
}

// Resident CTAs per SM of a kernel at a block size (queried once per pair).
cudaError_t per_sm_of(const void* fn, int threads, int* per_sm) {
    static std::mutex mu;
    static const void* fns[64] = {};
    static int thr[64] = {}, val[64] = {};
    static int n = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (fns[i] == fn && thr[i] == threads) {
            *per_sm = val[i];
            return cudaSuccess;
        }
    int v = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, fn, threads, 0);
    if (e != cudaSuccess) return e;
    if (v < 1) v = 1;
    if (n < 64) {
        fns[n] = fn;
        thr[n] = threads;
        val[n] = v;
        ++n;
    }
    *per_sm = v;
    return cudaSuccess;
}

template <class Recv, bool G>
void (*fp8_kernel_of(int vpt))(DispatchParams, Recv) {
    if (vpt <= 1) return dispatch_fp8_kernel<1, Recv, G>;
    if (vpt <= 2) return dispatch_fp8_kernel<2, Recv, G>;
    if (vpt <= 4) return dispatch_fp8_kernel<4, Recv, G>;
    return dispatch_fp8_kernel<8, Recv, G>;
}

template <class Recv, bool G>
void (*bf16_kernel_of(int vpt))(DispatchParams, Recv) {
    if (vpt <= 1) return dispatch_bf16_kernel<1, Recv, G>;
    if (vpt <= 2) return dispatch_bf16_kernel<2, Recv, G>;
    if (vpt <= 4) return dispatch_bf16_kernel<4, Recv, G>;
    return dispatch_bf16_kernel<8, Recv, G>;
}

// num_sms cap (Buffer.set_num_sms): at most sm_cap CTAs, so that no more than
// sm_cap SMs run the kernel (the block scheduler places CTAs breadth-first:
// 4 * sm_cap small CTAs would occupy 4 * sm_cap SMs). Each CTA holds as many
// token groups as fit one SM (up to 1024 threads), each group two 16-channel
// vectors per thread, so that an SM keeps as many bytes in flight as it
// would with several one-vector CTAs.
template <class Recv>
cudaError_t launch_capped(DispatchParams p, const Recv& rv, bool fp8, int sm_cap, cudaStream_t st) {
    int threads, vpt;
    shape_of(p.H, 2, &threads, &vpt);
    auto kern = fp8 ? fp8_kernel_of<Recv, true>(vpt) : bf16_kernel_of<Recv, true>(vpt);
    int per_sm = 0;
    cudaError_t e = per_sm_of((const void*)kern, threads, &per_sm);
    if (e != cudaSuccess) return e;
    int subs = per_sm < 1024 / threads ? per_sm : 1024 / threads;
    subs = subs < kMaxSub ? subs : kMaxSub;
    subs = subs > 1 ? subs : 1;
    int64_t grid = (p.N + subs - 1) / subs;
    grid = grid < sm_cap ? grid : sm_cap;
    p.sub_threads = threads;
    kern<<<(unsigned)grid, threads * subs, 0, st>>>(p, rv);
    return cudaGetLastError();
}

template <class Recv>
cudaError_t launch_any(const DispatchParams& p0, const Recv& rv, bool fp8, int sm_cap, int full_sms,
                       cudaStream_t st) {
    DispatchParams p = p0;
    p.ordered = 2 * sm_cap >= full_sms ? 1 : 0;
    if (sm_cap < full_sms) return launch_capped(p, rv, fp8, sm_cap, st);
    int threads, vpt;
    shape_of(p.H, fp8 ? 2 : 1, &threads, &vpt);
    if (!fp8) return launch_rows(bf16_kernel_of<Recv, false>(vpt), threads, p, rv, st);
    auto kern = fp8_kernel_of<Recv, false>(vpt);
    // A batch a little over one wave of CTAs (decode: 1024 tokens against
    // 888 resident CTAs of 224 threads) would leave a short second wave
    // running alone. Half as many threads with twice the vectors each fit it
    // in one wave when they can.
    int per_sm = 0;
    cudaError_t e = per_sm_of((const void*)kern, threads, &per_sm);
    if (e != cudaSuccess) return e;
    const int64_t wave = (int64_t)per_sm * full_sms;
    if (p.N > wave && p.N <= 2 * wave) {
        int t4, v4;
        shape_of(p.H, 4, &t4, &v4);
        auto k4 = fp8_kernel_of<Recv, false>(v4);
        int per4 = 0;
        e = per_sm_of((const void*)k4, t4, &per4);
        if (e != cudaSuccess) return e;
        if (p.N <= (int64_t)per4 * full_sms) return launch_rows(k4, t4, p, rv, st);
    }
    return launch_rows(kern, threads, p, rv, st);
}

DispatchParams params_of(const ep_buffer& b, int64_t N, const void* x) {
    const ep_config_t& c = b.cfg;
    DispatchParams p{};
    p.N = N;
    p.K = c.topk;
    p.H = c.hidden;
    p.m_max = b.m_max;
    p.x = static_cast<const uint8_t*>(x);
    p.dst_row = b.dst_row;
    p.topk_w = b.topk_w;
    p.err = b.err;
    return p;
}

int sm_cap_of(const ep_buffer& b) {
    const ep_config_t& c = b.cfg;
    return (c.num_sms > 0 && c.num_sms < b.sm_count) ? c.num_sms : b.sm_count;
}

}  // namespace

cudaError_t launch_dispatch(const ep_buffer& b, int T, const void* x, cudaStream_t st) {
    const DispatchParams p = params_of(b, (int64_t)b.cfg.num_ranks * T, x);
    if (p.N == 0) return cudaSuccess;
    LocalRecv rv{static_cast<uint8_t*>(b.recv_x), b.recv_scale, b.recv_src, b.recv_w};
    return launch_any(p, rv, (b.cfg.flags & EP_FLAG_FP8) != 0, sm_cap_of(b), b.sm_count, st);
}

cudaError_t launch_shard_dispatch(const ep_buffer& b, int rank, int T, const void* x, void* const* peer_x,
                                  float* const* peer_scale, int32_t* const* peer_src, float* const* peer_w,
                                  cudaStream_t st) {
    DispatchParams p = params_of(b, T, x);
    if (p.N == 0) return cudaSuccess;
    p.dst_rank = b.dst_rank;
    p.num_peers = b.cfg.num_ranks;
    p.g_base = (int64_t)rank * T;
    PeerRecv rv{};
    for (int d = 0; d < b.cfg.num_ranks; ++d) {
        rv.x[d] = static_cast<uint8_t*>(peer_x[d]);
        rv.scale[d] = peer_scale ? peer_scale[d] : nullptr;
        rv.src[d] = peer_src[d];
        rv.w[d] = peer_w[d];
    }
    return launch_any(p, rv, (b.cfg.flags & EP_FLAG_FP8) != 0, sm_cap_of(b), b.sm_count, st);
}

}  // namespace ep
