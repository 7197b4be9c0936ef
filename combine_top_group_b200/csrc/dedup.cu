// Deduplicated (per destination rank) receive (sm_100a), after the pages'
// only-to-target-ranks rule ("DeepEP：年度总结中的计算通信重叠摘记",
// §节点内通信: is_token_in_rank, and no full all-to-all). A token crosses to a
// rank once, however many of that rank's experts it chose. The receiving
// rank then permutes rows into expert order, reduces its experts' outputs
// into one bf16 partial per (token, rank), and the partials are summed
// across ranks.
//   dispatch_dedup: x[g] -> dd_x[tok_row[g][r]] (bf16, or the same FP8 cast
//                   as dispatch), plus the token id and its top-k localised
//                   to rank r.
//   permute:        dd_x[d] -> recv_x[dst_row[g][k]] for each of the row's
//                   local slots: the same expert-grouped buffers dispatch
//                   writes.
//   local_reduce:   partial[d] = bf16( fma chain over the row's local slots,
//                   k ascending, of w * y[dst_row[g][k]] ).
//   combine_dedup:  out[g] = bf16( fp32 sum over ranks r ascending of
//                   partial[tok_row[g][r]] ).
// One CTA per token (grid-stride when num_sms caps the grid). The row
// vectors are the same 256-bit (bf16) / 16-channel (e4m3) units as
// dispatch.cu and combine.cu.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace ep {
namespace {

constexpr int kMaxRK = 32;
constexpr int kThreads = 128;    // permute / reduce / combine
constexpr int kReduceBatch = 4;  // local_reduce: gathers in flight per thread

struct DedupParams {
    int64_t N;
    int R, K, H, E, L;
    int64_t d_max, m_max;
    const uint8_t* x;
    const int32_t* topk_idx;
    const float* topk_w;
    const int32_t* dst_row;
    const int32_t* tok_row;
    uint8_t* dd_x;
    float* dd_scale;
    int32_t* dd_src;
    int32_t* dd_topk_idx;
    float* dd_topk_w;
    uint8_t* recv_x;
    float* recv_scale;
    int32_t* recv_src;
    float* recv_w;
    const uint8_t* y;
    const float* y_scale;
    uint16_t* partial;
    uint8_t* out;
    int fp8;
    uint32_t* err;
};

__device__ __forceinline__ int32_t checked(int32_t r, int64_t cap, uint32_t* err) {
    if (r >= cap) {
        set_error(err, EP_DEVERR_ROW_BOUNDS);
        return -1;
    }
    return r;
}

// ---------------------------------------------------------------------------
// dispatch_dedup
// ---------------------------------------------------------------------------
template <int VPT, bool FP8>
__global__ void __launch_bounds__(512) dispatch_dedup_kernel(DedupParams p) {
    __shared__ int32_t s_row[kMaxRK];
    const int nv = p.H / 16;  // 16-channel vectors
    const int nb = p.H / 128;
    const size_t rb_in = (size_t)p.H * 2;
    const int lane = threadIdx.x & 31;
    for (int64_t g = blockIdx.x; g < p.N; g += gridDim.x) {
        if (threadIdx.x < p.R) {
            const int32_t d = checked(__ldg(p.tok_row + g * p.R + threadIdx.x), p.d_max, p.err);
            s_row[threadIdx.x] = d;
            if (d >= 0) p.dd_src[d] = (int32_t)g;
        }
        for (int i = threadIdx.x; i < p.R * p.K; i += blockDim.x) {
            const int r = i / p.K, k = i % p.K;
            const int32_t d = __ldg(p.tok_row + g * p.R + r);
            if (d < 0 || d >= p.d_max) continue;
            const int e = __ldg(p.topk_idx + g * p.K + k);
            const bool here = e >= 0 && e < p.E && e / p.L == r;
            p.dd_topk_idx[(int64_t)d * p.K + k] = here ? e : -1;
            p.dd_topk_w[(int64_t)d * p.K + k] = here ? __ldg(p.topk_w + g * p.K + k) : 0.0f;
        }
        if constexpr (!FP8) {
            u32x8 v[VPT];
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int c = threadIdx.x + j * blockDim.x;
                if (c < nv) v[j] = ld256_stream(p.x + g * rb_in + (size_t)c * 32);
            }
            __syncthreads();
            for (int r = 0; r < p.R; ++r) {
                const int32_t d = s_row[r];
                if (d < 0) continue;
                uint8_t* dst = p.dd_x + (size_t)d * rb_in;
#pragma unroll
                for (int j = 0; j < VPT; ++j) {
                    const int c = threadIdx.x + j * blockDim.x;
                    if (c < nv) st256(dst + (size_t)c * 32, v[j]);
                }
            }
        } else {
            uint4 q[VPT];
            float sc[VPT];
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int c = threadIdx.x + j * blockDim.x;
                const bool act = c < nv;  // uniform over each aligned group of 8 lanes
                u32x8 xv = act ? ld256_stream(p.x + g * rb_in + (size_t)c * 32) : u32x8{};
                float f[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    f[2 * i] = bf16lo(xv.v[i]);
                    f[2 * i + 1] = bf16hi(xv.v[i]);
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
            __syncthreads();
            for (int r = 0; r < p.R; ++r) {
                const int32_t d = s_row[r];
                if (d < 0) continue;
                uint8_t* dst = p.dd_x + (size_t)d * p.H;
#pragma unroll
                for (int j = 0; j < VPT; ++j) {
                    const int c = threadIdx.x + j * blockDim.x;
                    if (c < nv) {
                        __stcs(reinterpret_cast<uint4*>(dst) + c, q[j]);
                        if ((lane & 7) == 0) p.dd_scale[(size_t)d * nb + c / 8] = sc[j];
                    }
                }
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// permute: dedup rows -> expert-grouped rows. Each (token, rank) row is read
// once into registers (256-bit) and written to every local slot's row.
// ---------------------------------------------------------------------------
template <int VPT>
__global__ void __launch_bounds__(512) permute_kernel(DedupParams p) {
    __shared__ int32_t s_d[kMaxRK];     // dedup row of the token on rank r
    __shared__ int32_t s_dst[kMaxRK];   // expert row of slot k (-1: not local / masked)
    __shared__ int32_t s_rank[kMaxRK];  // rank of slot k's expert
    const int nb = p.H / 128;
    const size_t rb = p.fp8 ? (size_t)p.H : (size_t)p.H * 2;
    const int nv = (int)(rb / 32);  // 32-byte vectors per row
    for (int64_t g = blockIdx.x; g < p.N; g += gridDim.x) {
        if (threadIdx.x < p.R) s_d[threadIdx.x] = checked(__ldg(p.tok_row + g * p.R + threadIdx.x), p.d_max, p.err);
        __syncthreads();
        if (threadIdx.x < p.K) {
            const int k = threadIdx.x;
            int32_t dst = -1, r = -1;
            const int e = __ldg(p.topk_idx + g * p.K + k);
            if (e >= 0 && e < p.E) {
                r = e / p.L;
                const int32_t d = s_d[r];
                // the receiving rank's own view: slot k is local to this row
                if (d >= 0 && p.dd_topk_idx[(int64_t)d * p.K + k] >= 0) {
                    dst = checked(__ldg(p.dst_row + g * p.K + k), p.m_max, p.err);
                    if (dst >= 0) {
                        p.recv_src[dst] = p.dd_src[d];
                        p.recv_w[dst] = p.dd_topk_w[(int64_t)d * p.K + k];
                    }
                }
            }
            s_dst[k] = dst;
            s_rank[k] = r;
        }
        __syncthreads();
        for (int r = 0; r < p.R; ++r) {
            const int32_t d = s_d[r];
            if (d < 0) continue;  // uniform
            u32x8 v[VPT];
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int c = threadIdx.x + j * blockDim.x;
                if (c < nv) v[j] = ld256_stream(p.dd_x + (size_t)d * rb + (size_t)c * 32);
            }
            for (int k = 0; k < p.K; ++k) {
                if (s_rank[k] != r || s_dst[k] < 0) continue;
                uint8_t* dst = p.recv_x + (size_t)s_dst[k] * rb;
#pragma unroll
                for (int j = 0; j < VPT; ++j) {
                    const int c = threadIdx.x + j * blockDim.x;
                    if (c < nv) st256(dst + (size_t)c * 32, v[j]);
                }
                if (p.fp8)
                    for (int i = threadIdx.x; i < nb; i += blockDim.x)
                        p.recv_scale[(size_t)s_dst[k] * nb + i] = p.dd_scale[(size_t)d * nb + i];
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// local_reduce: per (token, rank) weighted sum of that rank's expert outputs
// ---------------------------------------------------------------------------
template <bool FP8>
__global__ void __launch_bounds__(kThreads) local_reduce_kernel(DedupParams p) {
    __shared__ int32_t s_d[kMaxRK];
    __shared__ int32_t s_row[kMaxRK];  // the row's local slots, compacted, k ascending
    __shared__ float s_w[kMaxRK];
    __shared__ int s_nl;
    const int nvec = p.H / 16;  // 16 channels per thread: 32 B of bf16 y, or 16 B of e4m3 y
    const int nb = p.H / 128;
    for (int64_t g = blockIdx.x; g < p.N; g += gridDim.x) {
        if (threadIdx.x < p.R) s_d[threadIdx.x] = checked(__ldg(p.tok_row + g * p.R + threadIdx.x), p.d_max, p.err);
        __syncthreads();
        for (int r = 0; r < p.R; ++r) {
            const int32_t d = s_d[r];
            if (d < 0) continue;  // uniform
            if (threadIdx.x < 32) {  // warp 0 compacts the row's local slots (K <= 32)
                const int k = threadIdx.x;
                int32_t row = -1;
                if (k < p.K && p.dd_topk_idx[(int64_t)d * p.K + k] >= 0)
                    row = checked(__ldg(p.dst_row + g * p.K + k), p.m_max, p.err);
                const unsigned here = __ballot_sync(FULL, row >= 0);
                if (row >= 0) {
                    const int pos = __popc(here & ((1u << k) - 1u));
                    s_row[pos] = row;
                    s_w[pos] = p.dd_topk_w[(int64_t)d * p.K + k];
                }
                if (k == 0) s_nl = __popc(here);
            }
            __syncthreads();
            const int nl = s_nl;
            for (int v = threadIdx.x; v < nvec; v += kThreads) {
                float acc[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
                // up to kReduceBatch gathers in flight per thread; the fma chain
                // still runs over the slots in ascending k
                for (int i0 = 0; i0 < nl; i0 += kReduceBatch) {
                    if constexpr (!FP8) {
                        u32x8 q[kReduceBatch];
#pragma unroll
                        for (int i = 0; i < kReduceBatch; ++i)
                            if (i0 + i < nl) q[i] = ld256_stream(p.y + (size_t)s_row[i0 + i] * p.H * 2 + (size_t)v * 32);
#pragma unroll
                        for (int i = 0; i < kReduceBatch; ++i) {
                            if (i0 + i >= nl) break;
                            const float w = s_w[i0 + i];
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                acc[2 * j] = __fmaf_rn(w, bf16lo(q[i].v[j]), acc[2 * j]);
                                acc[2 * j + 1] = __fmaf_rn(w, bf16hi(q[i].v[j]), acc[2 * j + 1]);
                            }
                        }
                    } else {
                        uint4 q[kReduceBatch];
                        float sc[kReduceBatch];
#pragma unroll
                        for (int i = 0; i < kReduceBatch; ++i) {
                            if (i0 + i < nl) {
                                const int32_t row = s_row[i0 + i];
                                q[i] = __ldcs(reinterpret_cast<const uint4*>(p.y + (size_t)row * p.H) + v);
                                sc[i] = __ldg(p.y_scale + (size_t)row * nb + v / 8);
                            }
                        }
#pragma unroll
                        for (int i = 0; i < kReduceBatch; ++i) {
                            if (i0 + i >= nl) break;
                            const float w = s_w[i0 + i];
                            const uint32_t u[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float2 a = unpack_e4m3x2(u[j] & 0xffffu);
                                const float2 b = unpack_e4m3x2(u[j] >> 16);
                                acc[4 * j + 0] = __fmaf_rn(w, __fmul_rn(a.x, sc[i]), acc[4 * j + 0]);
                                acc[4 * j + 1] = __fmaf_rn(w, __fmul_rn(a.y, sc[i]), acc[4 * j + 1]);
                                acc[4 * j + 2] = __fmaf_rn(w, __fmul_rn(b.x, sc[i]), acc[4 * j + 2]);
                                acc[4 * j + 3] = __fmaf_rn(w, __fmul_rn(b.y, sc[i]), acc[4 * j + 3]);
                            }
                        }
                    }
                }
                u32x8 o;
#pragma unroll
                for (int j = 0; j < 8; ++j) o.v[j] = pack_bf16x2(acc[2 * j], acc[2 * j + 1]);
                st256(reinterpret_cast<uint8_t*>(p.partial) + (size_t)d * p.H * 2 + (size_t)v * 32, o);
            }
            __syncthreads();
        }
        __syncthreads();  // s_d is rewritten by the next token
    }
}

// ---------------------------------------------------------------------------
// combine_dedup: sum the bf16 partials across ranks
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) combine_dedup_kernel(DedupParams p) {
    __shared__ int32_t s_d[kMaxRK];
    const int nvec = p.H / 16;
    for (int64_t g = blockIdx.x; g < p.N; g += gridDim.x) {
        if (threadIdx.x < p.R) s_d[threadIdx.x] = checked(__ldg(p.tok_row + g * p.R + threadIdx.x), p.d_max, p.err);
        __syncthreads();
        for (int v = threadIdx.x; v < nvec; v += kThreads) {
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
            for (int r = 0; r < p.R; ++r) {
                const int32_t d = s_d[r];
                if (d < 0) continue;
                const u32x8 q = ld256_stream(reinterpret_cast<const uint8_t*>(p.partial) + (size_t)d * p.H * 2 +
                                             (size_t)v * 32);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    acc[2 * j] = __fadd_rn(acc[2 * j], bf16lo(q.v[j]));
                    acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1], bf16hi(q.v[j]));
                }
            }
            u32x8 o;
#pragma unroll
            for (int j = 0; j < 8; ++j) o.v[j] = pack_bf16x2(acc[2 * j], acc[2 * j + 1]);
            st256(p.out + (size_t)g * p.H * 2 + (size_t)v * 32, o);
        }
        __syncthreads();
    }
}

DedupParams params_of(const ep_buffer& b, int T) {
    const ep_config_t& c = b.cfg;
    DedupParams p{};
    p.N = (int64_t)c.num_ranks * T;
    p.R = c.num_ranks;
    p.K = c.topk;
    p.H = c.hidden;
    p.E = c.num_experts;
    p.L = c.num_experts / c.num_ranks;
    p.d_max = b.d_max;
    p.m_max = b.m_max;
    p.topk_idx = b.topk_idx;
    p.topk_w = b.topk_w;
    p.dst_row = b.dst_row;
    p.tok_row = b.tok_row;
    p.dd_x = static_cast<uint8_t*>(b.dd_x);
    p.dd_scale = b.dd_scale;
    p.dd_src = b.dd_src;
    p.dd_topk_idx = b.dd_topk_idx;
    p.dd_topk_w = b.dd_topk_w;
    p.recv_x = static_cast<uint8_t*>(b.recv_x);
    p.recv_scale = b.recv_scale;
    p.recv_src = b.recv_src;
    p.recv_w = b.recv_w;
    p.partial = b.partial;
    p.fp8 = (c.flags & EP_FLAG_FP8) ? 1 : 0;
    p.err = b.err;
    return p;
}

template <typename KernelT>
cudaError_t launch_tokens(KernelT kernel, int threads, const ep_buffer& b, const DedupParams& p, cudaStream_t st) {
    int64_t grid = p.N;
    // num_sms cap (Buffer.set_num_sms): at most sm_cap CTAs, so that no more
    // than sm_cap SMs run the kernel (the block scheduler places CTAs
    // breadth-first); each loops over tokens. One CTA of the usual size per
    // SM, not the several an SM could hold.
    const int sm_cap = (b.cfg.num_sms > 0 && b.cfg.num_sms < b.sm_count) ? b.cfg.num_sms : b.sm_count;
    if (sm_cap < b.sm_count && grid > sm_cap) grid = sm_cap;
    if (grid > 0x7fffffff) grid = 0x7fffffff;
    if (grid < 1) return cudaSuccess;
    kernel<<<(unsigned)grid, threads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dispatch_dedup(const ep_buffer& b, int T, const void* x, cudaStream_t st) {
    DedupParams p = params_of(b, T);
    p.x = static_cast<const uint8_t*>(x);
    if (p.N == 0) return cudaSuccess;
    const int nv = p.H / 16;
    int threads = nv < 512 ? nv : 512;
    threads = (threads + 31) / 32 * 32;
    const int vpt = (nv + threads - 1) / threads;
    if (!p.fp8) {
        if (vpt <= 1) return launch_tokens(dispatch_dedup_kernel<1, false>, threads, b, p, st);
        if (vpt <= 2) return launch_tokens(dispatch_dedup_kernel<2, false>, threads, b, p, st);
        if (vpt <= 4) return launch_tokens(dispatch_dedup_kernel<4, false>, threads, b, p, st);
        return launch_tokens(dispatch_dedup_kernel<8, false>, threads, b, p, st);
    }
    if (vpt <= 1) return launch_tokens(dispatch_dedup_kernel<1, true>, threads, b, p, st);
    if (vpt <= 2) return launch_tokens(dispatch_dedup_kernel<2, true>, threads, b, p, st);
    if (vpt <= 4) return launch_tokens(dispatch_dedup_kernel<4, true>, threads, b, p, st);
    return launch_tokens(dispatch_dedup_kernel<8, true>, threads, b, p, st);
}

cudaError_t launch_permute(const ep_buffer& b, int T, cudaStream_t st) {
    DedupParams p = params_of(b, T);
    if (p.N == 0) return cudaSuccess;
    const int nv = (int)((p.fp8 ? (size_t)p.H : (size_t)p.H * 2) / 32);
    int threads = nv < 512 ? nv : 512;
    threads = (threads + 31) / 32 * 32;
    const int vpt = (nv + threads - 1) / threads;
    if (vpt <= 1) return launch_tokens(permute_kernel<1>, threads, b, p, st);
    if (vpt <= 2) return launch_tokens(permute_kernel<2>, threads, b, p, st);
    if (vpt <= 4) return launch_tokens(permute_kernel<4>, threads, b, p, st);
    return launch_tokens(permute_kernel<8>, threads, b, p, st);
}

cudaError_t launch_local_reduce(const ep_buffer& b, int T, const void* y, const float* y_scale, cudaStream_t st) {
    DedupParams p = params_of(b, T);
    p.y = static_cast<const uint8_t*>(y);
    p.y_scale = y_scale;
    if (p.N == 0) return cudaSuccess;
    if (y_scale != nullptr) return launch_tokens(local_reduce_kernel<true>, kThreads, b, p, st);
    return launch_tokens(local_reduce_kernel<false>, kThreads, b, p, st);
}

cudaError_t launch_combine_dedup(const ep_buffer& b, int T, void* out, cudaStream_t st) {
    DedupParams p = params_of(b, T);
    p.out = static_cast<uint8_t*>(out);
    if (p.N == 0) return cudaSuccess;
    return launch_tokens(combine_dedup_kernel, kThreads, b, p, st);
}

}  // namespace ep
