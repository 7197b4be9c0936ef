// Dispatch (sm_100a): scatter each token's hidden vector to the receive row
// of every unmasked slot. Only target experts get a copy
// ("DeepEP：年度总结中的计算通信重叠摘记", §节点内通信: is_token_in_rank, no
// full all-to-all). The optional FP8 cast sends 1 byte per element instead of
// 2 (same section) and adds one fp32 scale per 128 channels.
//
// One CTA per token (a grid-stride loop when num_sms caps the grid). The
// threads read the token's row once into registers with 256-bit loads, then
// write it to each of the K receive rows:
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
#include <cuda_runtime.h>

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
    uint8_t* recv_x;
    float* recv_scale;
    int32_t* recv_src;
    float* recv_w;
    uint32_t* err;
};

constexpr int kMaxK = 32;

// Loads the token's K receive rows (checked) and writes recv_src / recv_w.
__device__ __forceinline__ void stage_rows(const DispatchParams& p, int64_t g, int32_t* s_row) {
    const int t = threadIdx.x;
    if (t < p.K) {
        int32_t r = __ldg(p.dst_row + g * p.K + t);
        if (r >= p.m_max) {
            set_error(p.err, EP_DEVERR_ROW_BOUNDS);
            r = -1;
        }
        s_row[t] = r;
        if (r >= 0) {
            p.recv_src[r] = (int32_t)g;
            p.recv_w[r] = __ldg(p.topk_w + g * p.K + t);
        }
    }
}

template <int VPT>
__global__ void __launch_bounds__(512) dispatch_bf16_kernel(DispatchParams p) {
    __shared__ int32_t s_row[kMaxK];
    const int nv = p.H / 16;  // 32-byte vectors per bf16 row
    const size_t rb = (size_t)p.H * 2;
    for (int64_t g = blockIdx.x; g < p.N; g += gridDim.x) {
        stage_rows(p, g, s_row);
        u32x8 v[VPT];
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int c = threadIdx.x + j * blockDim.x;
            if (c < nv) v[j] = ld256_stream(p.x + g * rb + (size_t)c * 32);
        }
        __syncthreads();
        for (int k = 0; k < p.K; ++k) {
            const int32_t r = s_row[k];
            if (r < 0) continue;
            uint8_t* dst = p.recv_x + (size_t)r * rb;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int c = threadIdx.x + j * blockDim.x;
                if (c < nv) st256(dst + (size_t)c * 32, v[j]);
            }
        }
        __syncthreads();  // s_row is rewritten by the next token
    }
}

template <int VPT>
__global__ void __launch_bounds__(512) dispatch_fp8_kernel(DispatchParams p) {
    __shared__ int32_t s_row[kMaxK];
    const int nv = p.H / 16;  // 16-channel vectors per row: 32 B in, 16 B out
    const int nb = p.H / 128;
    const size_t rb_in = (size_t)p.H * 2;
    const int lane = threadIdx.x & 31;
    for (int64_t g = blockIdx.x; g < p.N; g += gridDim.x) {
        stage_rows(p, g, s_row);
        uint4 q[VPT];
        float sc[VPT];
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int c = threadIdx.x + j * blockDim.x;
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
        __syncthreads();
        for (int k = 0; k < p.K; ++k) {
            const int32_t r = s_row[k];
            if (r < 0) continue;
            uint8_t* dst = p.recv_x + (size_t)r * p.H;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int c = threadIdx.x + j * blockDim.x;
                if (c < nv) {
                    __stcs(reinterpret_cast<uint4*>(dst) + c, q[j]);
                    if ((lane & 7) == 0) p.recv_scale[(size_t)r * nb + c / 8] = sc[j];
                }
            }
        }
        __syncthreads();
    }
}

template <typename KernelT>
cudaError_t launch_rows(KernelT kernel, int threads, int sm_cap, int full_sms, const DispatchParams& p,
                        cudaStream_t st) {
    int64_t grid = p.N;
    if (sm_cap < full_sms) {
        // num_sms cap (Buffer.set_num_sms): a resident grid on sm_cap SMs' worth of CTAs
        int per_sm = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0);
        if (e != cudaSuccess) return e;
        grid = (int64_t)sm_cap * (per_sm > 0 ? per_sm : 1);
        if (grid > p.N) grid = p.N;
    }
    if (grid > 0x7fffffff) grid = 0x7fffffff;
    kernel<<<(unsigned)grid, threads, 0, st>>>(p);
    return cudaGetLastError();
}

// Threads per CTA: one 16-channel vector per thread, at most 512 threads
// (a multiple of 32). VPT vectors per thread cover the rest.
void shape_of(int H, int* threads, int* vpt) {
    const int nv = H / 16;
    int t = nv < 512 ? nv : 512;
    t = (t + 31) / 32 * 32;
    *threads = t;
    *vpt = (nv + t - 1) / t;
}

}  // namespace

cudaError_t launch_dispatch(const ep_buffer& b, int T, const void* x, cudaStream_t st) {
    const ep_config_t& c = b.cfg;
    DispatchParams p{};
    p.N = (int64_t)c.num_ranks * T;
    p.K = c.topk;
    p.H = c.hidden;
    p.m_max = b.m_max;
    p.x = static_cast<const uint8_t*>(x);
    p.dst_row = b.dst_row;
    p.topk_w = b.topk_w;
    p.recv_x = static_cast<uint8_t*>(b.recv_x);
    p.recv_scale = b.recv_scale;
    p.recv_src = b.recv_src;
    p.recv_w = b.recv_w;
    p.err = b.err;
    if (p.N == 0) return cudaSuccess;
    const int sm_cap = (c.num_sms > 0 && c.num_sms < b.sm_count) ? c.num_sms : b.sm_count;
    int threads, vpt;
    shape_of(p.H, &threads, &vpt);
    if (!(c.flags & EP_FLAG_FP8)) {
        if (vpt <= 1) return launch_rows(dispatch_bf16_kernel<1>, threads, sm_cap, b.sm_count, p, st);
        if (vpt <= 2) return launch_rows(dispatch_bf16_kernel<2>, threads, sm_cap, b.sm_count, p, st);
        if (vpt <= 4) return launch_rows(dispatch_bf16_kernel<4>, threads, sm_cap, b.sm_count, p, st);
        return launch_rows(dispatch_bf16_kernel<8>, threads, sm_cap, b.sm_count, p, st);
    }
    if (vpt <= 1) return launch_rows(dispatch_fp8_kernel<1>, threads, sm_cap, b.sm_count, p, st);
    if (vpt <= 2) return launch_rows(dispatch_fp8_kernel<2>, threads, sm_cap, b.sm_count, p, st);
    if (vpt <= 4) return launch_rows(dispatch_fp8_kernel<4>, threads, sm_cap, b.sm_count, p, st);
    return launch_rows(dispatch_fp8_kernel<8>, threads, sm_cap, b.sm_count, p, st);
}

}  // namespace ep
