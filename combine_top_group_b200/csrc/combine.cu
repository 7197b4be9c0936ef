// Combine (sm_100a): gather every token's expert outputs back into token
// order as a top-k weighted sum ("DeepEP：面向MoE的高吞吐低延迟GPU通信库",
// §工程化: dispatch and combine).
//   out[g][h] = bf16_rne( fma(w[g,K-1], y[r_{K-1}][h], ... fma(w[g,0], y[r_0][h], 0)) )
// The chain runs in fp32, slot by slot in ascending k, and skips masked
// slots. FP8 expert outputs are dequantised in the same pass: e4m3 * scale
// in fp32.
//
// One CTA per token. Each thread owns a 16-byte column vector of y (8 bf16
// or 16 e4m3 channels). It issues the K gathers of that column before any
// arithmetic, so K loads are in flight per thread. Loads use the streaming
// cache hint (y is read once) and so do the output stores.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace ep {
namespace {

constexpr int kCombineThreads = 128;

struct CombineParams {
    int64_t N;
    int K, H;
    int64_t m_max;
    const uint8_t* y;
    const float* y_scale;
    const int32_t* dst_row;
    const float* topk_w;
    uint8_t* out;
    uint32_t* err;
};

template <int KMAX>
__device__ __forceinline__ void load_slots(const CombineParams& p, int64_t g, int32_t (&row)[KMAX],
                                           float (&w)[KMAX]) {
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        row[k] = -1;
        w[k] = 0.0f;
        if (k < p.K) {
            int32_t r = __ldg(p.dst_row + g * p.K + k);
            if (r >= p.m_max) r = -1;  // reported by the block's thread 0 below
            row[k] = r;
            w[k] = __ldg(p.topk_w + g * p.K + k);
        }
    }
}

template <int KMAX>
__global__ void __launch_bounds__(kCombineThreads) combine_bf16_kernel(CombineParams p) {
    const int64_t g = blockIdx.x;
    int32_t row[KMAX];
    float w[KMAX];
    load_slots<KMAX>(p, g, row, w);
    if (threadIdx.x == 0)
        for (int k = 0; k < p.K; ++k)
            if (__ldg(p.dst_row + g * p.K + k) >= p.m_max) set_error(p.err, EP_DEVERR_ROW_BOUNDS);
    const int nvec = p.H / 8;
    const size_t rb = (size_t)p.H * 2;
    for (int v = threadIdx.x; v < nvec; v += kCombineThreads) {
        uint4 q[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            q[k] = make_uint4(0, 0, 0, 0);
            if (row[k] >= 0) q[k] = __ldcs(reinterpret_cast<const uint4*>(p.y + (size_t)row[k] * rb) + v);
        }
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            if (row[k] >= 0) {
                const uint32_t u[4] = {q[k].x, q[k].y, q[k].z, q[k].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[2 * j] = __fmaf_rn(w[k], bf16lo(u[j]), acc[2 * j]);
                    acc[2 * j + 1] = __fmaf_rn(w[k], bf16hi(u[j]), acc[2 * j + 1]);
                }
            }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        __stcs(reinterpret_cast<uint4*>(p.out + (size_t)g * rb) + v, o);
    }
}

template <int KMAX>
__global__ void __launch_bounds__(kCombineThreads) combine_fp8_kernel(CombineParams p) {
    const int64_t g = blockIdx.x;
    int32_t row[KMAX];
    float w[KMAX];
    load_slots<KMAX>(p, g, row, w);
    if (threadIdx.x == 0)
        for (int k = 0; k < p.K; ++k)
            if (__ldg(p.dst_row + g * p.K + k) >= p.m_max) set_error(p.err, EP_DEVERR_ROW_BOUNDS);
    const int nvec = p.H / 16;  // 16 e4m3 channels per vector
    const int nb = p.H / 128;
    const size_t rb = (size_t)p.H;
    for (int v = threadIdx.x; v < nvec; v += kCombineThreads) {
        uint4 q[KMAX];
        float sc[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            q[k] = make_uint4(0, 0, 0, 0);
            sc[k] = 0.0f;
            if (row[k] >= 0) {
                q[k] = __ldcs(reinterpret_cast<const uint4*>(p.y + (size_t)row[k] * rb) + v);
                sc[k] = __ldg(p.y_scale + (size_t)row[k] * nb + (v * 16) / 128);
            }
        }
        float acc[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            if (row[k] >= 0) {
                const uint32_t u[4] = {q[k].x, q[k].y, q[k].z, q[k].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 a = unpack_e4m3x2(u[j] & 0xffffu);
                    const float2 b = unpack_e4m3x2(u[j] >> 16);
                    acc[4 * j + 0] = __fmaf_rn(w[k], __fmul_rn(a.x, sc[k]), acc[4 * j + 0]);
                    acc[4 * j + 1] = __fmaf_rn(w[k], __fmul_rn(a.y, sc[k]), acc[4 * j + 1]);
                    acc[4 * j + 2] = __fmaf_rn(w[k], __fmul_rn(b.x, sc[k]), acc[4 * j + 2]);
                    acc[4 * j + 3] = __fmaf_rn(w[k], __fmul_rn(b.y, sc[k]), acc[4 * j + 3]);
                }
            }
        }
        uint4 o0, o1;
        o0.x = pack_bf16x2(acc[0], acc[1]);
        o0.y = pack_bf16x2(acc[2], acc[3]);
        o0.z = pack_bf16x2(acc[4], acc[5]);
        o0.w = pack_bf16x2(acc[6], acc[7]);
        o1.x = pack_bf16x2(acc[8], acc[9]);
        o1.y = pack_bf16x2(acc[10], acc[11]);
        o1.z = pack_bf16x2(acc[12], acc[13]);
        o1.w = pack_bf16x2(acc[14], acc[15]);
        uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)g * p.H * 2) + 2 * v;
        __stcs(dst, o0);
        __stcs(dst + 1, o1);
    }
}

}  // namespace

cudaError_t launch_combine(const ep_buffer& b, int T, const void* y, const float* y_scale, void* out,
                           cudaStream_t st) {
    const ep_config_t& c = b.cfg;
    CombineParams p{};
    p.N = (int64_t)c.num_ranks * T;
    p.K = c.topk;
    p.H = c.hidden;
    p.m_max = b.m_max;
    p.y = static_cast<const uint8_t*>(y);
    p.y_scale = y_scale;
    p.dst_row = b.dst_row;
    p.topk_w = b.topk_w;
    p.out = static_cast<uint8_t*>(out);
    p.err = b.err;
    if (p.N == 0) return cudaSuccess;
    const unsigned grid = (unsigned)p.N;
    if (y_scale == nullptr) {
        if (p.K <= 4) combine_bf16_kernel<4><<<grid, kCombineThreads, 0, st>>>(p);
        else if (p.K <= 8) combine_bf16_kernel<8><<<grid, kCombineThreads, 0, st>>>(p);
        else combine_bf16_kernel<32><<<grid, kCombineThreads, 0, st>>>(p);
    } else {
        if (p.K <= 4) combine_fp8_kernel<4><<<grid, kCombineThreads, 0, st>>>(p);
        else if (p.K <= 8) combine_fp8_kernel<8><<<grid, kCombineThreads, 0, st>>>(p);
        else combine_fp8_kernel<32><<<grid, kCombineThreads, 0, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace ep
