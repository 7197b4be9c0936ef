// Combine (sm_100a): gather every token's expert outputs back into token
// order as a top-k weighted sum ("DeepEP：面向MoE的高吞吐低延迟GPU通信库",
// §工程化: dispatch and combine).
//   out[g][h] = bf16_rne( fma(w[g,K-1], y[r_{K-1}][h], ... fma(w[g,0], y[r_0][h], 0)) )
// The chain runs in fp32, slot by slot in ascending k, and skips masked
// slots. FP8 expert outputs are dequantised in the same pass: e4m3 * scale
// in fp32.
//
// One CTA per token (a grid-stride loop when num_sms caps the grid). Each
// thread owns 16 channels of y at a time: a 32-byte vector of
// bf16 (256-bit load) or a 16-byte vector of e4m3. It issues the K gathers of
// that column before any arithmetic, so K loads are in flight per thread.
// Loads use the streaming cache hint (y is read once). The 32 output bytes
// go out in one 256-bit store.
//
// The same kernels serve one rank of a one-process-per-GPU deployment (PeerY):
// each slot's row is then read from the expert output of its destination
// rank, through a table of that rank's device pointers (peer memory over
// NVLink on a multi-GPU node).
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace ep {
namespace {

// Threads per CTA (one token per CTA). bf16 y: 4 warps, 4 CTAs per SM at 128
// registers; 64, 192 and 256 threads were no faster on B200 over 1k-33k
// tokens. e4m3 y (fused dequantisation, issue-bound): 2 warps, 12 CTAs per SM
// at 80 registers; 1715 -> 1604 us against 4 warps on the large shape.
constexpr int kBf16Threads = 128;
constexpr int kFp8Threads = 64;

struct CombineParams {
    int64_t N;
    int K, H;
    int64_t m_max;
    const uint8_t* y;
    const float* y_scale;
    const int32_t* dst_row;
    const float* topk_w;
    const uint8_t* dst_rank;  // [N, K] destination rank of each slot (PeerY only)
    int num_peers;
    uint8_t* out;
    uint32_t* err;
};

// Expert output of the single-buffer layout: one array holds every row.
struct LocalY {
    static constexpr bool kPeer = false;
};

// Expert output of every rank (device pointers, peer-mapped where the rank is
// another GPU); scales only for FP8 y.
struct PeerY {
    static constexpr bool kPeer = true;
    const uint8_t* y[kMaxPeers];
    const float* scale[kMaxPeers];
};

constexpr int kChunk = 8;  // slots gathered per pass: kChunk loads in flight per thread

// Receive row of slot k, read by every thread (broadcast, L1 after the first
// warp) so that no warp waits on another; -1 for masked or out-of-range rows.
__device__ __forceinline__ int32_t row_of(const CombineParams& p, int64_t g, int k) {
    const int32_t r = __ldg(p.dst_row + g * p.K + k);
    return (r < p.m_max) ? r : -1;
}

// Start of the row of slot k in y (PeerY): the destination rank's array.
__device__ __forceinline__ const uint8_t* peer_row(const CombineParams& p, const PeerY& py, int64_t g, int k,
                                                   int32_t r, size_t rb) {
    const int d = __ldg(p.dst_rank + g * p.K + k);
    return (d < p.num_peers) ? py.y[d] + (size_t)r * rb : nullptr;
}

template <class Y>
__device__ __forceinline__ void report_rows(const CombineParams& p, int64_t g) {
    if (threadIdx.x < p.K) {
        const int32_t r = __ldg(p.dst_row + g * p.K + threadIdx.x);
        bool bad = r >= p.m_max;
        if constexpr (Y::kPeer) bad = bad || (r >= 0 && __ldg(p.dst_rank + g * p.K + threadIdx.x) >= p.num_peers);
        if (bad) set_error(p.err, EP_DEVERR_ROW_BOUNDS);
    }
}

template <class Y>
__global__ void __launch_bounds__(kBf16Threads) combine_bf16_kernel(CombineParams p, Y py) {
    const int nvec = p.H / 16;  // 32-byte vectors: 16 bf16 channels
    const size_t rb = (size_t)p.H * 2;
    for (int64_t g = blockIdx.x; g < p.N; g += gridDim.x) {  // grid-stride when num_sms caps the grid
        report_rows<Y>(p, g);
        for (int v = threadIdx.x; v < nvec; v += kBf16Threads) {
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
            for (int k0 = 0; k0 < p.K; k0 += kChunk) {
                u32x8 q[kChunk];
                int32_t row[kChunk];
                float w[kChunk];
#pragma unroll
                for (int i = 0; i < kChunk; ++i) {
                    row[i] = (k0 + i < p.K) ? row_of(p, g, k0 + i) : -1;
                    if constexpr (Y::kPeer) {
                        const uint8_t* base = (row[i] >= 0) ? peer_row(p, py, g, k0 + i, row[i], rb) : nullptr;
                        if (base == nullptr) row[i] = -1;
                        w[i] = (row[i] >= 0) ? __ldg(p.topk_w + g * p.K + k0 + i) : 0.0f;
                        if (row[i] >= 0) q[i] = ld256_stream(base + (size_t)v * 32);
                    } else {
                        w[i] = (row[i] >= 0) ? __ldg(p.topk_w + g * p.K + k0 + i) : 0.0f;
                        if (row[i] >= 0) q[i] = ld256_stream(p.y + (size_t)row[i] * rb + (size_t)v * 32);
                    }
                }
#pragma unroll
                for (int i = 0; i < kChunk; ++i) {
                    if (row[i] >= 0) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            acc[2 * j] = __fmaf_rn(w[i], bf16lo(q[i].v[j]), acc[2 * j]);
                            acc[2 * j + 1] = __fmaf_rn(w[i], bf16hi(q[i].v[j]), acc[2 * j + 1]);
                        }
                    }
                }
            }
            u32x8 o;
#pragma unroll
            for (int j = 0; j < 8; ++j) o.v[j] = pack_bf16x2(acc[2 * j], acc[2 * j + 1]);
            st256(p.out + (size_t)g * rb + (size_t)v * 32, o);
        }
    }
}

template <class Y>
__global__ void __launch_bounds__(kFp8Threads) combine_fp8_kernel(CombineParams p, Y py) {
    const int nvec = p.H / 16;  // 16 e4m3 channels (16 B) per vector
    const int nb = p.H / 128;
    const size_t rb = (size_t)p.H;
    for (int64_t g = blockIdx.x; g < p.N; g += gridDim.x) {
        report_rows<Y>(p, g);
        for (int v = threadIdx.x; v < nvec; v += kFp8Threads) {
            // acc[j] holds channels 2j and 2j+1 as an fp32 pair
            uint64_t acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0ull;
            for (int k0 = 0; k0 < p.K; k0 += kChunk) {
                uint4 q[kChunk];
                float sc[kChunk];
                int32_t row[kChunk];
                float w[kChunk];
#pragma unroll
                for (int i = 0; i < kChunk; ++i) {
                    row[i] = (k0 + i < p.K) ? row_of(p, g, k0 + i) : -1;
                    const uint8_t* base = nullptr;
                    const float* sbase = p.y_scale;
                    if constexpr (Y::kPeer) {
                        if (row[i] >= 0) {
                            const int d = __ldg(p.dst_rank + g * p.K + k0 + i);
                            if (d < p.num_peers) {
                                base = py.y[d] + (size_t)row[i] * rb;
                                sbase = py.scale[d];
                            } else {
                                row[i] = -1;
                            }
                        }
                    } else {
                        base = p.y + (size_t)row[i] * rb;
                    }
                    w[i] = (row[i] >= 0) ? __ldg(p.topk_w + g * p.K + k0 + i) : 0.0f;
                    if (row[i] >= 0) {
                        q[i] = __ldcs(reinterpret_cast<const uint4*>(base) + v);
                        sc[i] = __ldg(sbase + (size_t)row[i] * nb + v / 8);
                    }
                }
#pragma unroll
                for (int i = 0; i < kChunk; ++i) {
                    if (row[i] >= 0) {
                        // per channel: acc = fma(w, e4m3 * scale, acc), each step rounded
                        // as in the scalar chain, two channels per instruction
                        const uint64_t w2 = f32x2_pack(w[i], w[i]);
                        const uint64_t s2 = f32x2_pack(sc[i], sc[i]);
                        const uint32_t u[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float2 a = unpack_e4m3x2(u[j] & 0xffffu);
                            const float2 b = unpack_e4m3x2(u[j] >> 16);
                            acc[2 * j] = f32x2_fma_rn(w2, f32x2_mul_rn(f32x2_pack(a.x, a.y), s2), acc[2 * j]);
                            acc[2 * j + 1] =
                                f32x2_fma_rn(w2, f32x2_mul_rn(f32x2_pack(b.x, b.y), s2), acc[2 * j + 1]);
                        }
                    }
                }
            }
            u32x8 o;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 a = f32x2_unpack(acc[j]);
                o.v[j] = pack_bf16x2(a.x, a.y);
            }
            st256(p.out + (size_t)g * p.H * 2 + (size_t)v * 32, o);
        }
    }
}

template <class Y>
cudaError_t launch_y(const ep_buffer& b, const CombineParams& p, const Y& py, bool fp8, cudaStream_t st) {
    auto kern = fp8 ? combine_fp8_kernel<Y> : combine_bf16_kernel<Y>;
    const int threads = fp8 ? kFp8Threads : kBf16Threads;
    int64_t grid = p.N;
    const ep_config_t& c = b.cfg;
    const int sm_cap = (c.num_sms > 0 && c.num_sms < b.sm_count) ? c.num_sms : b.sm_count;
    if (sm_cap < b.sm_count) {
        // num_sms cap (Buffer.set_num_sms): a resident grid on sm_cap SMs' worth of CTAs
        int per_sm = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0);
        if (e != cudaSuccess) return e;
        grid = (int64_t)sm_cap * (per_sm > 0 ? per_sm : 1);
        if (grid > p.N) grid = p.N;
    }
    if (grid > 0x7fffffff) grid = 0x7fffffff;
    kern<<<(unsigned)grid, threads, 0, st>>>(p, py);
    return cudaGetLastError();
}

CombineParams params_of(const ep_buffer& b, int64_t N, const void* y, const float* y_scale, void* out) {
    const ep_config_t& c = b.cfg;
    CombineParams p{};
    p.N = N;
    p.K = c.topk;
    p.H = c.hidden;
    p.m_max = b.m_max;
    p.y = static_cast<const uint8_t*>(y);
    p.y_scale = y_scale;
    p.dst_row = b.dst_row;
    p.topk_w = b.topk_w;
    p.out = static_cast<uint8_t*>(out);
    p.err = b.err;
    return p;
}

}  // namespace

cudaError_t launch_combine(const ep_buffer& b, int T, const void* y, const float* y_scale, void* out,
                           cudaStream_t st) {
    const CombineParams p = params_of(b, (int64_t)b.cfg.num_ranks * T, y, y_scale, out);
    if (p.N == 0) return cudaSuccess;
    return launch_y(b, p, LocalY{}, y_scale != nullptr, st);
}

cudaError_t launch_shard_combine(const ep_buffer& b, int T, const void* const* peer_y,
                                 const float* const* peer_scale, void* out, cudaStream_t st) {
    CombineParams p = params_of(b, T, nullptr, nullptr, out);
    if (p.N == 0) return cudaSuccess;
    p.dst_rank = b.dst_rank;
    p.num_peers = b.cfg.num_ranks;
    PeerY py{};
    for (int d = 0; d < b.cfg.num_ranks; ++d) {
        py.y[d] = static_cast<const uint8_t*>(peer_y[d]);
        py.scale[d] = peer_scale ? peer_scale[d] : nullptr;
    }
    return launch_y(b, p, py, peer_scale != nullptr, st);
}

}  // namespace ep
