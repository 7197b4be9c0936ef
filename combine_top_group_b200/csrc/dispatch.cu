// Dispatch (sm_100a): scatter each token's hidden vector to the receive row
// of every unmasked slot. Only target experts get a copy
// ("DeepEP：年度总结中的计算通信重叠摘记", §节点内通信: is_token_in_rank, no
// full all-to-all). The optional FP8 cast sends 1 byte per element instead of
// 2 (same section) and adds one fp32 scale per 128 channels.
//
// Both kernels are persistent and move rows with the bulk-copy (TMA) engine:
//  - cp.async.bulk loads a token row HBM -> shared memory (mbarrier
//    completion);
//  - cp.async.bulk stores write it shared -> each receive row (bulk groups);
//  - loads run LA tokens ahead through S stage buffers.
// bf16: one warp per CTA, which only issues copies; the data never passes
//   through registers.
// FP8: 256 threads read the staged row, reduce amax over each 128-channel
//   block (16 lanes x 8 channels), cast with cvt.rn.satfinite.e4m3x2 into a
//   double-buffered output stage, and the bulk engine writes it K times.
// Every wait is bounded (EP_DEVERR_TIMEOUT). Every row index is checked
// against the buffer (EP_DEVERR_ROW_BOUNDS).
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

// ---------------------------------------------------------------------------
// bf16: pure bulk copies
// ---------------------------------------------------------------------------
template <int S, int LA>
__global__ void __launch_bounds__(32) dispatch_bf16_kernel(DispatchParams p) {
    static_assert(LA >= 1 && LA < S, "lookahead must leave a stage for the stores");
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t rb = (uint32_t)p.H * 2u;  // row bytes, multiple of 16
    uint8_t* stage = smem;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + (size_t)S * rb);
    int32_t* ring_row = reinterpret_cast<int32_t*>(bar + S);
    float* ring_w = reinterpret_cast<float*>(ring_row + S * p.K);

    const int lane = threadIdx.x;
    const int64_t n_my = (p.N > blockIdx.x) ? (p.N - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&bar[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const uint64_t pol = l2_evict_first_policy();

    auto issue = [&](int64_t i) {
        const int s = (int)(i % S);
        const int64_t g = blockIdx.x + i * gridDim.x;
        if (lane < p.K) {
            ring_row[s * p.K + lane] = p.dst_row[g * p.K + lane];
            ring_w[s * p.K + lane] = p.topk_w[g * p.K + lane];
        }
        if (lane == 0) {
            mbar_arrive_expect_tx(&bar[s], rb);
            bulk_g2s(stage + (size_t)s * rb, p.x + (size_t)g * rb, rb, &bar[s], pol);
        }
    };

    const int64_t pro = n_my < LA ? n_my : LA;
    for (int64_t i = 0; i < pro; ++i) issue(i);

    int64_t fail_i = -1;
    for (int64_t i = 0; i < n_my; ++i) {
        const int s = (int)(i % S);
        const uint32_t parity = (uint32_t)((i / S) & 1);
        const int64_t g = blockIdx.x + i * gridDim.x;
        __syncwarp();
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&bar[s], parity);
        ok = __shfl_sync(FULL, ok, 0);
        if (!ok) {
            fail_i = i;
            break;
        }
        int32_t row = (lane < p.K) ? ring_row[s * p.K + lane] : -1;
        const float w = (lane < p.K) ? ring_w[s * p.K + lane] : 0.0f;
        if (row >= p.m_max) {
            set_error(p.err, EP_DEVERR_ROW_BOUNDS);
            row = -1;
        }
        const uint32_t vm = __ballot_sync(FULL, row >= 0);
        for (int k = 0; k < p.K; ++k) {
            const int32_t r = __shfl_sync(FULL, row, k);
            if (lane == 0 && ((vm >> k) & 1u))
                bulk_s2g(p.recv_x + (size_t)r * rb, stage + (size_t)s * rb, rb, pol);
        }
        if (lane == 0) bulk_commit();
        if (row >= 0) {
            p.recv_src[row] = (int32_t)g;
            p.recv_w[row] = w;
        }
        if (i + LA < n_my) {
            // the stage of token i+LA was last read by the stores of token
            // i+LA-S: at most S-LA younger groups may still be reading
            if (lane == 0) bulk_wait_read<S - LA>();
            __syncwarp();
            issue(i + LA);
        }
    }
    if (fail_i >= 0 && lane == 0) {
        set_error(p.err, EP_DEVERR_TIMEOUT);
        // loads for tokens fail_i+1 .. fail_i+LA-1 may still be in flight:
        // wait (bounded) for each before the CTA's shared memory goes away
        for (int64_t j = fail_i + 1; j < fail_i + LA && j < n_my; ++j)
            (void)mbar_wait_bounded(&bar[j % S], (uint32_t)((j / S) & 1));
    }
    if (lane == 0) bulk_wait_all<0>();
}

// ---------------------------------------------------------------------------
// FP8: fused amax -> e4m3 cast with per-128-channel fp32 scales
// ---------------------------------------------------------------------------
constexpr int kFp8Threads = 256;

template <int S, int LA>
__global__ void __launch_bounds__(kFp8Threads) dispatch_fp8_kernel(DispatchParams p) {
    static_assert(LA >= 1 && LA < S, "lookahead must leave a stage free");
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t rb_in = (uint32_t)p.H * 2u;
    const uint32_t rb_out = (uint32_t)p.H;  // e4m3 payload
    const int nb = p.H / 128;
    uint8_t* in_stage = smem;
    uint8_t* out_stage = smem + (size_t)S * rb_in;  // [2][H]
    uint64_t* bar = reinterpret_cast<uint64_t*>(out_stage + 2 * (size_t)rb_out);
    int32_t* ring_row = reinterpret_cast<int32_t*>(bar + S);
    float* ring_w = reinterpret_cast<float*>(ring_row + S * p.K);
    volatile int& s_ok = *reinterpret_cast<int*>(ring_w + S * p.K);  // in the dynamic region (alignment)

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int64_t n_my = (p.N > blockIdx.x) ? (p.N - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&bar[s], 1);
        fence_mbar_init();
        s_ok = 1;
    }
    __syncthreads();
    const uint64_t pol = l2_evict_first_policy();
    int64_t fail_i = -1;  // meaningful on thread 0 only

    auto issue = [&](int64_t i) {  // called by warp 0 only
        const int s = (int)(i % S);
        const int64_t g = blockIdx.x + i * gridDim.x;
        if (lane < p.K) {
            ring_row[s * p.K + lane] = p.dst_row[g * p.K + lane];
            ring_w[s * p.K + lane] = p.topk_w[g * p.K + lane];
        }
        if (lane == 0) {
            mbar_arrive_expect_tx(&bar[s], rb_in);
            bulk_g2s(in_stage + (size_t)s * rb_in, p.x + (size_t)g * rb_in, rb_in, &bar[s], pol);
        }
    };
    if (tid < 32) {
        const int64_t pro = n_my < LA ? n_my : LA;
        for (int64_t i = 0; i < pro; ++i) issue(i);
    }

    const int nvec = p.H / 8;  // 16-byte vectors of 8 bf16 per row
    for (int64_t i = 0; i < n_my; ++i) {
        const int s = (int)(i % S);
        const int o = (int)(i & 1);
        const uint32_t parity = (uint32_t)((i / S) & 1);
        const int64_t g = blockIdx.x + i * gridDim.x;
        if (tid < 32) {
            // stage (i+LA)%S was consumed in iteration i+LA-S < i
            if (i + LA < n_my) issue(i + LA);
            if (lane == 0) {
                if (!mbar_wait_bounded(&bar[s], parity)) {
                    s_ok = 0;
                    fail_i = i;
                }
                bulk_wait_read<1>();  // output stage o (token i-2) is free again
            }
        }
        __syncthreads();
        if (!s_ok) break;
        (void)mbar_try_wait(&bar[s], parity);  // completed phase: each thread acquires the staged row

        const uint8_t* src = in_stage + (size_t)s * rb_in;
        uint8_t* dst = out_stage + (size_t)o * rb_out;
        for (int v0 = 0; v0 < nvec; v0 += kFp8Threads) {
            const int v = v0 + tid;
            const bool act = v < nvec;  // uniform across each 16-lane block
            uint4 q = act ? *reinterpret_cast<const uint4*>(src + (size_t)v * 16) : make_uint4(0, 0, 0, 0);
            float f[8] = {bf16lo(q.x), bf16hi(q.x), bf16lo(q.y), bf16hi(q.y),
                          bf16lo(q.z), bf16hi(q.z), bf16lo(q.w), bf16hi(q.w)};
            float a = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(f[j]));
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, off));
            const float amax = fmaxf(a, 1e-4f);
            const float inv = __fdiv_rn(448.0f, amax);
            if (act) {
                uint2 out;
                out.x = pack_e4m3x2(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv)) |
                        (pack_e4m3x2(__fmul_rn(f[2], inv), __fmul_rn(f[3], inv)) << 16);
                out.y = pack_e4m3x2(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv)) |
                        (pack_e4m3x2(__fmul_rn(f[6], inv), __fmul_rn(f[7], inv)) << 16);
                *reinterpret_cast<uint2*>(dst + (size_t)v * 8) = out;
                if ((lane & 15) == 0) {
                    const float scale = __fdiv_rn(amax, 448.0f);
                    const int b = v / 16;
                    for (int k = 0; k < p.K; ++k) {
                        int32_t r = ring_row[s * p.K + k];
                        if (r >= 0 && r < p.m_max) p.recv_scale[(size_t)r * nb + b] = scale;
                    }
                }
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid < 32) {
            int32_t row = (lane < p.K) ? ring_row[s * p.K + lane] : -1;
            const float w = (lane < p.K) ? ring_w[s * p.K + lane] : 0.0f;
            if (row >= p.m_max) {
                set_error(p.err, EP_DEVERR_ROW_BOUNDS);
                row = -1;
            }
            const uint32_t vm = __ballot_sync(FULL, row >= 0);
            for (int k = 0; k < p.K; ++k) {
                const int32_t r = __shfl_sync(FULL, row, k);
                if (lane == 0 && ((vm >> k) & 1u))
                    bulk_s2g(p.recv_x + (size_t)r * rb_out, dst, rb_out, pol);
            }
            if (lane == 0) bulk_commit();
            if (row >= 0) {
                p.recv_src[row] = (int32_t)g;
                p.recv_w[row] = w;
            }
        }
    }
    if (tid == 0) {
        if (!s_ok) {
            set_error(p.err, EP_DEVERR_TIMEOUT);
            // loads for tokens fail_i+1 .. fail_i+LA may still be in flight
            for (int64_t j = fail_i + 1; j <= fail_i + LA && j < n_my; ++j)
                (void)mbar_wait_bounded(&bar[j % S], (uint32_t)((j / S) & 1));
        }
        bulk_wait_all<0>();
    }
}

template <typename KernelT>
cudaError_t launch_persistent(KernelT kernel, int threads, size_t smem, int sm_cap, int64_t N,
                              const DispatchParams& p, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t grid = (int64_t)sm_cap * per_sm;
    if (grid > N) grid = N;
    if (grid < 1) return cudaSuccess;
    kernel<<<(unsigned)grid, threads, smem, st>>>(p);
    return cudaGetLastError();
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
    int sm_cap = (c.num_sms > 0 && c.num_sms < b.sm_count) ? c.num_sms : b.sm_count;
    const size_t ring = (size_t)2 * 8 * kMaxK * 4 + 16;  // ring rows + weights (S <= 8) + flag
    if (!(c.flags & EP_FLAG_FP8)) {
        const size_t rb = (size_t)p.H * 2;
        // aim for ~200 KB of stages per SM: 6 stages for rows up to ~16 KB
        if (rb * 6 + ring + 64 <= 100 * 1024) {
            constexpr int S = 6, LA = 3;
            size_t smem = (size_t)S * rb + S * 8 + ring;
            return launch_persistent(dispatch_bf16_kernel<S, LA>, 32, smem, sm_cap, p.N, p, st);
        }
        constexpr int S = 3, LA = 1;
        size_t smem = (size_t)S * rb + S * 8 + ring;
        return launch_persistent(dispatch_bf16_kernel<S, LA>, 32, smem, sm_cap, p.N, p, st);
    }
    const size_t rb_in = (size_t)p.H * 2, rb_out = (size_t)p.H;
    if (rb_in * 4 + 2 * rb_out + ring + 64 <= 110 * 1024) {
        constexpr int S = 4, LA = 2;
        size_t smem = (size_t)S * rb_in + 2 * rb_out + S * 8 + ring;
        return launch_persistent(dispatch_fp8_kernel<S, LA>, kFp8Threads, smem, sm_cap, p.N, p, st);
    }
    constexpr int S = 2, LA = 1;
    size_t smem = (size_t)S * rb_in + 2 * rb_out + S * 8 + ring;
    return launch_persistent(dispatch_fp8_kernel<S, LA>, kFp8Threads, smem, sm_cap, p.N, p, st);
}

}  // namespace ep
