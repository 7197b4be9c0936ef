// Combine (sm_100a): gather every token's expert outputs back into token
// order as a top-k weighted sum ("DeepEP：面向MoE的高吞吐低延迟GPU通信库",
// §工程化: dispatch and combine).
//   out[g][h] = bf16_rne( fma(w[g,K-1], y[r_{K-1}][h], ... fma(w[g,0], y[r_0][h], 0)) )
// The chain runs in fp32, slot by slot in ascending k, and skips masked
// slots. FP8 expert outputs are dequantised in the same pass: e4m3 * scale
// in fp32.
//
// One CTA per token; under a num_sms cap, at most num_sms CTAs of several
// token groups each, looping over tokens, or for bf16 y the bulk-copy
// pipeline further down. Each thread owns 16 channels of y at a time: a
// 32-byte vector of bf16 (256-bit load) or a 16-byte vector of e4m3. It
// issues the K gathers of that column before any arithmetic, so K loads are
// in flight per thread. For K <= 8 (the *_k8 kernels) a thread reads the
// token's K row addresses and weights once, not once per vector. Loads use
// the streaming cache hint (y is read once). The 32 output bytes go out in
// one 256-bit store.
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
// Under a num_sms cap of n the grid is at most n CTAs, so that no more than n
// SMs run the kernel (the block scheduler places CTAs breadth-first: 4n small
// CTAs would occupy 4n SMs). Each CTA then holds as many of the token groups
// above as one SM does: kSub groups of the same size, each looping over its
// own tokens.
constexpr int kBf16Sub = 4;   // 512 threads, 128 registers each: the register file
constexpr int kFp8Sub = 12;   // 768 threads at 80 registers

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
constexpr int kMaxKFp8 = 8;  // slots held in registers by the *_k8 kernels

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
__device__ __forceinline__ void report_rows(const CombineParams& p, int64_t g, int tid) {
    if (tid < p.K) {
        const int32_t r = __ldg(p.dst_row + g * p.K + tid);
        bool bad = r >= p.m_max;
        if constexpr (Y::kPeer) bad = bad || (r >= 0 && __ldg(p.dst_rank + g * p.K + tid) >= p.num_peers);
        if (bad) set_error(p.err, EP_DEVERR_ROW_BOUNDS);
    }
}

// SUB groups of kBf16Threads threads per CTA; group j of CTA b takes tokens
// b * SUB + j, then strides by the grid's groups.
template <class Y, int SUB>
__global__ void __launch_bounds__(kBf16Threads * SUB) combine_bf16_kernel(CombineParams p, Y py) {
    const int nvec = p.H / 16;  // 32-byte vectors: 16 bf16 channels
    const size_t rb = (size_t)p.H * 2;
    const int sub = threadIdx.x / kBf16Threads, tid = threadIdx.x - sub * kBf16Threads;
    for (int64_t g = (int64_t)blockIdx.x * SUB + sub; g < p.N; g += (int64_t)gridDim.x * SUB) {
        report_rows<Y>(p, g, tid);
        for (int v = tid; v < nvec; v += kBf16Threads) {
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

// Row addresses (and, with sbase, scale-row addresses) and weights of token
// g's K <= kMaxKFp8 slots, for the *_k8 kernels. Every index, rank and weight
// load is issued at once, none waiting on another; masked and refused slots
// get no address. Returns the mask of slots to read.
template <class Y>
__device__ __forceinline__ uint32_t slot_bases(const CombineParams& p, const Y& py, int64_t g, size_t rb,
                                               const uint8_t* (&base)[kMaxKFp8], float (&w)[kMaxKFp8],
                                               const float** sbase = nullptr, int nb = 0) {
    int32_t r[kMaxKFp8];
    int d[kMaxKFp8];
#pragma unroll
    for (int i = 0; i < kMaxKFp8; ++i) {
        const bool in = i < p.K;
        r[i] = in ? __ldg(p.dst_row + g * p.K + i) : -1;
        w[i] = in ? __ldg(p.topk_w + g * p.K + i) : 0.0f;
        d[i] = 0;
        if constexpr (Y::kPeer) d[i] = in ? (int)__ldg(p.dst_rank + g * p.K + i) : 0;
    }
    uint32_t live = 0;
#pragma unroll
    for (int i = 0; i < kMaxKFp8; ++i) {
        base[i] = nullptr;
        if (sbase) sbase[i] = nullptr;
        if (r[i] < 0 || r[i] >= p.m_max) continue;  // masked, or refused (reported by report_rows)
        if constexpr (Y::kPeer) {
            if (d[i] >= p.num_peers) continue;
            base[i] = py.y[d[i]] + (size_t)r[i] * rb;
            if (sbase) sbase[i] = py.scale[d[i]] + (size_t)r[i] * nb;
        } else {
            base[i] = p.y + (size_t)r[i] * rb;
            if (sbase) sbase[i] = p.y_scale + (size_t)r[i] * nb;
        }
        live |= 1u << i;
    }
    return live;
}

// combine_bf16_kernel for K <= kMaxKFp8: the token's K row addresses and
// weights are read once per token into registers (masked and refused slots
// are skipped), then each thread walks its 32-byte vectors. One token per
// CTA is held to 5 CTAs per SM (at most 102 registers; 94 used, no spills):
// measured on B200 at 126 registers and 4 CTAs per SM, prefill combine ran
// 617.0 against 609.0 us.
template <class Y, int SUB>
__global__ void __launch_bounds__(kBf16Threads * SUB, SUB == 1 ? 5 : 1) combine_bf16_k8_kernel(CombineParams p, Y py) {
    const int nvec = p.H / 16;  // 32-byte vectors: 16 bf16 channels
    const size_t rb = (size_t)p.H * 2;
    const int sub = threadIdx.x / kBf16Threads, tid = threadIdx.x - sub * kBf16Threads;
    for (int64_t g = (int64_t)blockIdx.x * SUB + sub; g < p.N; g += (int64_t)gridDim.x * SUB) {
        report_rows<Y>(p, g, tid);
        const uint8_t* base[kMaxKFp8];
        float w[kMaxKFp8];
        const uint32_t live = slot_bases<Y>(p, py, g, rb, base, w);  // bit i: slot i is read
        for (int v = tid; v < nvec; v += kBf16Threads) {
            u32x8 q[kMaxKFp8];
#pragma unroll
            for (int i = 0; i < kMaxKFp8; ++i)
                if ((live >> i) & 1u) q[i] = ld256_stream(base[i] + (size_t)v * 32);
            uint64_t acc[8];  // channel pairs (2j, 2j+1) as fp32 pairs
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0ull;
#pragma unroll
            for (int i = 0; i < kMaxKFp8; ++i) {
                if ((live >> i) & 1u) {
                    const uint64_t w2 = f32x2_pack(w[i], w[i]);
#pragma unroll
                    for (int j = 0; j < 8; ++j)  // per channel: acc = fma(w, y, acc), rounded as the scalar chain
                        acc[j] = f32x2_fma_rn(w2, f32x2_pack(bf16lo(q[i].v[j]), bf16hi(q[i].v[j])), acc[j]);
                }
            }
            u32x8 o;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 a = f32x2_unpack(acc[j]);
                o.v[j] = pack_bf16x2(a.x, a.y);
            }
            st256(p.out + (size_t)g * rb + (size_t)v * 32, o);
        }
    }
}

// SUB groups of kFp8Threads threads per CTA, as in combine_bf16_kernel.
template <class Y, int SUB>
__global__ void __launch_bounds__(kFp8Threads * SUB) combine_fp8_kernel(CombineParams p, Y py) {
    const int nvec = p.H / 16;  // 16 e4m3 channels (16 B) per vector
    const int nb = p.H / 128;
    const size_t rb = (size_t)p.H;
    const int sub = threadIdx.x / kFp8Threads, tid = threadIdx.x - sub * kFp8Threads;
    for (int64_t g = (int64_t)blockIdx.x * SUB + sub; g < p.N; g += (int64_t)gridDim.x * SUB) {
        report_rows<Y>(p, g, tid);
        for (int v = tid; v < nvec; v += kFp8Threads) {
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

// The same for K <= kMaxKFp8: the token's K row and scale-row addresses and
// weights are read once per token into registers (masked and refused slots
// are skipped), then each thread walks its 16-channel vectors.
template <class Y, int SUB>
__global__ void __launch_bounds__(kFp8Threads * SUB) combine_fp8_k8_kernel(CombineParams p, Y py) {
    const int nvec = p.H / 16;  // 16 e4m3 channels (16 B) per vector
    const int nb = p.H / 128;
    const size_t rb = (size_t)p.H;
    const int sub = threadIdx.x / kFp8Threads, tid = threadIdx.x - sub * kFp8Threads;
    for (int64_t g = (int64_t)blockIdx.x * SUB + sub; g < p.N; g += (int64_t)gridDim.x * SUB) {
        report_rows<Y>(p, g, tid);
        const uint8_t* base[kMaxKFp8];
        const float* sbase[kMaxKFp8];
        float w[kMaxKFp8];
        const uint32_t live = slot_bases<Y>(p, py, g, rb, base, w, sbase, nb);  // bit i: slot i is read
        for (int v = tid; v < nvec; v += kFp8Threads) {
            // acc[j] holds channels 2j and 2j+1 as an fp32 pair
            uint64_t acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0ull;
            uint4 q[kMaxKFp8];
            float sc[kMaxKFp8];
#pragma unroll
            for (int i = 0; i < kMaxKFp8; ++i) {
                if ((live >> i) & 1u) {
                    q[i] = __ldcs(reinterpret_cast<const uint4*>(base[i]) + v);
                    sc[i] = __ldg(sbase[i] + v / 8);
                }
            }
#pragma unroll
            for (int i = 0; i < kMaxKFp8; ++i) {
                if ((live >> i) & 1u) {
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
                        acc[2 * j + 1] = f32x2_fma_rn(w2, f32x2_mul_rn(f32x2_pack(b.x, b.y), s2), acc[2 * j + 1]);
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

// ---- bf16 combine under a num_sms cap: a TMA bulk-copy pipeline ------------
//
// Under a num_sms cap the grid is one CTA per SM. The register gather above
// then keeps at most 128 KB per SM in flight (512 threads, 8 loads of 32 B
// each). Here the bulk-copy (TMA) engine moves the rows into shared memory
// instead: 4 stages, each K row segments of kTmaChunk channels (56 KB at
// K = 8), so the threads issue only the arithmetic. Used where H is a
// multiple of kTmaChunk. Measured on B200 at the prefill shape (8 x 4096
// tokens, H = 7168, K = 8): 2.2 ms at 20 SMs and 0.66 ms at 74 SMs, against
// 2.4 and 0.79 ms for the register gather (combine_bf16_k8_kernel). Every
// byte crosses shared memory twice (the copy, then the consumers' reads),
// which bounds this design at about half the shared-memory bandwidth.
// Slower, as measured:
//  - more and smaller stages (2-4 KB copies, 6-12 stages);
//  - whole-row copies (14 KB, 4 slots per stage);
//  - 448 consumers of 8 channels with a sleep hint in the waits.
//
// One CTA per SM: kTmaConsumers consumer threads and one producer warp. A
// unit is one token and one block of kTmaChunk channels; CTA b takes a
// contiguous range of tokens, all blocks of each. The producer warp reads the
// (row, weight) pairs of kTmaBatch tokens at once, lane 8j + k holding slot k
// of token j (one coalesced load of each table), a batch ahead of the copies
// so that their latency overlaps the copies of the batch before. For a unit it
// writes the token, the slot mask and the weights next to the stage, arms the
// stage's "full" barrier with the bytes to come, and each lane of the token's
// group with an unmasked slot issues that row's bulk copy. A consumer thread
// t owns channels 8t.. and kTmaChunk/2 + 8t.. of the block (16-byte reads,
// contiguous across a warp: no bank conflicts). It moves them to registers
// for all K rows, and every consumer warp then arrives on the stage's "empty"
// barrier, which frees the stage for the producer. The sum is the register
// kernel's: an fp32 fma chain over k ascending, one bf16 rounding.
//
// Every wait is bounded (kWaitLimitNs): a wait that gives up sets
// EP_DEVERR_TIMEOUT, and before the CTA returns the producer waits, bounded
// again, for the copies it issued, so none lands in shared memory after the
// CTA has left. A consumer arrives on "empty" only after its "full" wait
// succeeded, so a stage is refilled only once its previous copies landed:
// only the last kTmaStages units issued can still be in flight.
constexpr int kTmaConsumers = 224;
constexpr int kTmaThreads = kTmaConsumers + 32;
constexpr int kTmaStages = 4;
constexpr int kTmaMaxK = 8;
constexpr int kTmaBatch = 32 / kTmaMaxK;  // tokens whose slots the producer warp reads at once
constexpr int kTmaVec = 16;               // channels per consumer
constexpr int kTmaChunk = kTmaConsumers * kTmaVec;  // channels per unit
constexpr size_t kTmaStageBytes = (size_t)kTmaMaxK * kTmaChunk * 2;
// What the producer tells the consumers about the unit in a stage.
struct TmaUnit {
    int64_t g;          // token
    int cb;             // channel block
    uint32_t mask;      // bit k: slot k's row is in the stage
    float w[kTmaMaxK];  // the slots' weights
};
constexpr size_t kTmaSmem =
    kTmaStages * kTmaStageBytes + 2 * kTmaStages * sizeof(uint64_t) + kTmaStages * sizeof(TmaUnit);

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_arrive(uint64_t* bar, uint32_t tx) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(tx) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok)
                 : "r"(smem_addr(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}
// Waits for the phase of `bar` with this parity to complete; false if it
// has not after limit_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > limit_ns) return false;
    return true;
}

// Self-test of the bounded mbarrier wait: a barrier that expects one arrival
// nobody makes. The wait must give up after limit_ns; thread 0 then records
// that in gave_up and sets EP_DEVERR_TIMEOUT. No copy is in flight.
__global__ void mbarrier_timeout_selftest_kernel(uint32_t* err, uint32_t* gave_up, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit_ns)) {
        *gave_up = 1u;
        set_error(err, EP_DEVERR_TIMEOUT);
    }
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// One lane's slot (token g, slot k), as the producer warp reads it: every
// load is issued without waiting on another, so a batch's loads overlap.
struct TmaSlot {
    const uint8_t* src;  // start of the row in y, nullptr when masked or refused
    float w;
    bool bad;  // a row the buffer cannot hold, or a rank the table lacks
};

template <class Y>
__device__ __forceinline__ TmaSlot tma_slot(const CombineParams& p, const Y& py, int64_t g, int k, size_t rb) {
    const int64_t at = g * p.K + k;
    const int32_t r = __ldg(p.dst_row + at);
    TmaSlot sl;
    sl.w = __ldg(p.topk_w + at);
    sl.bad = r >= p.m_max;
    const bool use = r >= 0 && !sl.bad;
    if constexpr (Y::kPeer) {
        const int d = __ldg(p.dst_rank + at);
        const bool known = d >= 0 && d < p.num_peers;
        sl.bad = sl.bad || (r >= 0 && !known);
        sl.src = (use && known) ? py.y[d] + (size_t)r * rb : nullptr;
    } else {
        sl.src = use ? p.y + (size_t)r * rb : nullptr;
    }
    return sl;
}

template <class Y>
__global__ void __launch_bounds__(kTmaThreads, 1) combine_bf16_tma_kernel(CombineParams p, Y py) {
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kTmaStages * kTmaStageBytes);
    uint64_t* empty = full + kTmaStages;
    TmaUnit* meta = reinterpret_cast<TmaUnit*>(empty + kTmaStages);
    const int t = threadIdx.x, lane = t & 31;
    const int nblk = (p.H + kTmaChunk - 1) / kTmaChunk;
    const size_t rb = (size_t)p.H * 2;
    // this CTA's tokens [g0, g1)
    const int64_t g0 = (int64_t)blockIdx.x * p.N / gridDim.x, g1 = (int64_t)(blockIdx.x + 1) * p.N / gridDim.x;
    const int64_t mine = (g1 - g0) * nblk;
    if (t == 0) {
        for (int s = 0; s < kTmaStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kTmaConsumers / 32);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (t >= kTmaConsumers) {  // the producer warp
        const int j = lane / kTmaMaxK, k = lane % kTmaMaxK;  // token j of a batch, slot k
        const bool slot = k < p.K;
        int64_t issued = 0;
        bool ok = true;
        // the batch at gb, and the next one, read while this one's copies go out
        TmaSlot cur{nullptr, 0.0f, false};
        if (slot && g0 + j < g1) cur = tma_slot<Y>(p, py, g0 + j, k, rb);
        for (int64_t gb = g0; gb < g1 && ok; gb += kTmaBatch) {
            TmaSlot next{nullptr, 0.0f, false};
            if (slot && gb + kTmaBatch + j < g1) next = tma_slot<Y>(p, py, gb + kTmaBatch + j, k, rb);
            if (cur.bad) set_error(p.err, EP_DEVERR_ROW_BOUNDS);
            const uint32_t have = __ballot_sync(0xffffffffu, cur.src != nullptr);
            for (int jj = 0; jj < kTmaBatch && gb + jj < g1 && ok; ++jj) {
                const uint32_t mask = (have >> (jj * kTmaMaxK)) & ((1u << kTmaMaxK) - 1);
                for (int cb = 0; cb < nblk; ++cb) {
                    const int64_t i = issued;
                    const int s = (int)(i % kTmaStages);
                    if (i >= kTmaStages && lane == 0) ok = mbar_wait(&empty[s], (uint32_t)((i / kTmaStages - 1) & 1));
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) {
                        if (lane == 0) set_error(p.err, EP_DEVERR_TIMEOUT);
                        break;
                    }
                    const uint32_t bytes = (uint32_t)min(kTmaChunk, p.H - cb * kTmaChunk) * 2;
                    TmaUnit& m = meta[s];
                    if (j == jj) m.w[k] = cur.w;
                    __syncwarp();
                    if (lane == 0) {
                        m.g = gb + jj;
                        m.cb = cb;
                        m.mask = mask;
                        // releases the metadata with the arrival
                        mbar_expect_arrive(&full[s], (uint32_t)__popc(mask) * bytes);
                    }
                    __syncwarp();
                    if (j == jj && cur.src != nullptr)
                        bulk_load(sm + (size_t)s * kTmaStageBytes + (size_t)k * kTmaChunk * 2,
                                  cur.src + (size_t)cb * kTmaChunk * 2, bytes, &full[s]);
                    issued = i + 1;
                }
            }
            cur = next;
        }
        // copies issued and possibly not landed: only the last kTmaStages units
        if (lane == 0)
            for (int64_t i = (issued > kTmaStages ? issued - kTmaStages : 0); i < issued; ++i)
                if (!mbar_wait(&full[i % kTmaStages], (uint32_t)((i / kTmaStages) & 1))) break;
        return;
    }

    for (int64_t i = 0; i < mine; ++i) {
        const int s = (int)(i % kTmaStages);
        if (!mbar_wait(&full[s], (uint32_t)((i / kTmaStages) & 1))) {
            set_error(p.err, EP_DEVERR_TIMEOUT);
            break;
        }
        const TmaUnit& m = meta[s];
        const int64_t g = m.g;
        const uint32_t mask = m.mask;
        // This thread's channels of the block: 8 at c0 and 8 at c1, so that a
        // warp's 16-byte shared-memory reads are contiguous (no bank conflict).
        const int wb = min(kTmaChunk, p.H - m.cb * kTmaChunk);  // channels in the block
        const int c0 = 8 * t, c1 = kTmaChunk / 2 + 8 * t;
        const bool h0 = c0 < wb, h1 = c1 < wb;
        // the stage's rows into registers, then the stage goes back to the producer
        const uint8_t* stage = sm + (size_t)s * kTmaStageBytes;
        uint32_t q[kTmaMaxK][8];
        float w[kTmaMaxK];
#pragma unroll
        for (int k = 0; k < kTmaMaxK; ++k) {
            w[k] = m.w[k];
            if ((mask >> k) & 1u) {
                const uint8_t* row = stage + (size_t)k * kTmaChunk * 2;
                if (h0) {
                    const uint4 a = *reinterpret_cast<const uint4*>(row + c0 * 2);
                    q[k][0] = a.x, q[k][1] = a.y, q[k][2] = a.z, q[k][3] = a.w;
                }
                if (h1) {
                    const uint4 a = *reinterpret_cast<const uint4*>(row + c1 * 2);
                    q[k][4] = a.x, q[k][5] = a.y, q[k][6] = a.z, q[k][7] = a.w;
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (h0) {  // h1 implies h0
            uint64_t acc[8];  // channel pairs as fp32 pairs: 0-3 at c0, 4-7 at c1
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0ull;
#pragma unroll
            for (int k = 0; k < kTmaMaxK; ++k) {
                if (!((mask >> k) & 1u)) continue;
                const uint64_t w2 = f32x2_pack(w[k], w[k]);
#pragma unroll
                for (int j = 0; j < 8; ++j)  // per channel: acc = fma(w, y, acc), rounded as the scalar chain
                    if (j < 4 || h1) acc[j] = f32x2_fma_rn(w2, f32x2_pack(bf16lo(q[k][j]), bf16hi(q[k][j])), acc[j]);
            }
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 a = f32x2_unpack(acc[j]);
                o[j] = pack_bf16x2(a.x, a.y);
            }
            uint8_t* dst = p.out + (size_t)g * rb + (size_t)m.cb * kTmaChunk * 2;
            *reinterpret_cast<uint4*>(dst + c0 * 2) = make_uint4(o[0], o[1], o[2], o[3]);
            if (h1) *reinterpret_cast<uint4*>(dst + c1 * 2) = make_uint4(o[4], o[5], o[6], o[7]);
        }
    }
}

template <class Y>
cudaError_t launch_tma(const CombineParams& p, const Y& py, int sm_cap, cudaStream_t st) {
    // per launch: the attribute belongs to the current device
    cudaError_t e = cudaFuncSetAttribute(combine_bf16_tma_kernel<Y>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kTmaSmem);
    if (e != cudaSuccess) return e;
    const int64_t grid = p.N < sm_cap ? p.N : sm_cap;  // one CTA per SM
    combine_bf16_tma_kernel<Y><<<(unsigned)grid, kTmaThreads, kTmaSmem, st>>>(p, py);
    return cudaGetLastError();
}

template <class Y>
cudaError_t launch_y(const ep_buffer& b, const CombineParams& p, const Y& py, bool fp8, cudaStream_t st) {
    const ep_config_t& c = b.cfg;
    const int sm_cap = (c.num_sms > 0 && c.num_sms < b.sm_count) ? c.num_sms : b.sm_count;
    const bool k8 = p.K <= kMaxKFp8;
    if (sm_cap == b.sm_count) {  // one CTA per token (a grid-stride loop past 2^31 - 1 tokens)
        const unsigned grid = (unsigned)(p.N < 0x7fffffff ? p.N : 0x7fffffff);
        if (fp8 && k8) combine_fp8_k8_kernel<Y, 1><<<grid, kFp8Threads, 0, st>>>(p, py);
        else if (fp8) combine_fp8_kernel<Y, 1><<<grid, kFp8Threads, 0, st>>>(p, py);
        // bf16 y: small batches keep the general kernel (measured on B200,
        // N * H < 2^24: decode 31.6 against 32.0 us, tiny 6.4 against 7.0 us)
        else if (k8 && p.N * p.H >= (int64_t)1 << 24) combine_bf16_k8_kernel<Y, 1><<<grid, kBf16Threads, 0, st>>>(p, py);
        else combine_bf16_kernel<Y, 1><<<grid, kBf16Threads, 0, st>>>(p, py);
        return cudaGetLastError();
    }
    // num_sms cap (Buffer.set_num_sms): at most sm_cap CTAs, each filling an
    // SM. bf16 y: the bulk-copy pipeline where the rows split into whole
    // units (measured on B200, 20 SMs: prefill H = 7168 2.2 ms against 2.4
    // for the register gather below; skewed H = 4096, whose 512-channel tail
    // unit would hold a whole stage, 1.66 against 1.24 ms).
    if (!fp8 && p.K <= kTmaMaxK && p.H % kTmaChunk == 0) return launch_tma(p, py, sm_cap, st);
    const int sub = fp8 ? kFp8Sub : kBf16Sub;
    int64_t grid = (p.N + sub - 1) / sub;
    if (grid > sm_cap) grid = sm_cap;
    if (fp8) combine_fp8_kernel<Y, kFp8Sub><<<(unsigned)grid, kFp8Threads * kFp8Sub, 0, st>>>(p, py);
    else if (k8) combine_bf16_k8_kernel<Y, kBf16Sub><<<(unsigned)grid, kBf16Threads * kBf16Sub, 0, st>>>(p, py);
    else combine_bf16_kernel<Y, kBf16Sub><<<(unsigned)grid, kBf16Threads * kBf16Sub, 0, st>>>(p, py);
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

cudaError_t launch_mbarrier_timeout_selftest(uint32_t* err, uint32_t* gave_up, unsigned long long limit_ns,
                                             cudaStream_t st) {
    mbarrier_timeout_selftest_kernel<<<1, 32, 0, st>>>(err, gave_up, limit_ns);
    return cudaGetLastError();
}

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
