// Device helpers shared by the sm_100a kernels of libep: 256-bit global
// loads and stores, number-format conversions, the block scan, and the clock
// behind the bounded wait of every spin in this library.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"

namespace ep {

constexpr unsigned FULL = 0xffffffffu;

// A wait that has not finished after this long gives up and sets
// EP_DEVERR_TIMEOUT. The only waits are the layout's grid barriers, whose
// CTAs are all resident and finish their phase within microseconds, so
// reaching it means a bug.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- 256-bit global loads and stores (sm_100) ------------------------------

struct __align__(32) u32x8 {
    uint32_t v[8];
};

// Streaming 256-bit load: the data is read once.
__device__ __forceinline__ u32x8 ld256_stream(const void* p) {
    u32x8 a;
    asm volatile("ld.global.cs.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(a.v[0]), "=r"(a.v[1]), "=r"(a.v[2]), "=r"(a.v[3]), "=r"(a.v[4]), "=r"(a.v[5]),
                   "=r"(a.v[6]), "=r"(a.v[7])
                 : "l"(p));
    return a;
}

__device__ __forceinline__ void st256(void* p, const u32x8& a) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a.v[0]), "r"(a.v[1]),
                 "r"(a.v[2]), "r"(a.v[3]), "r"(a.v[4]), "r"(a.v[5]), "r"(a.v[6]), "r"(a.v[7])
                 : "memory");
}

// ---- number formats -------------------------------------------------------

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Two fp32 -> two bf16 (round to nearest even); `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two fp32 -> two e4m3 (round to nearest even, saturate to +-448); `lo`
// lands in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two e4m3 (low byte first) -> two fp32, exactly (via f16x2, which holds
// every e4m3 value).
__device__ __forceinline__ float2 unpack_e4m3x2(uint32_t two_bytes) {
    uint32_t h2;
    uint16_t in = static_cast<uint16_t>(two_bytes);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    __half2_raw raw;
    raw.x = static_cast<unsigned short>(h2 & 0xffffu);
    raw.y = static_cast<unsigned short>(h2 >> 16);
    return __half22float2(__half2(raw));
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic) ---------------------------
// A pair of fp32 values in one 64-bit register: `lo` in the low half. The
// paired multiply and fused multiply-add round each lane on its own (RN), so
// a pair op gives the same bits as two scalar __fmul_rn / __fmaf_rn.

__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f32x2_unpack(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t f32x2_mul_rn(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// a * b + c per lane, one rounding.
__device__ __forceinline__ uint64_t f32x2_fma_rn(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// Order-preserving map from a (non-NaN) float to uint32: a < b <=> key(a) <
// key(b). -0 is folded into +0 first, so equal values get equal keys.
// Key 0 is never produced, so 0 can mean "no candidate".
__device__ __forceinline__ uint32_t order_key(float v) {
    uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// SplitMix64 (Steele, Lea and Flood, OOPSLA 2014): first output of the
// generator whose state starts at `counter`.
__device__ __forceinline__ uint64_t splitmix64(uint64_t counter) {
    uint64_t z = counter + 0x9e3779b97f4a7c15ull;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bit) { atomicOr(err, bit); }

// Exclusive scan of n <= 4 * blockDim.x values in[j * stride] into out[0..n],
// with out[n] = total. Called by every thread of the block.
__device__ inline void block_exclusive_scan(const int32_t* in, int stride, int n, int* out, int* warp_tot) {
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
        const int o = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int wv = (lane < nw) ? warp_tot[lane] : 0;
        int wi = wv;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(FULL, wi, off);
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

}  // namespace ep
