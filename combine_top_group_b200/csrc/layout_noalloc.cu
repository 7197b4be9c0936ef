// ep_get_layout_noalloc: routing + layout for callers that cannot allocate
// device memory. Think of code inside a host framework whose memory planner
// owns every device byte, or a runtime with a fixed memory budget that may
// not call cudaMalloc (or any allocator) after start-up. Such a caller has
// its input and output tensors but no way to get a workspace.
//
// The only scratch the layout kernel needs is two grid-barrier counters plus
// the per-chunk counts and their prefix sums. Here that scratch lives in the
// file-scope device array below, so this entry point allocates nothing: no
// cudaMalloc, cudaFree or allocating library routine.
//
// Shared scratch: every call on a device uses the same array, and it keeps
// whatever the last call left in it. Each call zeroes the barrier counters
// (a stream-ordered memset of 256 bytes). The kernel overwrites every other
// entry it reads within the call. Calls whose work overlaps on the GPU (two
// streams, or two host threads) race on the array and give wrong layouts.
// Order them on one stream. Every GPU that loads
// this library holds the array (2 MiB) until the process exits.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "ep.h"
#include "internal.h"

namespace {

// 2 MiB. The layout grid is capped so its chunk scratch fits:
// (2 MiB/4 - 64 - (E+R)) / (E+R) CTAs, e.g. all 1024 at E = 256, R = 8,
// and 495 at E = 1024, R = 32.
constexpr int64_t kNoAllocScratchInts = (2 << 20) / 4;

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Device address of g_noalloc_scratch per device, and the id of the context
// it was looked up in. A context created anew (cudaDeviceReset) loads the
// module again, and the array may then sit at another address.
int32_t* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

ep_status_t fail(ep_status_t st, const char* msg) {
    ep::set_last_error(msg);
    return st;
}

// The driver's unique id of the current context (cuCtxGetCurrent +
// cuCtxGetId, reached through the runtime's driver entry points, so the
// library needs no link to libcuda). Ids are never reused within a process.
cudaError_t current_context_id(unsigned long long* id) {
    using get_current_t = int (*)(void**);
    using get_id_t = int (*)(void*, unsigned long long*);
    static get_current_t get_current = nullptr;
    static get_id_t get_id = nullptr;
    if (!get_current || !get_id) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        cudaError_t e = cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 12000, cudaEnableDefault, &q1);
        if (e == cudaSuccess)
            e = cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &q2);
        if (e != cudaSuccess) return e;
        if (q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
            return cudaErrorSymbolNotFound;
        get_current = reinterpret_cast<get_current_t>(f1);
        get_id = reinterpret_cast<get_id_t>(f2);
    }
    void* ctx = nullptr;
    if (get_current(&ctx) != 0 || !ctx) return cudaErrorDeviceUninitialized;
    if (get_id(ctx, id) != 0) return cudaErrorDeviceUninitialized;
    return cudaSuccess;
}

// With the device current: the device address of the scratch array, looked
// up once per device and context. In host code the symbol itself is only a
// host-side stand-in, so a kernel must never be given &g_noalloc_scratch
// directly.
cudaError_t scratch_for_current_device(int32_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    unsigned long long ctx = 0;
    // fails when this host thread has no current context yet
    const bool have_ctx = current_context_id(&ctx) == cudaSuccess;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!have_ctx || !g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // makes the device's primary context current
        if (e != cudaSuccess) return e;
        e = current_context_id(&ctx);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = static_cast<int32_t*>(p);
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" ep_status_t ep_get_layout_noalloc(const ep_config_t* cfg, int T, const float* d_logits,
                                             const int32_t* d_topk_idx, const float* d_topk_w, int route,
                                             uint64_t mask_seed, float mask_frac, const ep_layout_t* out,
                                             uint32_t* d_error_word, void* stream) {
    size_t ignored = 0;
    ep_status_t st = ep_buffer_workspace_bytes(cfg, &ignored);  // validates the config
    if (st != EP_OK) return st;
    if (cfg->flags & (EP_FLAG_DEDUP | EP_FLAG_SHARD))
        return fail(EP_ERR_UNSUPPORTED, "EP_FLAG_DEDUP and EP_FLAG_SHARD layouts need a buffer: use ep_get_layout "
                                        "or ep_shard_layout");
    if (!out || !d_error_word) return fail(EP_ERR_INVALID, "out and d_error_word must be non-NULL");
    if (!out->topk_idx || !out->topk_w || !out->is_token_in_rank || !out->num_tokens_per_rank ||
        !out->cnt_src_expert || !out->num_tokens_per_expert || !out->expert_off || !out->rank_off ||
        !out->src_off || !out->dst_row)
        return fail(EP_ERR_INVALID, "every ep_layout_t output pointer must be set");
    if (T < 0) return fail(EP_ERR_INVALID, "T must be >= 0");
    if (T > cfg->max_tokens_per_rank) return fail(EP_ERR_CAPACITY, "T exceeds max_tokens_per_rank");
    const bool have_logits = d_logits != nullptr;
    const bool have_idx = d_topk_idx != nullptr || d_topk_w != nullptr;
    if (have_logits == have_idx) return fail(EP_ERR_INVALID, "pass either d_logits or d_topk_idx + d_topk_w");
    if (have_idx && (!d_topk_idx || !d_topk_w)) return fail(EP_ERR_INVALID, "d_topk_idx and d_topk_w go together");
    if (have_logits && (route < EP_ROUTE_SOFTMAX || route > EP_ROUTE_GROUP_SIGMOID))
        return fail(EP_ERR_INVALID, "unknown route");
    if (!(mask_frac >= 0.0f && mask_frac <= 1.0f)) return fail(EP_ERR_INVALID, "mask_frac must be in [0, 1]");
    const int64_t J = (int64_t)cfg->num_experts + cfg->num_ranks;
    int64_t max_ctas = (kNoAllocScratchInts - ep::layout_scratch_ints(*cfg, 0)) / J;
    if (max_ctas > ep::kMaxLayoutCtas) max_ctas = ep::kMaxLayoutCtas;

    int32_t* scratch = nullptr;
    cudaError_t e = scratch_for_current_device(&scratch);
    if (e != cudaSuccess) {
        char m[200];
        snprintf(m, sizeof m, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        return fail(EP_ERR_CUDA, m);
    }
    ep::LayoutArgs a{};
    a.T = T;
    a.logits = d_logits;
    a.in_idx = d_topk_idx;
    a.in_w = d_topk_w;
    a.route = route;
    a.mask_seed = mask_seed;
    a.mask_threshold = (uint64_t)floor((double)mask_frac * 4294967296.0);
    a.low_latency = (cfg->flags & EP_FLAG_LOW_LATENCY) ? 1 : 0;
    a.T_max = cfg->max_tokens_per_rank;
    a.m_max = a.low_latency ? (int64_t)cfg->num_experts * cfg->num_ranks * cfg->max_tokens_per_rank
                            : (int64_t)cfg->num_ranks * T * cfg->topk;  // no receive buffer: this call's rows
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    // zero the barrier words first: a call that timed out may have left them set
    e = cudaMemsetAsync(scratch, 0, sizeof(int32_t) * ep::kLayoutControlInts, cs);
    if (e == cudaSuccess)
        e = ep::launch_layout_raw(*cfg, a, *out, scratch, (int)max_ctas, d_error_word, cs);
    if (e != cudaSuccess) {
        char m[200];
        snprintf(m, sizeof m, "layout launch: %s", cudaGetErrorString(e));
        return fail(EP_ERR_CUDA, m);
    }
    ep::set_last_error("");
    return EP_OK;
}
