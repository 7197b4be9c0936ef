// C ABI of libep (declared in include/ep.h): argument validation, worst-case
// buffer sizing and partitioning, and the launches. Host code only. Every
// device computation happens in layout.cu, dispatch.cu, combine.cu, dedup.cu
// and shard.cu.
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <new>

#include "ep.h"
#include "internal.h"

namespace {

thread_local char g_msg[256] = "";

ep_status_t fail(ep_status_t st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

ep_status_t cuda_fail(cudaError_t e, const char* what) {
    return fail(EP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

ep_status_t ok() {
    g_msg[0] = '\0';
    return EP_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

ep_status_t validate(const ep_config_t* c) {
    if (!c) return fail(EP_ERR_INVALID, "config is NULL");
    if (c->num_ranks < 1 || c->num_ranks > 32) return fail(EP_ERR_UNSUPPORTED, "num_ranks must be in [1, 32]");
    if (c->max_tokens_per_rank < 1) return fail(EP_ERR_INVALID, "max_tokens_per_rank must be >= 1");
    if (c->hidden < 128 || c->hidden % 128 != 0) return fail(EP_ERR_UNSUPPORTED, "hidden must be a positive multiple of 128");
    if (c->hidden > 65536) return fail(EP_ERR_UNSUPPORTED, "hidden must be <= 65536");
    if (c->num_experts < 1 || c->num_experts > 1024) return fail(EP_ERR_UNSUPPORTED, "num_experts must be in [1, 1024]");
    if (c->num_experts % c->num_ranks != 0) return fail(EP_ERR_INVALID, "num_experts must be a multiple of num_ranks");
    if (c->topk < 1 || c->topk > 32 || c->topk > c->num_experts)
        return fail(EP_ERR_INVALID, "topk must be in [1, min(32, num_experts)]");
    if (c->num_groups < 1 || c->num_groups > 32 || c->num_experts % c->num_groups != 0)
        return fail(EP_ERR_INVALID, "num_groups must be in [1, 32] and divide num_experts");
    if (c->topk_groups < 1 || c->topk_groups > c->num_groups)
        return fail(EP_ERR_INVALID, "topk_groups must be in [1, num_groups]");
    if (c->num_groups > 1) {
        const int gs = c->num_experts / c->num_groups;
        if (gs < 2) return fail(EP_ERR_INVALID, "group-limited gating needs >= 2 experts per group");
        if (c->topk > c->topk_groups * gs) return fail(EP_ERR_INVALID, "topk exceeds the experts of the kept groups");
    }
    if (c->num_sms < 0) return fail(EP_ERR_INVALID, "num_sms must be >= 0");
    if (c->flags & ~(EP_FLAG_FP8 | EP_FLAG_LOW_LATENCY | EP_FLAG_DEDUP | EP_FLAG_SHARD))
        return fail(EP_ERR_INVALID, "unknown flag bits");
    if ((c->flags & EP_FLAG_SHARD) && (c->flags & (EP_FLAG_LOW_LATENCY | EP_FLAG_DEDUP)))
        return fail(EP_ERR_UNSUPPORTED, "EP_FLAG_SHARD does not combine with EP_FLAG_LOW_LATENCY or EP_FLAG_DEDUP");
    const int64_t m_max = (int64_t)c->num_ranks * c->max_tokens_per_rank * c->topk;
    if (m_max >= (int64_t)1 << 31) return fail(EP_ERR_UNSUPPORTED, "R*T_max*K must be < 2^31 (int32 row ids)");
    if ((c->flags & EP_FLAG_LOW_LATENCY) &&
        (int64_t)c->num_experts * c->num_ranks * c->max_tokens_per_rank >= (int64_t)1 << 31)
        return fail(EP_ERR_UNSUPPORTED, "low-latency layout: E*R*T_max must be < 2^31 (int32 row ids)");
    return EP_OK;
}

struct Plan {
    size_t off[32];
    size_t total;
};

// Region order inside the workspace; every region is 256-byte aligned.
enum {
    R_TOPK_IDX, R_TOPK_W, R_ITR, R_NTPR, R_CNT, R_NTPE, R_EOFF, R_ROFF, R_SOFF, R_DST,
    R_SCRATCH, R_ERR, R_RECV_X, R_RECV_SCALE, R_RECV_SRC, R_RECV_W,
    R_TOK_ROW, R_RANK_ROW_OFF, R_RANK_SRC_OFF, R_DD_X, R_DD_SCALE, R_DD_SRC, R_DD_TOPK_IDX, R_DD_TOPK_W, R_PARTIAL,
    R_CNT_ALL, R_DST_RANK, R_RECV_COUNT, R_RECV_OFF,
    R_COUNT
};

Plan plan_of(const ep_config_t* c, int64_t* n_max, int64_t* m_max, int64_t* nc_max) {
    const int64_t R = c->num_ranks, T = c->max_tokens_per_rank, H = c->hidden, E = c->num_experts,
                  K = c->topk;
    // one rank per GPU: the buffer holds this rank's T_max tokens, one source
    // row of counts, and receive rows for the worst case (every slot of every
    // rank lands here)
    const bool sh = (c->flags & EP_FLAG_SHARD) != 0;
    const int64_t S = sh ? 1 : R;  // source ranks whose tokens the buffer routes
    const int64_t N = S * T;
    const int64_t M = (c->flags & EP_FLAG_LOW_LATENCY) ? E * R * T : R * T * K;
    const int64_t scratch = ep::layout_scratch_ints(*c, ep::kMaxLayoutCtas);
    const bool fp8 = (c->flags & EP_FLAG_FP8) != 0;
    size_t sz[R_COUNT];
    sz[R_TOPK_IDX] = 4 * N * K;
    sz[R_TOPK_W] = 4 * N * K;
    sz[R_ITR] = N * R;
    sz[R_NTPR] = 4 * S * R;
    sz[R_CNT] = 4 * S * E;
    sz[R_NTPE] = 4 * E;
    sz[R_EOFF] = 4 * (E + 1);
    sz[R_ROFF] = 4 * (R + 1);
    sz[R_SOFF] = 4 * E * S;
    sz[R_DST] = 4 * N * K;
    sz[R_SCRATCH] = 4 * scratch;
    sz[R_ERR] = 16;
    sz[R_RECV_X] = (size_t)M * H * (fp8 ? 1 : 2);
    sz[R_RECV_SCALE] = fp8 ? (size_t)M * (H / 128) * 4 : 0;
    sz[R_RECV_SRC] = 4 * M;
    sz[R_RECV_W] = 4 * M;
    const bool dd = (c->flags & EP_FLAG_DEDUP) != 0;
    const int64_t D = dd ? R * T * (R < K ? R : K) : 0;
    sz[R_TOK_ROW] = dd ? 4 * N * R : 0;
    sz[R_RANK_ROW_OFF] = dd ? 4 * (R + 1) : 0;
    sz[R_RANK_SRC_OFF] = dd ? 4 * R * R : 0;
    sz[R_DD_X] = (size_t)D * H * (fp8 ? 1 : 2);
    sz[R_DD_SCALE] = fp8 ? (size_t)D * (H / 128) * 4 : 0;
    sz[R_DD_SRC] = 4 * D;
    sz[R_DD_TOPK_IDX] = 4 * D * K;
    sz[R_DD_TOPK_W] = 4 * D * K;
    sz[R_PARTIAL] = (size_t)D * H * 2;
    const int64_t L = E / R;
    sz[R_CNT_ALL] = sh ? 4 * R * E : 0;
    sz[R_DST_RANK] = sh ? N * K : 0;
    sz[R_RECV_COUNT] = sh ? 4 * L : 0;
    sz[R_RECV_OFF] = sh ? 4 * (L + 1) : 0;
    Plan p{};
    size_t cur = 0;
    for (int i = 0; i < R_COUNT; ++i) {
        p.off[i] = cur;
        cur += align256(sz[i]);
    }
    p.total = cur;
    *n_max = N;
    *m_max = M;
    *nc_max = ep::kMaxLayoutCtas;
    return p;
}

ep_status_t check_buf(const ep_buffer_t* b) {
    if (!b) return fail(EP_ERR_INVALID, "buffer is NULL");
    return EP_OK;
}

}  // namespace

namespace ep {
void set_last_error(const char* msg) { snprintf(g_msg, sizeof g_msg, "%s", msg); }
}  // namespace ep

extern "C" {

int ep_abi_version(void) { return EP_ABI_VERSION; }

const char* ep_status_string(ep_status_t s) {
    switch (s) {
        case EP_OK: return "EP_OK";
        case EP_ERR_INVALID: return "EP_ERR_INVALID";
        case EP_ERR_CAPACITY: return "EP_ERR_CAPACITY";
        case EP_ERR_OOM: return "EP_ERR_OOM";
        case EP_ERR_CUDA: return "EP_ERR_CUDA";
        case EP_ERR_UNSUPPORTED: return "EP_ERR_UNSUPPORTED";
        case EP_ERR_DEVICE: return "EP_ERR_DEVICE";
    }
    return "EP_ERR_UNKNOWN";
}

const char* ep_last_error_message(void) { return g_msg; }

ep_config_t ep_default_config(int num_ranks, int max_tokens_per_rank, int hidden, int num_experts, int topk) {
    ep_config_t c;
    memset(&c, 0, sizeof c);
    c.num_ranks = num_ranks;
    c.max_tokens_per_rank = max_tokens_per_rank;
    c.hidden = hidden;
    c.num_experts = num_experts;
    c.topk = topk;
    c.num_groups = 1;
    c.topk_groups = 1;
    c.num_sms = 0;
    c.flags = 0;
    return c;
}

ep_status_t ep_buffer_workspace_bytes(const ep_config_t* cfg, size_t* bytes) {
    ep_status_t st = validate(cfg);
    if (st != EP_OK) return st;
    if (!bytes) return fail(EP_ERR_INVALID, "bytes is NULL");
    int64_t n, m, nc;
    *bytes = plan_of(cfg, &n, &m, &nc).total;
    return ok();
}

ep_status_t ep_buffer_create(const ep_config_t* cfg, void* d_workspace, size_t bytes, ep_buffer_t** out) {
    ep_status_t st = validate(cfg);
    if (st != EP_OK) return st;
    if (!out) return fail(EP_ERR_INVALID, "out is NULL");
    *out = nullptr;
    if (!d_workspace) return fail(EP_ERR_INVALID, "workspace is NULL");
    if ((uintptr_t)d_workspace % 256 != 0) return fail(EP_ERR_INVALID, "workspace must be 256-byte aligned");
    int64_t n, m, nc;
    const Plan p = plan_of(cfg, &n, &m, &nc);
    if (bytes < p.total)
        return fail(EP_ERR_OOM, "workspace has %zu bytes, the worst case needs %zu", bytes, p.total);
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, d_workspace);
    if (e != cudaSuccess) return cuda_fail(e, "cudaPointerGetAttributes");
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
        return fail(EP_ERR_INVALID, "workspace is not device memory");
    int dev = attr.device, sms = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute");
    ep_buffer_t* b = new (std::nothrow) ep_buffer_t();
    if (!b) return fail(EP_ERR_OOM, "host allocation of the buffer struct failed");
    uint8_t* w = static_cast<uint8_t*>(d_workspace);
    b->cfg = *cfg;
    b->n_max = n;
    b->m_max = m;
    b->nc_max = nc;
    b->device = dev;
    b->sm_count = sms;
    b->last_T = -1;
    b->topk_idx = reinterpret_cast<int32_t*>(w + p.off[R_TOPK_IDX]);
    b->topk_w = reinterpret_cast<float*>(w + p.off[R_TOPK_W]);
    b->is_token_in_rank = w + p.off[R_ITR];
    b->num_tokens_per_rank = reinterpret_cast<int32_t*>(w + p.off[R_NTPR]);
    b->cnt = reinterpret_cast<int32_t*>(w + p.off[R_CNT]);
    b->num_tokens_per_expert = reinterpret_cast<int32_t*>(w + p.off[R_NTPE]);
    b->expert_off = reinterpret_cast<int32_t*>(w + p.off[R_EOFF]);
    b->rank_off = reinterpret_cast<int32_t*>(w + p.off[R_ROFF]);
    b->src_off = reinterpret_cast<int32_t*>(w + p.off[R_SOFF]);
    b->dst_row = reinterpret_cast<int32_t*>(w + p.off[R_DST]);
    b->scratch = reinterpret_cast<int32_t*>(w + p.off[R_SCRATCH]);
    b->err = reinterpret_cast<uint32_t*>(w + p.off[R_ERR]);
    b->recv_x = w + p.off[R_RECV_X];
    b->recv_scale = (cfg->flags & EP_FLAG_FP8) ? reinterpret_cast<float*>(w + p.off[R_RECV_SCALE]) : nullptr;
    b->recv_src = reinterpret_cast<int32_t*>(w + p.off[R_RECV_SRC]);
    b->recv_w = reinterpret_cast<float*>(w + p.off[R_RECV_W]);
    const bool dd = (cfg->flags & EP_FLAG_DEDUP) != 0;
    const int64_t R = cfg->num_ranks, K = cfg->topk;
    b->d_max = dd ? R * cfg->max_tokens_per_rank * (R < K ? R : K) : 0;
    b->tok_row = dd ? reinterpret_cast<int32_t*>(w + p.off[R_TOK_ROW]) : nullptr;
    b->rank_row_off = dd ? reinterpret_cast<int32_t*>(w + p.off[R_RANK_ROW_OFF]) : nullptr;
    b->rank_src_off = dd ? reinterpret_cast<int32_t*>(w + p.off[R_RANK_SRC_OFF]) : nullptr;
    b->dd_x = dd ? w + p.off[R_DD_X] : nullptr;
    b->dd_scale = (dd && (cfg->flags & EP_FLAG_FP8)) ? reinterpret_cast<float*>(w + p.off[R_DD_SCALE]) : nullptr;
    b->dd_src = dd ? reinterpret_cast<int32_t*>(w + p.off[R_DD_SRC]) : nullptr;
    b->dd_topk_idx = dd ? reinterpret_cast<int32_t*>(w + p.off[R_DD_TOPK_IDX]) : nullptr;
    b->dd_topk_w = dd ? reinterpret_cast<float*>(w + p.off[R_DD_TOPK_W]) : nullptr;
    b->partial = dd ? reinterpret_cast<uint16_t*>(w + p.off[R_PARTIAL]) : nullptr;
    const bool sh = (cfg->flags & EP_FLAG_SHARD) != 0;
    b->cnt_all = sh ? reinterpret_cast<int32_t*>(w + p.off[R_CNT_ALL]) : nullptr;
    b->dst_rank = sh ? w + p.off[R_DST_RANK] : nullptr;
    b->recv_count = sh ? reinterpret_cast<int32_t*>(w + p.off[R_RECV_COUNT]) : nullptr;
    b->recv_off = sh ? reinterpret_cast<int32_t*>(w + p.off[R_RECV_OFF]) : nullptr;
    b->shard_rank = -1;
    b->placed = false;
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != dev) cudaSetDevice(dev);
    // legacy-stream memset, then wait for it: callers' streams may be
    // non-blocking and would not be ordered after it otherwise
    e = cudaMemset(b->err, 0, 16);
    if (e == cudaSuccess) e = cudaMemset(b->scratch, 0, sizeof(int32_t) * ep::kLayoutControlInts);
    if (e == cudaSuccess) e = cudaStreamSynchronize(nullptr);
    if (prev != dev) cudaSetDevice(prev);
    if (e != cudaSuccess) {
        delete b;
        return cuda_fail(e, "cudaMemset(error word)");
    }
    *out = b;
    return ok();
}

ep_status_t ep_buffer_destroy(ep_buffer_t* buf) {
    delete buf;
    return ok();
}

ep_status_t ep_buffer_set_num_sms(ep_buffer_t* b, int num_sms) {
    if (ep_status_t st = check_buf(b)) return st;
    if (num_sms < 0) return fail(EP_ERR_INVALID, "num_sms must be >= 0");
    b->cfg.num_sms = num_sms;
    return ok();
}

ep_status_t ep_buffer_layout(const ep_buffer_t* b, ep_layout_t* out) {
    if (ep_status_t st = check_buf(b)) return st;
    if (!out) return fail(EP_ERR_INVALID, "out is NULL");
    out->topk_idx = b->topk_idx;
    out->topk_w = b->topk_w;
    out->is_token_in_rank = b->is_token_in_rank;
    out->num_tokens_per_rank = b->num_tokens_per_rank;
    out->cnt_src_expert = b->cnt;
    out->num_tokens_per_expert = b->num_tokens_per_expert;
    out->expert_off = b->expert_off;
    out->rank_off = b->rank_off;
    out->src_off = b->src_off;
    out->dst_row = b->dst_row;
    return ok();
}

ep_status_t ep_buffer_recv(const ep_buffer_t* b, void** recv_x, float** recv_scale, int32_t** recv_src,
                           float** recv_w, int64_t* max_rows) {
    if (ep_status_t st = check_buf(b)) return st;
    if (recv_x) *recv_x = b->recv_x;
    if (recv_scale) *recv_scale = b->recv_scale;
    if (recv_src) *recv_src = b->recv_src;
    if (recv_w) *recv_w = b->recv_w;
    if (max_rows) *max_rows = b->m_max;
    return ok();
}

static ep_status_t layout_args(const ep_buffer_t* b, int T, const float* d_logits, const int32_t* d_topk_idx,
                               const float* d_topk_w, int route, uint64_t mask_seed, float mask_frac,
                               ep::LayoutArgs* a) {
    if (T < 0) return fail(EP_ERR_INVALID, "T must be >= 0");
    if (T > b->cfg.max_tokens_per_rank)
        return fail(EP_ERR_CAPACITY, "T=%d exceeds max_tokens_per_rank=%d", T, b->cfg.max_tokens_per_rank);
    const bool have_logits = d_logits != nullptr;
    const bool have_idx = d_topk_idx != nullptr || d_topk_w != nullptr;
    if (have_logits == have_idx) return fail(EP_ERR_INVALID, "pass either d_logits or d_topk_idx + d_topk_w");
    if (have_idx && (!d_topk_idx || !d_topk_w)) return fail(EP_ERR_INVALID, "d_topk_idx and d_topk_w go together");
    if (have_logits && (route < EP_ROUTE_SOFTMAX || route > EP_ROUTE_GROUP_SIGMOID))
        return fail(EP_ERR_INVALID, "unknown route %d", route);
    if (have_logits && route == EP_ROUTE_GROUP_SIGMOID && b->cfg.num_groups > 1 &&
        b->cfg.topk > b->cfg.topk_groups * (b->cfg.num_experts / b->cfg.num_groups))
        return fail(EP_ERR_INVALID, "topk exceeds the experts of the kept groups");
    if (!(mask_frac >= 0.0f && mask_frac <= 1.0f)) return fail(EP_ERR_INVALID, "mask_frac must be in [0, 1]");
    *a = ep::LayoutArgs{};
    a->T = T;
    a->logits = d_logits;
    a->in_idx = d_topk_idx;
    a->in_w = d_topk_w;
    a->route = route;
    a->mask_seed = mask_seed;
    double thr = floor((double)mask_frac * 4294967296.0);
    a->mask_threshold = (uint64_t)thr;
    a->m_max = b->m_max;
    return EP_OK;
}

// True if [p, p + 1) lies inside the n bytes at base.
static bool points_into(const void* p, const void* base, size_t n) {
    const uintptr_t a = (uintptr_t)p, lo = (uintptr_t)base;
    return base != nullptr && a >= lo && a - lo < n;
}

// An FP8 buffer's e4m3 rows hold 1 byte per channel. Read as bf16 y (no
// scale given), rows of 2*H bytes would run past the end of the array, so
// that call is refused.
static ep_status_t check_y_not_e4m3_rows(const ep_buffer_t* b, const void* d_y, const float* d_y_scale) {
    if (!(b->cfg.flags & EP_FLAG_FP8) || d_y_scale) return EP_OK;
    const size_t H = (size_t)b->cfg.hidden;
    if (points_into(d_y, b->recv_x, (size_t)b->m_max * H) || points_into(d_y, b->dd_x, (size_t)b->d_max * H))
        return fail(EP_ERR_INVALID, "d_y points into the buffer's e4m3 rows: pass d_y_scale (fused dequant) "
                                    "or a bf16 expert output");
    return EP_OK;
}

static ep_status_t check_single(const ep_buffer_t* b) {
    if (ep_status_t st = check_buf(b)) return st;
    if (b->cfg.flags & EP_FLAG_SHARD)
        return fail(EP_ERR_INVALID, "buffer was created with EP_FLAG_SHARD: use the ep_shard_* calls");
    return EP_OK;
}

ep_status_t ep_get_layout(ep_buffer_t* b, int T, const float* d_logits, const int32_t* d_topk_idx,
                          const float* d_topk_w, int route, uint64_t mask_seed, float mask_frac, void* stream) {
    if (ep_status_t st = check_single(b)) return st;
    ep::LayoutArgs a;
    if (ep_status_t st = layout_args(b, T, d_logits, d_topk_idx, d_topk_w, route, mask_seed, mask_frac, &a))
        return st;
    cudaError_t e = ep::launch_layout(*b, a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "layout launch");
    b->last_T = T;
    return ok();
}

ep_status_t ep_dispatch(ep_buffer_t* b, int T, const void* d_x, void* stream) {
    if (ep_status_t st = check_single(b)) return st;
    if (T != b->last_T) return fail(EP_ERR_INVALID, "T=%d does not match the last ep_get_layout (T=%d)", T, b->last_T);
    if (T > 0 && !d_x) return fail(EP_ERR_INVALID, "d_x is NULL");
    if ((uintptr_t)d_x % 32 != 0) return fail(EP_ERR_INVALID, "d_x must be 32-byte aligned");
    cudaError_t e = ep::launch_dispatch(*b, T, d_x, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    return ok();
}

ep_status_t ep_combine(ep_buffer_t* b, int T, const void* d_y, const float* d_y_scale, void* d_out, void* stream) {
    if (ep_status_t st = check_single(b)) return st;
    if (T != b->last_T) return fail(EP_ERR_INVALID, "T=%d does not match the last ep_get_layout (T=%d)", T, b->last_T);
    if (T > 0 && (!d_y || !d_out)) return fail(EP_ERR_INVALID, "d_y and d_out must be non-NULL");
    if ((uintptr_t)d_y % 32 != 0 || (uintptr_t)d_out % 32 != 0)
        return fail(EP_ERR_INVALID, "d_y and d_out must be 32-byte aligned");
    if (d_y_scale && (uintptr_t)d_y_scale % 4 != 0) return fail(EP_ERR_INVALID, "d_y_scale must be 4-byte aligned");
    if (ep_status_t st = check_y_not_e4m3_rows(b, d_y, d_y_scale)) return st;
    cudaError_t e = ep::launch_combine(*b, T, d_y, d_y_scale, d_out, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    return ok();
}

ep_status_t ep_buffer_dedup(const ep_buffer_t* b, int32_t** tok_row, int32_t** rank_row_off, int32_t** rank_src_off,
                            void** dd_x, float** dd_scale, int32_t** dd_src, int32_t** dd_topk_idx, float** dd_topk_w,
                            uint16_t** partial, int64_t* max_rows) {
    if (ep_status_t st = check_buf(b)) return st;
    if (!(b->cfg.flags & EP_FLAG_DEDUP)) return fail(EP_ERR_INVALID, "buffer was created without EP_FLAG_DEDUP");
    if (tok_row) *tok_row = b->tok_row;
    if (rank_row_off) *rank_row_off = b->rank_row_off;
    if (rank_src_off) *rank_src_off = b->rank_src_off;
    if (dd_x) *dd_x = b->dd_x;
    if (dd_scale) *dd_scale = b->dd_scale;
    if (dd_src) *dd_src = b->dd_src;
    if (dd_topk_idx) *dd_topk_idx = b->dd_topk_idx;
    if (dd_topk_w) *dd_topk_w = b->dd_topk_w;
    if (partial) *partial = b->partial;
    if (max_rows) *max_rows = b->d_max;
    return ok();
}

static ep_status_t check_dedup_call(const ep_buffer_t* b, int T) {
    if (ep_status_t st = check_buf(b)) return st;
    if (!(b->cfg.flags & EP_FLAG_DEDUP)) return fail(EP_ERR_INVALID, "buffer was created without EP_FLAG_DEDUP");
    if (T != b->last_T) return fail(EP_ERR_INVALID, "T=%d does not match the last ep_get_layout (T=%d)", T, b->last_T);
    return EP_OK;
}

ep_status_t ep_dispatch_dedup(ep_buffer_t* b, int T, const void* d_x, void* stream) {
    if (ep_status_t st = check_dedup_call(b, T)) return st;
    if (T > 0 && !d_x) return fail(EP_ERR_INVALID, "d_x is NULL");
    if ((uintptr_t)d_x % 32 != 0) return fail(EP_ERR_INVALID, "d_x must be 32-byte aligned");
    cudaError_t e = ep::launch_dispatch_dedup(*b, T, d_x, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dispatch_dedup launch");
    return ok();
}

ep_status_t ep_permute(ep_buffer_t* b, int T, void* stream) {
    if (ep_status_t st = check_dedup_call(b, T)) return st;
    cudaError_t e = ep::launch_permute(*b, T, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "permute launch");
    return ok();
}

ep_status_t ep_local_reduce(ep_buffer_t* b, int T, const void* d_y, const float* d_y_scale, void* stream) {
    if (ep_status_t st = check_dedup_call(b, T)) return st;
    if (T > 0 && !d_y) return fail(EP_ERR_INVALID, "d_y is NULL");
    if ((uintptr_t)d_y % 32 != 0) return fail(EP_ERR_INVALID, "d_y must be 32-byte aligned");
    if (d_y_scale && (uintptr_t)d_y_scale % 4 != 0) return fail(EP_ERR_INVALID, "d_y_scale must be 4-byte aligned");
    if (ep_status_t st = check_y_not_e4m3_rows(b, d_y, d_y_scale)) return st;
    cudaError_t e = ep::launch_local_reduce(*b, T, d_y, d_y_scale, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "local_reduce launch");
    return ok();
}

ep_status_t ep_combine_dedup(ep_buffer_t* b, int T, void* d_out, void* stream) {
    if (ep_status_t st = check_dedup_call(b, T)) return st;
    if (T > 0 && !d_out) return fail(EP_ERR_INVALID, "d_out is NULL");
    if ((uintptr_t)d_out % 32 != 0) return fail(EP_ERR_INVALID, "d_out must be 32-byte aligned");
    cudaError_t e = ep::launch_combine_dedup(*b, T, d_out, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "combine_dedup launch");
    return ok();
}

/* ---- one rank per GPU (EP_FLAG_SHARD) ------------------------------------ */

static ep_status_t check_shard(const ep_buffer_t* b) {
    if (ep_status_t st = check_buf(b)) return st;
    if (!(b->cfg.flags & EP_FLAG_SHARD)) return fail(EP_ERR_INVALID, "buffer was created without EP_FLAG_SHARD");
    return EP_OK;
}

static ep_status_t check_shard_step(const ep_buffer_t* b, int rank, int T, bool need_placed) {
    if (ep_status_t st = check_shard(b)) return st;
    if (b->shard_rank < 0) return fail(EP_ERR_INVALID, "no ep_shard_layout on this buffer yet");
    if (rank != b->shard_rank)
        return fail(EP_ERR_INVALID, "rank=%d does not match the last ep_shard_layout (rank=%d)", rank, b->shard_rank);
    if (T != b->last_T) return fail(EP_ERR_INVALID, "T=%d does not match the last ep_shard_layout (T=%d)", T, b->last_T);
    if (need_placed && !b->placed) return fail(EP_ERR_INVALID, "call ep_shard_place after ep_shard_layout first");
    return EP_OK;
}

ep_status_t ep_buffer_shard(const ep_buffer_t* b, int32_t** cnt_row, int32_t** cnt_all, uint8_t** dst_rank,
                            int32_t** recv_count, int32_t** recv_off) {
    if (ep_status_t st = check_shard(b)) return st;
    if (cnt_row) *cnt_row = b->cnt;
    if (cnt_all) *cnt_all = b->cnt_all;
    if (dst_rank) *dst_rank = b->dst_rank;
    if (recv_count) *recv_count = b->recv_count;
    if (recv_off) *recv_off = b->recv_off;
    return ok();
}

ep_status_t ep_shard_layout(ep_buffer_t* b, int rank, int T, const float* d_logits, const int32_t* d_topk_idx,
                            const float* d_topk_w, int route, uint64_t mask_seed, float mask_frac, void* stream) {
    if (ep_status_t st = check_shard(b)) return st;
    if (rank < 0 || rank >= b->cfg.num_ranks)
        return fail(EP_ERR_INVALID, "rank=%d outside [0, %d)", rank, b->cfg.num_ranks);
    ep::LayoutArgs a;
    if (ep_status_t st = layout_args(b, T, d_logits, d_topk_idx, d_topk_w, route, mask_seed, mask_frac, &a))
        return st;
    a.S = 1;
    a.g_base = (int64_t)rank * T;
    cudaError_t e = ep::launch_layout(*b, a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "shard layout launch");
    b->last_T = T;
    b->shard_rank = rank;
    b->placed = false;
    return ok();
}

ep_status_t ep_shard_place(ep_buffer_t* b, int rank, int T, void* stream) {
    if (ep_status_t st = check_shard_step(b, rank, T, false)) return st;
    if (b->placed) return fail(EP_ERR_INVALID, "ep_shard_place already ran for this ep_shard_layout");
    cudaError_t e = ep::launch_shard_place(*b, rank, T, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "shard place launch");
    b->placed = true;
    return ok();
}

ep_status_t ep_shard_dispatch(ep_buffer_t* b, int rank, int T, const void* d_x, void* const* peer_recv_x,
                              float* const* peer_recv_scale, int32_t* const* peer_recv_src,
                              float* const* peer_recv_w, void* stream) {
    if (ep_status_t st = check_shard_step(b, rank, T, true)) return st;
    if (T > 0 && !d_x) return fail(EP_ERR_INVALID, "d_x is NULL");
    if ((uintptr_t)d_x % 32 != 0) return fail(EP_ERR_INVALID, "d_x must be 32-byte aligned");
    if (!peer_recv_x || !peer_recv_src || !peer_recv_w)
        return fail(EP_ERR_INVALID, "peer_recv_x, peer_recv_src and peer_recv_w must be non-NULL");
    const bool fp8 = (b->cfg.flags & EP_FLAG_FP8) != 0;
    if (fp8 && !peer_recv_scale) return fail(EP_ERR_INVALID, "EP_FLAG_FP8 needs peer_recv_scale");
    for (int d = 0; d < b->cfg.num_ranks; ++d) {
        if (!peer_recv_x[d] || !peer_recv_src[d] || !peer_recv_w[d] || (fp8 && !peer_recv_scale[d]))
            return fail(EP_ERR_INVALID, "peer table entry %d is NULL", d);
        if ((uintptr_t)peer_recv_x[d] % 32 != 0) return fail(EP_ERR_INVALID, "peer_recv_x[%d] must be 32-byte aligned", d);
        if ((uintptr_t)peer_recv_src[d] % 4 != 0 || (uintptr_t)peer_recv_w[d] % 4 != 0 ||
            (fp8 && (uintptr_t)peer_recv_scale[d] % 4 != 0))
            return fail(EP_ERR_INVALID, "peer table entry %d must be 4-byte aligned", d);
    }
    cudaError_t e = ep::launch_shard_dispatch(*b, rank, T, d_x, peer_recv_x, fp8 ? peer_recv_scale : nullptr,
                                              peer_recv_src, peer_recv_w, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "shard dispatch launch");
    return ok();
}

ep_status_t ep_shard_combine(ep_buffer_t* b, int rank, int T, const void* const* peer_y,
                             const float* const* peer_y_scale, void* d_out, void* stream) {
    if (ep_status_t st = check_shard_step(b, rank, T, true)) return st;
    if (T > 0 && !d_out) return fail(EP_ERR_INVALID, "d_out is NULL");
    if ((uintptr_t)d_out % 32 != 0) return fail(EP_ERR_INVALID, "d_out must be 32-byte aligned");
    if (!peer_y) return fail(EP_ERR_INVALID, "peer_y is NULL");
    for (int d = 0; d < b->cfg.num_ranks; ++d) {
        if (!peer_y[d] || (peer_y_scale && !peer_y_scale[d]))
            return fail(EP_ERR_INVALID, "peer table entry %d is NULL", d);
        if ((uintptr_t)peer_y[d] % 32 != 0) return fail(EP_ERR_INVALID, "peer_y[%d] must be 32-byte aligned", d);
        if (peer_y_scale && (uintptr_t)peer_y_scale[d] % 4 != 0)
            return fail(EP_ERR_INVALID, "peer_y_scale[%d] must be 4-byte aligned", d);
    }
    cudaError_t e = ep::launch_shard_combine(*b, T, peer_y, peer_y_scale, d_out, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "shard combine launch");
    return ok();
}

ep_status_t ep_check_errors(ep_buffer_t* b, uint32_t* word, int clear, void* stream) {
    if (ep_status_t st = check_buf(b)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, b->err, sizeof v, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && clear) {
        // also reset the layout's barrier words, which a timed-out launch may leave set
        e = cudaMemsetAsync(b->err, 0, sizeof v, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(b->scratch, 0, sizeof(int32_t) * ep::kLayoutControlInts, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "ep_check_errors");
    if (word) *word = v;
    if (v) return fail(EP_ERR_DEVICE, "device error word 0x%x", v);
    return ok();
}

ep_status_t ep_selftest_wait_timeout(uint32_t* d_words, uint64_t limit_ns, uint32_t* word, void* stream) {
    if (!d_words || !word) return fail(EP_ERR_INVALID, "d_words and word must be non-NULL");
    if (limit_ns < 1000 || limit_ns > 2000000000ull) return fail(EP_ERR_INVALID, "limit_ns must be in [1 us, 2 s]");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = ep::launch_barrier_timeout_selftest(d_words, limit_ns, s);
    if (e == cudaSuccess) e = ep::launch_mbarrier_timeout_selftest(d_words + 2, d_words + 3, limit_ns, s);
    uint32_t v = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&v, d_words + 2, sizeof v, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "ep_selftest_wait_timeout");
    *word = v;
    return ok();
}

}  // extern "C"
