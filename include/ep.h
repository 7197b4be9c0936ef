/*
 * ep.h -- C ABI of libep.so: MoE expert-parallel routing + layout, dispatch
 * and combine on one B200 (sm_100a). EP ranks are emulated as disjoint
 * receive partitions of one GPU's memory.
 *
 * The operations follow the DeepEP pages:
 *  - "DeepEP：年度总结中的计算通信重叠摘记" (DeepEP overlap notes):
 *    - §计算-通信重叠: group-limited gating;
 *    - §节点内通信: Top-K fused into the communication kernel,
 *      is_token_in_rank, sending only to target ranks, FP8 at 1 byte per
 *      element.
 *  - "DeepEP：面向MoE的高吞吐低延迟GPU通信库" (DeepEP summary):
 *    - §工程化: dispatch and combine kernels;
 *    - "如何调优 Buffer.set_num_sms": get_*_config and set_num_sms.
 *  - the rocSHMEM / DeepEP buffer notes (mlqm.cn), §3.2 "RDMA buffer的问题":
 *    one communication buffer, allocated once and sized for the worst case.
 *
 * Conventions for every function below:
 *  - Pointers named d_* and every pointer handed out by ep_buffer_* are DEVICE
 *    pointers. All others are host pointers.
 *  - The caller owns all device memory: the workspace, the inputs and the
 *    outputs. The library never allocates or frees device memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is stream-ordered. Only ep_check_errors blocks the host.
 *  - Argument errors are caught on the host before any launch and returned as
 *    a status. ep_last_error_message() then gives a one-line reason.
 *  - Data errors found on the device (an expert id out of range, a row index
 *    outside the buffer, a bounded wait that gave up) set bits of the
 *    buffer's device error word. The kernels never trap. ep_check_errors
 *    reads the word.
 *  - A buffer is not thread-safe. Use one buffer per stream.
 */
#ifndef COMBINE_TOP_GROUP_EP_H
#define COMBINE_TOP_GROUP_EP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EP_ABI_VERSION 2

typedef enum {
    EP_OK = 0,
    EP_ERR_INVALID = 1,     /* bad argument or shape */
    EP_ERR_CAPACITY = 2,    /* more tokens than the buffer was sized for */
    EP_ERR_OOM = 3,         /* workspace smaller than ep_buffer_workspace_bytes */
    EP_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    EP_ERR_UNSUPPORTED = 5, /* a valid shape the library does not handle */
    EP_ERR_DEVICE = 6       /* ep_check_errors found device error bits */
} ep_status_t;

/* Bits of the device error word. */
#define EP_DEVERR_EXPERT_ID 0x1u  /* an expert id outside [-1, E); the slot was treated as masked */
#define EP_DEVERR_ROW_BOUNDS 0x2u /* a receive row outside [0, M_max); the copy was skipped */
#define EP_DEVERR_TIMEOUT 0x4u    /* a bounded wait inside a kernel gave up */

/* ep_config_t.flags */
#define EP_FLAG_FP8 0x1u /* dispatch casts to FP8 e4m3 with one fp32 scale per 128 channels */
/* Low-latency (decode) receive layout, after the pages' low-latency kernels
 * (DeepEP overlap notes, §计算-通信重叠). Expert e's rows from source rank s
 * live in a fixed region of T_max rows: row = (e*R + s)*T_max + j, where j
 * counts s's earlier slots (in token, slot order) that chose e. No prefix sum
 * across ranks places a row. The buffer then holds M_max = E*R*T_max receive
 * rows. The counts and prefix sums in ep_layout_t keep their meaning. In this
 * mode cnt_src_expert[s][e] tells how much of region (e, s) is filled. A
 * region overflows only if a caller's top-k repeats an expert; the extra
 * slots are dropped with EP_DEVERR_ROW_BOUNDS. */
#define EP_FLAG_LOW_LATENCY 0x2u
/* Deduplicated receive (DeepEP overlap notes, §节点内通信: a token is sent only
 * to the ranks is_token_in_rank marks). The buffer also holds one row per
 * (token, destination rank): at most R*T_max*min(R, K) rows, ordered by
 * (destination rank, source rank, token). ep_get_layout then also fills the
 * dedup layout (ep_buffer_dedup), and ep_dispatch_dedup, ep_permute,
 * ep_local_reduce and ep_combine_dedup become available. */
#define EP_FLAG_DEDUP 0x4u
/* One rank per GPU: the buffer belongs to ONE rank of R and holds its own
 * T_max tokens' layout and its own receive rows (the ep_shard_* calls below).
 * Not combinable with EP_FLAG_LOW_LATENCY or EP_FLAG_DEDUP. */
#define EP_FLAG_SHARD 0x8u

/* Routing rule applied by ep_get_layout to router logits. */
typedef enum {
    EP_ROUTE_SOFTMAX = 0,        /* top-K by logit; w = softmax probability */
    EP_ROUTE_SOFTMAX_RENORM = 1, /* as above, w renormalised over the K chosen */
    EP_ROUTE_GROUP_SIGMOID = 2   /* group-limited sigmoid gating (DeepEP overlap notes, §计算-通信重叠) */
} ep_route_t;

/* Buffer configuration. The ep_default_config analogue of DeepEP's
 * Buffer.get_*_config (DeepEP summary, "如何调优 Buffer.set_num_sms"). */
typedef struct {
    int32_t num_ranks;           /* R: emulated EP ranks, 1..32 */
    int32_t max_tokens_per_rank; /* T_max: capacity per rank, >= 1 */
    int32_t hidden;              /* H: channels per token, a multiple of 128 */
    int32_t num_experts;         /* E: a multiple of R, at most 1024; expert e lives on rank e / (E/R) */
    int32_t topk;                /* K: 1..min(32, E) */
    int32_t num_groups;          /* G: expert groups for group-limited gating (1 = none); E % G == 0 */
    int32_t topk_groups;         /* KG: groups kept per token, 1..G */
    int32_t num_sms;             /* SM cap for the data-movement kernels (0 = all), cf. Buffer.set_num_sms */
    uint32_t flags;              /* EP_FLAG_* */
} ep_config_t;

typedef struct ep_buffer ep_buffer_t;

/* Device views of the layout produced by ep_get_layout. N = R*T of the last
 * call. Row-major arrays, int32 unless stated. */
typedef struct {
    int32_t *topk_idx;              /* [N, K]; -1 = masked slot */
    float *topk_w;                  /* [N, K] fp32; 0 for masked slots */
    uint8_t *is_token_in_rank;      /* [N, R] 0/1 (DeepEP overlap notes, §节点内通信) */
    int32_t *num_tokens_per_rank;   /* [R_src, R_dst]: distinct tokens of source s that go to rank r */
    int32_t *cnt_src_expert;        /* [R_src, E]: slots of source s routed to expert e */
    int32_t *num_tokens_per_expert; /* [E]: receive rows of expert e */
    int32_t *expert_off;            /* [E+1]: exclusive prefix sum of num_tokens_per_expert */
    int32_t *rank_off;              /* [R+1]: rank_off[r] = expert_off[r*E/R] (partition of rank r) */
    int32_t *src_off;               /* [E, R]: offset of source s inside expert e's rows */
    int32_t *dst_row;               /* [N, K]: receive row of slot (g,k); -1 if masked */
} ep_layout_t;

/* Returns EP_ABI_VERSION. */
int ep_abi_version(void);

/* Static name of a status code. */
const char *ep_status_string(ep_status_t status);

/* One-line reason for the last non-OK status returned on this host thread
 * ("" if none). */
const char *ep_last_error_message(void);

/* Config with no group limit, num_sms = 0, flags = 0. */
ep_config_t ep_default_config(int num_ranks, int max_tokens_per_rank, int hidden,
                              int num_experts, int topk);

/* Workspace bytes needed by a buffer with this config. This is the worst
 * case: M_max = R * T_max * K receive rows in total, which no routing can
 * exceed (rocSHMEM / DeepEP buffer notes, §3.2: size for the worst case,
 * allocate once). EP_ERR_INVALID / EP_ERR_UNSUPPORTED for bad configs. */
ep_status_t ep_buffer_workspace_bytes(const ep_config_t *cfg, size_t *bytes);

/* Wrap a caller-allocated device workspace (256-byte aligned, at least
 * ep_buffer_workspace_bytes long) in a buffer handle. Zeroes the device error
 * word with a synchronous cudaMemset. The handle is a small host struct, freed
 * by ep_buffer_destroy. The workspace must outlive the handle.
 * Errors: EP_ERR_INVALID (NULL or misaligned), EP_ERR_OOM (too small),
 * EP_ERR_CUDA. */
ep_status_t ep_buffer_create(const ep_config_t *cfg, void *d_workspace, size_t bytes,
                             ep_buffer_t **out);

/* Frees the host struct only. NULL is a no-op. */
ep_status_t ep_buffer_destroy(ep_buffer_t *buf);

/* Sets the SM budget of the buffer's dispatch and combine kernels (the
 * standard, shard and deduplicated ones; not ep_get_layout): with
 * 0 < num_sms < the device's SM count, each such kernel launches at most
 * num_sms CTAs, so it occupies at most num_sms SMs, and each CTA loops over
 * tokens. A CTA is made as large as one SM holds where the kernel allows it
 * (several token groups per CTA in dispatch and the register combines; a
 * bulk-copy pipeline of one CTA per SM in the bf16 combine). 0, or a count
 * at or above the SM count, = all SMs. This is the analogue of DeepEP's
 * Buffer.set_num_sms (DeepEP summary, "如何调优 Buffer.set_num_sms"; DeepEP
 * overlap notes, §节点内通信: 20 communication SMs, the rest for compute).
 * It takes effect from the next call. Results are identical under any
 * budget.
 * Errors: EP_ERR_INVALID for num_sms < 0. */
ep_status_t ep_buffer_set_num_sms(ep_buffer_t *buf, int num_sms);

/* Device views of the layout arrays inside the workspace. */
ep_status_t ep_buffer_layout(const ep_buffer_t *buf, ep_layout_t *out);

/* Device views of the receive buffers, M_max rows each (R*T_max*K, or
 * E*R*T_max with EP_FLAG_LOW_LATENCY):
 *  recv_x      bf16 [M_max, H], or e4m3 [M_max, H] with EP_FLAG_FP8;
 *  recv_scale  fp32 [M_max, H/128] with EP_FLAG_FP8, else NULL;
 *  recv_src    int32 [M_max]: source token g of each row;
 *  recv_w      fp32 [M_max]: routing weight of each row.
 * The rows of rank r are [rank_off[r], rank_off[r+1]) (low-latency mode:
 * [r*(E/R)*R*T_max, (r+1)*(E/R)*R*T_max)). Any out-pointer may be
 * NULL. Also returns M_max through *max_rows if it is not NULL. */
ep_status_t ep_buffer_recv(const ep_buffer_t *buf, void **recv_x, float **recv_scale,
                           int32_t **recv_src, float **recv_w, int64_t *max_rows);

/* Routing + layout for T tokens per rank (N = R*T, token g = s*T + t of
 * source rank s). Top-K fused with the layout (DeepEP overlap notes,
 * §节点内通信).
 * Inputs, exactly one of:
 *  - d_logits: fp32 [N, E] router logits, routed by `route`;
 *  - d_topk_idx: int32 [N, K] plus d_topk_w: fp32 [N, K], taken as given.
 *    Ids outside [-1, E) set EP_DEVERR_EXPERT_ID and become masked slots.
 * mask_frac > 0 then masks slot (g,k) to -1 (weight 0) when the high 32 bits
 * of splitmix64(mask_seed ^ (g*K + k)) fall below floor(mask_frac * 2^32).
 * Writes every ep_layout_t array. Receive rows are ordered by
 * (expert, source rank, token, slot).
 * Errors: EP_ERR_CAPACITY if T > T_max; EP_ERR_INVALID for bad pointers, T,
 * route or mask_frac. */
ep_status_t ep_get_layout(ep_buffer_t *buf, int T, const float *d_logits,
                          const int32_t *d_topk_idx, const float *d_topk_w, int route,
                          uint64_t mask_seed, float mask_frac, void *stream);

/* Dispatch (DeepEP summary, §工程化; only to the target experts, DeepEP
 * overlap notes, §节点内通信). For every unmasked slot (g,k):
 *  - recv_x[dst_row[g,k]] = x[g];
 *  - recv_src[row] = g;
 *  - recv_w[row] = topk_w[g,k].
 * With EP_FLAG_FP8 each 128-channel block is cast as:
 *  - amax = max(max|x|, 1e-4);
 *  - q = e4m3_rne_satfinite(x * (448/amax));
 *  - recv_scale = amax/448.
 * d_x: bf16 [N, H] row-major, 32-byte aligned. T must equal the T of the
 * last ep_get_layout on this buffer. Errors: EP_ERR_INVALID. */
ep_status_t ep_dispatch(ep_buffer_t *buf, int T, const void *d_x, void *stream);

/* Combine (DeepEP summary, §工程化):
 *   out[g] = bf16_rne( sum over k ascending, unmasked, of w[g,k] * y[dst_row[g,k]] )
 * accumulated in fp32 with one fused multiply-add per slot. d_y_scale == NULL:
 * d_y is bf16 [rows, H]. Otherwise d_y is e4m3 [rows, H] and is dequantised
 * in the kernel as e4m3 * d_y_scale[row, h/128] (fp32) before the fma.
 * rows >= expert_off[E]. d_out: bf16 [N, H]. d_y and d_out 32-byte aligned.
 * T must equal the T of the last ep_get_layout. A token whose slots are all
 * masked gets +0. Errors: EP_ERR_INVALID, also when the buffer has
 * EP_FLAG_FP8, d_y_scale is NULL and d_y points into the buffer's own e4m3
 * rows (read as bf16 they would run past the end of the array). */
ep_status_t ep_combine(ep_buffer_t *buf, int T, const void *d_y, const float *d_y_scale,
                       void *d_out, void *stream);

/* Synchronises `stream` and reads the device error word into *word. clear != 0
 * then resets it to 0, together with the layout's grid-barrier words. After
 * EP_DEVERR_TIMEOUT, call it with clear != 0 before the next ep_get_layout. Returns EP_ERR_DEVICE if any bit was set, EP_OK if
 * none, EP_ERR_CUDA on a CUDA failure. */
ep_status_t ep_check_errors(ep_buffer_t *buf, uint32_t *word, int clear, void *stream);

/* ---- deduplicated receive (EP_FLAG_DEDUP) ---------------------------------
 * DeepEP overlap notes, §节点内通信: a token travels only to the ranks
 * is_token_in_rank marks, once per rank. The receiving rank then:
 *  - permutes the rows into expert order for its experts;
 *  - reduces its experts' outputs into one bf16 partial row per (token, rank);
 *  - hands the partials back, where they are summed across ranks.
 * All calls below need a buffer created with EP_FLAG_DEDUP, and T equal to the
 * last ep_get_layout's. They are stream-ordered, so each call follows the one
 * before it on the same stream. */

/* Device views of the dedup layout and buffers:
 *  tok_row      int32 [N, R]: row of token g on rank r, -1 if not sent;
 *  rank_row_off int32 [R+1]: exclusive prefix of the rows per destination rank (D = rank_row_off[R]);
 *  rank_src_off int32 [R, R]: [r][s] = offset of source s inside rank r's rows;
 *  dd_x         [D_max, H]: bf16, or e4m3 with dd_scale fp32 [D_max, H/128] (EP_FLAG_FP8);
 *  dd_src       int32 [D_max]: source token of each row;
 *  dd_topk_idx  int32 [D_max, K]: the token's top-k, -1 where the expert is not on this rank;
 *  dd_topk_w    fp32 [D_max, K]: the matching weights (0 where -1);
 *  partial      bf16 [D_max, H]: ep_local_reduce output.
 * D_max = R*T_max*min(R, K). Any out-pointer may be NULL. */
ep_status_t ep_buffer_dedup(const ep_buffer_t *buf, int32_t **tok_row, int32_t **rank_row_off,
                            int32_t **rank_src_off, void **dd_x, float **dd_scale, int32_t **dd_src,
                            int32_t **dd_topk_idx, float **dd_topk_w, uint16_t **partial, int64_t *max_rows);

/* Dedup dispatch: for every rank r with tok_row[g][r] != -1, row tok_row[g][r]
 * gets x[g] (bf16 copy, or the same FP8 cast as ep_dispatch), g, and the
 * localised top-k. d_x as for ep_dispatch. Errors: EP_ERR_INVALID. */
ep_status_t ep_dispatch_dedup(ep_buffer_t *buf, int T, const void *d_x, void *stream);

/* Local expert permutation: each dedup row is copied to the expert-grouped
 * receive row (recv_x, recv_scale, recv_src, recv_w, as ep_dispatch writes
 * them) of each of its local slots. Follows ep_dispatch_dedup. */
ep_status_t ep_permute(ep_buffer_t *buf, int T, void *stream);

/* Local reduce: partial[d] = bf16( sum over the row's local slots k
 * ascending, fp32 fma, of w * y[dst_row[g][k]] ). y as for ep_combine (bf16,
 * or e4m3 + d_y_scale), 32-byte aligned. Errors: EP_ERR_INVALID, also for
 * the buffer's own e4m3 rows (recv_x or dd_x) passed without d_y_scale. */
ep_status_t ep_local_reduce(ep_buffer_t *buf, int T, const void *d_y, const float *d_y_scale, void *stream);

/* Dedup combine: out[g] = bf16( sum over ranks r ascending, fp32, of
 * partial[tok_row[g][r]] ); +0 for a token sent nowhere. d_out bf16 [N, H],
 * 32-byte aligned. */
ep_status_t ep_combine_dedup(ep_buffer_t *buf, int T, void *d_out, void *stream);

/* ---- one rank per GPU (EP_FLAG_SHARD) -------------------------------------
 * The method as a node runs it: one process per GPU, each rank holding its own
 * T tokens and the receive rows of its own E/R experts. Dispatch and combine
 * then cross NVLink inside the node. The counts are exchanged first, and each
 * rank writes its tokens straight into the receivers' buffers (DeepEP overlap
 * notes, §节点内通信).
 *
 * A rank's buffer, created with EP_FLAG_SHARD and the same config on every
 * rank, holds:
 *  - the layout of the rank's own tokens, as ep_buffer_layout views with
 *    N = T (one source rank):
 *    - topk_idx, topk_w and dst_row [T, K], is_token_in_rank [T, R];
 *    - num_tokens_per_rank [1, R] and cnt_src_expert [1, E]: this rank's row;
 *  - cnt_all [R, E], dst_rank [T_max, K] and the receive counts
 *    (ep_buffer_shard);
 *  - receive rows for the worst case: M_max = R*T_max*K, every slot of every
 *    rank on this rank (ep_buffer_recv).
 *
 * One step, on every rank s. Token g = s*T + t, with T the same on every rank:
 *  1. ep_shard_layout: routing and the rank-local layout of s's T tokens. It
 *     fills s's count row cnt[s][e].
 *  2. The caller all-gathers the R count rows into every rank's cnt_all, for
 *     example with an NCCL all-gather of R*E int32.
 *  3. ep_shard_place: the row of each of s's slots on its destination rank
 *     d = e / (E/R), and s's own receive counts.
 *  4. The caller's barrier: every rank has finished reading its receive rows
 *     from the step before.
 *  5. ep_shard_dispatch: s's rows are stored into the destination ranks'
 *     receive arrays, through tables of their device pointers. These are
 *     peer-mapped pointers when the rank is another GPU.
 *  6. The caller's barrier. Then expert work runs on each rank's own rows
 *     [0, recv_off[E/R]).
 *  7. ep_shard_combine: s's tokens are gathered from the ranks' expert
 *     outputs, through pointer tables.
 * There is no wait inside a kernel. The caller orders the ranks with
 * collectives or barriers between the calls.
 *
 * Rank d's receive rows are rows [rank_off[d], rank_off[d+1]) of the
 * single-buffer layout (ep_get_layout over all R*T tokens), shifted to start
 * at 0: the same rows in the same order, (expert, source rank, token, slot).
 * recv_src holds global token ids. dst_rank and dst_row index the
 * destination's arrays. */

/* Device views of the shard arrays:
 *  cnt_row     int32 [E]: this rank's slots per expert (from ep_shard_layout),
 *              the row to all-gather;
 *  cnt_all     int32 [R, E]: the gathered rows; row s = rank s's cnt_row;
 *  dst_rank    uint8 [T_max, K]: destination rank of each slot (after ep_shard_place);
 *  recv_count  int32 [E/R]: rows this rank receives for each local expert;
 *  recv_off    int32 [E/R + 1]: their exclusive prefix; recv_off[E/R] is
 *              this rank's receive row count.
 * Any out-pointer may be NULL. EP_ERR_INVALID without EP_FLAG_SHARD. */
ep_status_t ep_buffer_shard(const ep_buffer_t *buf, int32_t **cnt_row, int32_t **cnt_all, uint8_t **dst_rank,
                            int32_t **recv_count, int32_t **recv_off);

/* Step 1: routing and the rank-local layout of rank `rank`'s T tokens. The
 * inputs are as for ep_get_layout, but over [T, E] logits or [T, K] top-k.
 * The slot mask hashes global ids (g = rank*T + t). Afterwards dst_row holds
 * rank-local rows: this rank's exclusive expert offset plus the slot's
 * position among the rank's earlier slots of that expert.
 * Errors: as ep_get_layout, and EP_ERR_INVALID for a rank outside [0, R). */
ep_status_t ep_shard_layout(ep_buffer_t *buf, int rank, int T, const float *d_logits,
                            const int32_t *d_topk_idx, const float *d_topk_w, int route,
                            uint64_t mask_seed, float mask_frac, void *stream);

/* Step 3: reads cnt_all (the caller has filled it by step 2 on the same
 * stream) and turns every slot's dst_row into its row on the destination
 * rank, with that rank in dst_rank. Also writes this rank's recv_count and
 * recv_off. Once per ep_shard_layout. rank and T must be those of the last
 * ep_shard_layout. A row outside [0, M_max) sets EP_DEVERR_ROW_BOUNDS and
 * becomes -1. */
ep_status_t ep_shard_place(ep_buffer_t *buf, int rank, int T, void *stream);

/* Step 5: for every unmasked slot (t,k) of this rank, destination d =
 * dst_rank[t,k] and row r = dst_row[t,k]:
 *  - peer_recv_x[d][r] = x[t], bf16 or cast to FP8 as in ep_dispatch;
 *  - peer_recv_scale[d][r] = the FP8 scales;
 *  - peer_recv_src[d][r] = rank*T + t;
 *  - peer_recv_w[d][r] = topk_w[t,k].
 * The peer_* arguments are HOST arrays of R device pointers: entry d is rank
 * d's receive array (ep_buffer_recv on rank d). Pointers into other GPUs must
 * be usable from this GPU: peer access enabled, or IPC or symmetric-memory
 * mappings. Every entry is non-NULL. peer_recv_x entries are 32-byte aligned;
 * peer_recv_scale may be NULL without EP_FLAG_FP8. d_x: bf16 [T, H], 32-byte
 * aligned. Needs ep_shard_place first. The kernel makes its stores complete
 * at system scope before it ends, so a collective that follows it on
 * `stream` (the barrier of step 6) orders them for the receiving ranks.
 * Errors: EP_ERR_INVALID. */
ep_status_t ep_shard_dispatch(ep_buffer_t *buf, int rank, int T, const void *d_x,
                              void *const *peer_recv_x, float *const *peer_recv_scale,
                              int32_t *const *peer_recv_src, float *const *peer_recv_w, void *stream);

/* Step 7: out[t] = bf16_rne( sum over k ascending, unmasked, of
 * w[t,k] * y_d[dst_row[t,k]] ), with d = dst_rank[t,k]. The sum is fp32 with
 * one fused multiply-add per slot, as ep_combine computes it. peer_y is a
 * HOST array of R device pointers to each rank's expert output: bf16
 * [rows, H], or e4m3 [rows, H] with peer_y_scale (a host array of R fp32
 * [rows, H/128] pointers) for the fused dequantisation. NULL peer_y_scale
 * means bf16. d_out: bf16 [T, H]. peer_y entries and d_out are 32-byte
 * aligned. Needs ep_shard_place first. Errors: EP_ERR_INVALID. */
ep_status_t ep_shard_combine(ep_buffer_t *buf, int rank, int T, const void *const *peer_y,
                             const float *const *peer_y_scale, void *d_out, void *stream);

/* Diagnostic: proves that the library's bounded waits end. Runs, each with a
 * limit of limit_ns (1 us .. 2 s):
 *  - the layout's grid barrier on 2 CTAs with a target that can never be
 *    reached: every CTA must give up and set EP_DEVERR_TIMEOUT;
 *  - the capped combine pipeline's mbarrier wait on a phase that never
 *    completes: it must give up, set EP_DEVERR_TIMEOUT and write 1 to
 *    d_words[3].
 * d_words: 4 device uint32 of scratch, owned by the caller. The call
 * synchronises `stream` and returns the error bits in *word. It never traps,
 * and the CUDA context stays usable. (The pages have no counterpart: it checks
 * this implementation's failure detection.) */
ep_status_t ep_selftest_wait_timeout(uint32_t *d_words, uint64_t limit_ns, uint32_t *word, void *stream);

/* Routing + layout that allocates nothing, for callers that cannot get device
 * memory beyond their own inputs and outputs: code under a host framework
 * whose memory planner owns every device byte, or a runtime with a fixed
 * budget that may not call cudaMalloc after start-up. The paper has no
 * counterpart: it is a deployment variant of ep_get_layout.
 *
 * Computes exactly what ep_get_layout computes, with the same inputs and
 * meaning. The outputs go to the caller's device arrays in *out, a host
 * struct of device pointers, every one required, sized for N = R*T as
 * ep_layout_t lists. The layout's scratch lives in a file-scope device array
 * of 2 MiB that every GPU loading the library holds until exit: two barrier
 * counters, plus the per-chunk counts and their prefix sums. The call makes no
 * cudaMalloc, cudaFree or other allocating call.
 *  - Limit: the 2 MiB bound the layout grid (one CTA per chunk) to
 *    (524288 - 64 - (E+R)) / (E+R) CTAs, at most 1024. All 1024 fit at
 *    E = 256, R = 8, and 495 at E = 1024, R = 32. No valid config is
 *    rejected; a smaller grid only means longer chunks.
 *  - d_error_word: a device uint32 that receives EP_DEVERR_* bits with
 *    atomicOr. The caller zeroes and reads it.
 *  - cfg: the layout's shape, as for ep_buffer_workspace_bytes. EP_FLAG_FP8
 *    does not change the layout and is ignored; EP_FLAG_LOW_LATENCY gives the
 *    low-latency dst_row. EP_FLAG_DEDUP and EP_FLAG_SHARD are refused with
 *    EP_ERR_UNSUPPORTED: their extra arrays have no place in ep_layout_t.
 *  - Runs on the current device. `stream` must belong to it.
 *  - Set-up: the first call on each device, and the first call after that
 *    device's context was created anew (after cudaDeviceReset), looks up the
 *    device address of the static scratch (cudaGetSymbolAddress). Make those
 *    calls before any stream capture.
 *  - Every call on a device shares the one scratch array and leaves its
 *    contents behind. Each call first zeroes the barrier counters with a
 *    stream-ordered cudaMemsetAsync of 256 bytes (not an allocation). The
 *    kernel rewrites every other entry it reads. Calls whose GPU work
 *    overlaps (different streams or host threads) race and give wrong
 *    results.
 * Errors: as ep_get_layout, plus EP_ERR_INVALID for a NULL output pointer. */
ep_status_t ep_get_layout_noalloc(const ep_config_t *cfg, int T, const float *d_logits,
                                  const int32_t *d_topk_idx, const float *d_topk_w, int route,
                                  uint64_t mask_seed, float mask_frac, const ep_layout_t *out,
                                  uint32_t *d_error_word, void *stream);

#ifdef __cplusplus
}
#endif
#endif
