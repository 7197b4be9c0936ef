/*
 * CPU oracle for MoE expert-parallel dispatch / combine with group-limited top-k.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * bench's CPU-baseline leg may load this library. The product path (the CUDA
 * library and its Python binding) never calls it and shares no code with it.
 *
 * Plain single-threaded C11. Each function states the definition it writes out.
 * Floating point is IEEE binary64 wherever the method leaves the precision
 * open (routing scores and weights). It is binary32 where the method fixes
 * binary32:
 *  - the FP8 scale arithmetic;
 *  - the top-k weighted combine, accumulated in fp32 with one rounding to bf16.
 *
 * Parity unpinned (conventions, not results; no independent pin exists):
 *  - the group-limited weight normalisation w_k = s_k / sum_j s_j, with no
 *    extra routed scaling factor;
 *  - the amax floor 1e-4 used by the FP8 quantiser for all-zero blocks.
 */
#ifndef COMBINE_TOP_GROUP_ORACLE_H
#define COMBINE_TOP_GROUP_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- number formats ---------------------------------------------------- */
float    orc_bf16_to_f32(uint16_t b);
uint16_t orc_f32_to_bf16(float f);           /* round to nearest even */
uint8_t  orc_e4m3_encode(float v);           /* OCP e4m3fn, RNE, saturate to +-448 */
float    orc_e4m3_decode(uint8_t c);
uint64_t orc_splitmix64(uint64_t counter);   /* first output of SplitMix64 seeded with counter */

/* ---- routing ----------------------------------------------------------- */
/* Softmax top-K. idx [N,K] int32, w [N,K] fp32. renorm != 0 rescales the K
 * selected probabilities to sum 1. */
void orc_route_softmax(const float *logits, int64_t N, int E, int K, int renorm,
                       int32_t *idx, float *w);

/* Group-limited sigmoid gating. margin [N] (may be NULL) receives, per token,
 * the fp64 gap between the last kept group score and the best dropped one
 * (+inf when every group is kept). */
void orc_route_group_sigmoid(const float *logits, int64_t N, int E, int K, int G, int KG,
                             int32_t *idx, float *w, double *margin);

/* Mask slot (g,k) to -1 (weight 0) when the high 32 bits of
 * splitmix64(seed ^ (g*K + k)) are below threshold. */
void orc_apply_mask(int32_t *idx, float *w, int64_t N, int K, uint64_t seed, uint64_t threshold);

/* ---- layout ------------------------------------------------------------ */
/* Returns a bitmask of data errors: bit 0 = expert id outside [-1, E) (the slot
 * is then treated as masked). Output shapes:
 *   is_token_in_rank u8 [N,R], num_tokens_per_rank i32 [R,R], cnt i32 [R,E],
 *   num_tokens_per_expert i32 [E], expert_off i32 [E+1], rank_off i32 [R+1],
 *   src_off i32 [E,R], dst_row i32 [N,K]. */
int orc_layout(const int32_t *idx, int R, int T, int E, int K,
               uint8_t *is_token_in_rank, int32_t *num_tokens_per_rank, int32_t *cnt,
               int32_t *num_tokens_per_expert, int32_t *expert_off, int32_t *rank_off,
               int32_t *src_off, int32_t *dst_row);

/* Low-latency layout: a fixed region of T_max rows per (expert e, source rank
 * s). dst_row[g][k] = (e*R + s)*T_max + j, where j counts source s's earlier
 * slots (in (token, slot) order) that chose e. A slot whose j reaches T_max
 * (only possible with duplicate ids) gets -1, and bit 1 of the return value
 * is set. Bit 0 flags ids outside [-1, E) (treated as masked). */
int orc_layout_ll(const int32_t *idx, int R, int T, int T_max, int E, int K, int32_t *dst_row);

/* ---- deduplicated (per destination rank) receive ------------------------ */
/* Rank-dedup layout (DeepEP overlap notes, §节点内通信: send each token only to
 * the ranks is_token_in_rank marks). Token g goes once to every rank r it has
 * an expert on. Receive rows are ordered by (destination rank r, source rank
 * s, token t). Outputs:
 *   rank_row_off i32 [R+1]      exclusive prefix of the rows per destination rank
 *   rank_src_off i32 [R, R]     [r][s]: offset of source s inside rank r's rows
 *   tok_row      i32 [N, R]     [g][r]: row of token g on rank r, -1 if not sent
 * Returns the number of rows D. */
int64_t orc_layout_dedup(const uint8_t *is_token_in_rank, int R, int T, int32_t *rank_row_off,
                         int32_t *rank_src_off, int32_t *tok_row);

/* Dedup dispatch: row tok_row[g][r] gets token g's hidden vector (bf16 copy,
 * or the same FP8 cast as orc_dispatch), its id, and its top-k localised to
 * rank r: recv_topk_idx[row][k] = idx[g][k] if expert idx[g][k] lives on r,
 * else -1; recv_topk_w likewise (0 where -1). */
void orc_dispatch_dedup(const uint16_t *x, const int32_t *tok_row, const int32_t *topk_idx,
                        const float *topk_w, int64_t N, int R, int E, int H, int K, int fp8,
                        void *recv_x, float *recv_scale, int32_t *recv_src, int32_t *recv_topk_idx,
                        float *recv_topk_w);

/* Local expert permutation on the receiving rank: dedup row d (token g =
 * recv_src[d]) is copied to the expert-grouped row dst_row[g][k] of every slot
 * k with recv_topk_idx[d][k] != -1 (plus its source id and weight). The
 * result equals orc_dispatch's receive buffers. */
void orc_permute(const void *dedup_x, const float *dedup_scale, const int32_t *dedup_src,
                 const int32_t *dedup_topk_idx, const float *dedup_topk_w, int64_t D, const int32_t *dst_row,
                 int H, int K, int fp8, void *recv_x, float *recv_scale, int32_t *recv_src, float *recv_w);

/* Local reduce on the receiving rank: partial[d] = bf16( fma chain over k
 * ascending with recv_topk_idx[d][k] != -1 of w * y[dst_row[g][k]] ) for
 * token g = recv_src[d]. It is the rank's share of the combine, sent back as
 * bf16. y as in orc_combine (bf16, or e4m3 + scales). */
void orc_local_reduce(const void *y, const float *y_scale, const int32_t *dedup_src,
                      const int32_t *dedup_topk_idx, const float *dedup_topk_w, int64_t D,
                      const int32_t *dst_row, int H, int K, uint16_t *partial);

/* Dedup combine: out[g] = bf16( sum over ranks r ascending with tok_row[g][r]
 * != -1 of float(partial[tok_row[g][r]]) ), accumulated in fp32. Tokens not
 * sent anywhere give +0. */
void orc_combine_dedup(const uint16_t *partial, const int32_t *tok_row, int64_t N, int R, int H,
                       uint16_t *out);

/* ---- dispatch ---------------------------------------------------------- */
/* Quantise one bf16 row of H channels (H % 128 == 0) to e4m3 with one fp32
 * scale per 128-channel block. */
void orc_quant_fp8_row(const uint16_t *x, int H, uint8_t *q, float *scale);

/* Full dispatch. fp8 == 0: recv_x is bf16 [M,H]; fp8 != 0: recv_x is e4m3
 * [M,H] and recv_scale fp32 [M,H/128]. recv_src i32 [M], recv_w fp32 [M]. */
void orc_dispatch(const uint16_t *x, const int32_t *dst_row, const float *topk_w,
                  int64_t N, int H, int K, int fp8,
                  void *recv_x, float *recv_scale, int32_t *recv_src, float *recv_w);

/* Identity expert for FP8 receive rows: y = bf16(e4m3_decode(q) * scale). */
void orc_identity_expert_fp8(const uint8_t *q, const float *scale, int64_t M, int H,
                             uint16_t *y);

/* ---- combine ----------------------------------------------------------- */
/* out[g] = bf16( sum_k w[g,k] * y[dst_row[g,k]] ), k ascending, fp32 fma.
 * y_scale == NULL: y is bf16 [M,H]. Otherwise y is e4m3 [M,H] and each value is
 * dequantised as e4m3_decode(q) * y_scale[row, h/128] before the fma.
 * Computes the listed tokens only (tokens == NULL: all N in order); out has one
 * row per computed token. */
void orc_combine(const void *y, const float *y_scale, const int32_t *dst_row,
                 const float *topk_w, int64_t N, int H, int K,
                 const int64_t *tokens, int64_t n_tokens, uint16_t *out);

#ifdef __cplusplus
}
#endif
#endif
