/*
 * CPU oracle: plain, single-threaded definitions of MoE expert-parallel
 * routing, layout, dispatch and combine. TEST INFRASTRUCTURE ONLY: the product
 * path never loads it (header oracle.h has the list of parity-unpinned parts).
 *
 * Sources:
 *  - "DeepEP：年度总结中的计算通信重叠摘记" (DeepEP overlap notes):
 *    - §计算-通信重叠: group-limited gating;
 *    - §节点内通信: is_token_in_rank, only sending to target ranks, FP8 halving
 *      the bytes per element.
 *  - "DeepEP：面向MoE的高吞吐低延迟GPU通信库" (DeepEP summary), §核心亮点 and
 *    §工程化: all-to-all dispatch and combine, FP8.
 * The pages name these steps but do not spell out their arithmetic. The
 * readings used here:
 *  - contiguous expert-to-rank blocks;
 *  - receive rows ordered by (expert, source rank, token, slot);
 *  - e4m3fn with one fp32 scale per 128 channels;
 *  - a k-ascending fp32 fma combine.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared (no fast-math), so
 * every fp32 operation below is one IEEE operation.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32. */
float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary32 to the nearest bf16, ties to even. The two candidates are
 * the truncation t and the next bf16 up. Compare the dropped 16 bits with the
 * halfway point. */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u); /* NaN stays NaN (quiet) */
    uint32_t t = u >> 16;
    uint32_t rest = u & 0xffffu;
    if (rest > 0x8000u || (rest == 0x8000u && (t & 1u)))
        t += 1; /* carries into the exponent correctly, up to infinity */
    return (uint16_t)t;
}

/* OCP 8-bit floating point (OFP8), format E4M3 ("e4m3fn"): 1 sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits. There are no infinities, and
 * S.1111.111 is NaN. The largest finite magnitude is 1.75 * 2^8 = 448. The
 * smallest normal is 2^-6, and the subnormals are m * 2^-9 for m = 1..7. */
float orc_e4m3_decode(uint8_t c)
{
    int sign = c >> 7;
    int e = (c >> 3) & 0xf;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(sign ? -v : v);
}

/* Encode with round-to-nearest-even and saturation to the largest finite value
 * (the "satfinite" rule): every magnitude >= 448, infinity included, becomes
 * 448. Each branch scales |v| exactly by a power of two. It then rounds the
 * scaled value to an integer, ties to even. */
uint8_t orc_e4m3_encode(float vf)
{
    double v = (double)vf;
    uint8_t sign = signbit(vf) ? 0x80 : 0x00;
    if (isnan(vf))
        return (uint8_t)(sign | 0x7f);
    double a = fabs(v);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7e);
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: the grid step is 2^-9; m = 8 is the smallest normal */
        double m = nearbyint(a * 512.0);
        return (uint8_t)(sign | (uint8_t)m);
    }
    int e2;
    double fr = frexp(a, &e2); /* a = fr * 2^e2, fr in [0.5, 1) */
    int e = e2 - 1;            /* a = (2 fr) * 2^e, 2 fr in [1, 2) */
    double m = nearbyint((2.0 * fr - 1.0) * 8.0);
    if (m == 8.0) {
        m = 0.0;
        e += 1;
    }
    int code = ((e + 7) << 3) | (int)m;
    if (code > 0x7e)
        code = 0x7e;
    return (uint8_t)(sign | code);
}

/* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014), used here as a counter-based hash: the first
 * output of the generator whose state starts at `counter`. */
uint64_t orc_splitmix64(uint64_t counter)
{
    uint64_t z = counter + 0x9e3779b97f4a7c15ull;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

/* ------------------------------------------------------------------------ */
/* Routing                                                                   */
/* ------------------------------------------------------------------------ */

/* "a ranks above b" in every top-k: the larger value first, and among equal
 * values the lower index. */
static int ranks_above(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

/* Select the K best entries of row[0..n) among those with allowed[i] != 0,
 * best first, by repeated scans. */
static void select_topk(const float *row, const unsigned char *allowed, int n, int K, int32_t *out)
{
    unsigned char *taken = calloc((size_t)n, 1);
    for (int k = 0; k < K; ++k) {
        int best = -1;
        for (int i = 0; i < n; ++i) {
            if ((allowed && !allowed[i]) || taken[i])
                continue;
            if (best < 0 || ranks_above(row[i], i, row[best], best))
                best = i;
        }
        out[k] = best;
        if (best >= 0)
            taken[best] = 1;
    }
    free(taken);
}

/* Softmax routing: p_e = exp(l_e - max_j l_j) / sum_j exp(l_j - max_j l_j).
 * Softmax is strictly increasing in the logit, so the top-K by probability is
 * the top-K by logit. The oracle selects on the logits, which are exact.
 * The sum runs e = 0..E-1 in fp64. */
void orc_route_softmax(const float *logits, int64_t N, int E, int K, int renorm,
                       int32_t *idx, float *w)
{
    double *p = malloc(sizeof(double) * (size_t)K);
    for (int64_t n = 0; n < N; ++n) {
        const float *row = logits + n * E;
        int32_t *ix = idx + n * K;
        select_topk(row, NULL, E, K, ix);
        double mx = row[0];
        for (int e = 1; e < E; ++e)
            if (row[e] > mx)
                mx = row[e];
        double z = 0.0;
        for (int e = 0; e < E; ++e)
            z += exp((double)row[e] - mx);
        double s = 0.0;
        for (int k = 0; k < K; ++k) {
            p[k] = exp((double)row[ix[k]] - mx) / z;
            s += p[k];
        }
        for (int k = 0; k < K; ++k)
            w[n * K + k] = (float)(renorm ? p[k] / s : p[k]);
    }
    free(p);
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Group-limited gating (DeepEP overlap notes, §计算-通信重叠 names the
 * "group-limited gated" algorithm that DeepEP targets). Read as DeepSeek-V3
 * node-limited routing:
 *  1. s_e = sigmoid(l_e), in fp64.
 *  2. The experts form G groups of E/G contiguous ids. A group's score is the
 *     sum of its two largest s_e.
 *  3. Keep the KG groups with the highest scores (ties: lower group id).
 *  4. Among the experts of the kept groups, take the top K by s_e. sigmoid is
 *     strictly increasing, so this is the top K by logit.
 *  5. w_k = s_k / sum_j s_j over the K chosen, summed in k order.
 */
void orc_route_group_sigmoid(const float *logits, int64_t N, int E, int K, int G, int KG,
                             int32_t *idx, float *w, double *margin)
{
    int gs = E / G;
    double *score = malloc(sizeof(double) * (size_t)G);
    unsigned char *kept = malloc((size_t)G);
    unsigned char *allowed = malloc((size_t)E);
    double *s = malloc(sizeof(double) * (size_t)K);
    for (int64_t n = 0; n < N; ++n) {
        const float *row = logits + n * E;
        for (int g = 0; g < G; ++g) {
            int32_t top2[2];
            select_topk(row + g * gs, NULL, gs, 2, top2);
            score[g] = sigmoid((double)row[g * gs + top2[0]]) + sigmoid((double)row[g * gs + top2[1]]);
        }
        memset(kept, 0, (size_t)G);
        double last_kept = INFINITY;
        for (int j = 0; j < KG; ++j) {
            int best = -1;
            for (int g = 0; g < G; ++g) {
                if (kept[g])
                    continue;
                if (best < 0 || score[g] > score[best])
                    best = g; /* strict: equal scores keep the lower id */
            }
            kept[best] = 1;
            last_kept = score[best];
        }
        double best_dropped = -INFINITY;
        for (int g = 0; g < G; ++g)
            if (!kept[g] && score[g] > best_dropped)
                best_dropped = score[g];
        if (margin)
            margin[n] = (KG < G) ? last_kept - best_dropped : INFINITY;
        for (int e = 0; e < E; ++e)
            allowed[e] = kept[e / gs];
        int32_t *ix = idx + n * K;
        select_topk(row, allowed, E, K, ix);
        double sum = 0.0;
        for (int k = 0; k < K; ++k) {
            s[k] = sigmoid((double)row[ix[k]]);
            sum += s[k];
        }
        for (int k = 0; k < K; ++k)
            w[n * K + k] = (float)(s[k] / sum);
    }
    free(score);
    free(kept);
    free(allowed);
    free(s);
}

void orc_apply_mask(int32_t *idx, float *w, int64_t N, int K, uint64_t seed, uint64_t threshold)
{
    for (int64_t n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            uint64_t h = orc_splitmix64(seed ^ (uint64_t)(n * K + k));
            if ((h >> 32) < threshold) {
                idx[n * K + k] = -1;
                w[n * K + k] = 0.0f;
            }
        }
}

/* ------------------------------------------------------------------------ */
/* Layout                                                                    */
/* ------------------------------------------------------------------------ */

/* Token g = s*T + t belongs to source rank s. Expert e lives on rank e / L,
 * with L = E / R (contiguous blocks). is_token_in_rank (DeepEP overlap notes,
 * §节点内通信) marks the ranks a token must be sent to. Receive rows are
 * ordered by (expert, source rank, token, slot). */
int orc_layout(const int32_t *idx, int R, int T, int E, int K,
               uint8_t *is_token_in_rank, int32_t *num_tokens_per_rank, int32_t *cnt,
               int32_t *num_tokens_per_expert, int32_t *expert_off, int32_t *rank_off,
               int32_t *src_off, int32_t *dst_row)
{
    int err = 0;
    int L = E / R;
    int64_t N = (int64_t)R * T;
    int64_t *run = malloc(sizeof(int64_t) * (size_t)E);

    memset(is_token_in_rank, 0, (size_t)(N * R));
    memset(num_tokens_per_rank, 0, sizeof(int32_t) * (size_t)R * R);
    memset(cnt, 0, sizeof(int32_t) * (size_t)R * E);

    /* which ranks each token goes to, and per-(source rank, expert) counts */
    for (int64_t g = 0; g < N; ++g) {
        int s = (int)(g / T);
        for (int k = 0; k < K; ++k) {
            int e = idx[g * K + k];
            if (e < -1 || e >= E) {
                err |= 1;
                continue;
            }
            if (e == -1)
                continue;
            is_token_in_rank[g * R + e / L] = 1;
            cnt[(int64_t)s * E + e] += 1;
        }
        for (int r = 0; r < R; ++r)
            num_tokens_per_rank[s * R + r] += is_token_in_rank[g * R + r];
    }

    /* per-expert totals and their exclusive prefix sum */
    expert_off[0] = 0;
    for (int e = 0; e < E; ++e) {
        int32_t tot = 0;
        for (int s = 0; s < R; ++s)
            tot += cnt[(int64_t)s * E + e];
        num_tokens_per_expert[e] = tot;
        expert_off[e + 1] = expert_off[e] + tot;
    }
    for (int r = 0; r <= R; ++r)
        rank_off[r] = expert_off[r * L];

    /* offset of source rank s inside expert e's receive block */
    for (int e = 0; e < E; ++e) {
        int32_t acc = 0;
        for (int s = 0; s < R; ++s) {
            src_off[(int64_t)e * R + s] = acc;
            acc += cnt[(int64_t)s * E + e];
        }
    }

    /* placement: a token's copy for expert e goes after every earlier
     * (token, slot) of the same source rank that also chose e */
    for (int s = 0; s < R; ++s) {
        for (int e = 0; e < E; ++e)
            run[e] = 0;
        for (int t = 0; t < T; ++t) {
            int64_t g = (int64_t)s * T + t;
            for (int k = 0; k < K; ++k) {
                int e = idx[g * K + k];
                if (e < 0 || e >= E) {
                    dst_row[g * K + k] = -1;
                    continue;
                }
                dst_row[g * K + k] = (int32_t)(expert_off[e] + src_off[(int64_t)e * R + s] + run[e]);
                run[e] += 1;
            }
        }
    }
    free(run);
    return err;
}

/* Low-latency layout, after the low-latency kernels of the DeepEP pages
 * (DeepEP overlap notes, §计算-通信重叠: the decode-phase mode). Each
 * (expert, source rank) pair owns a fixed region of T_max rows, so a row's
 * place needs no prefix sum across ranks. */
int orc_layout_ll(const int32_t *idx, int R, int T, int T_max, int E, int K, int32_t *dst_row)
{
    int err = 0;
    int64_t *run = malloc(sizeof(int64_t) * (size_t)E);
    for (int s = 0; s < R; ++s) {
        for (int e = 0; e < E; ++e)
            run[e] = 0;
        for (int t = 0; t < T; ++t) {
            int64_t g = (int64_t)s * T + t;
            for (int k = 0; k < K; ++k) {
                int e = idx[g * K + k];
                if (e < -1 || e >= E)
                    err |= 1;
                if (e < 0 || e >= E) {
                    dst_row[g * K + k] = -1;
                    continue;
                }
                if (run[e] >= T_max) {
                    err |= 2;
                    dst_row[g * K + k] = -1;
                    continue;
                }
                dst_row[g * K + k] = (int32_t)(((int64_t)e * R + s) * T_max + run[e]);
                run[e] += 1;
            }
        }
    }
    free(run);
    return err;
}

/* ------------------------------------------------------------------------ */
/* Deduplicated (per destination rank) receive                                */
/* ------------------------------------------------------------------------ */

/* DeepEP overlap notes, §节点内通信: a token goes only to the ranks
 * is_token_in_rank marks, once per rank, however many of that rank's experts
 * it chose. */
int64_t orc_layout_dedup(const uint8_t *is_token_in_rank, int R, int T, int32_t *rank_row_off,
                         int32_t *rank_src_off, int32_t *tok_row)
{
    int64_t N = (int64_t)R * T;
    int64_t *cnt = calloc((size_t)R * R, sizeof(int64_t)); /* [r][s] tokens of s sent to r */
    for (int64_t g = 0; g < N; ++g)
        for (int r = 0; r < R; ++r)
            if (is_token_in_rank[g * R + r])
                cnt[(int64_t)r * R + g / T] += 1;
    int64_t acc = 0;
    for (int r = 0; r < R; ++r) {
        rank_row_off[r] = (int32_t)acc;
        for (int s = 0; s < R; ++s) {
            rank_src_off[r * R + s] = (int32_t)(acc - rank_row_off[r]);
            acc += cnt[(int64_t)r * R + s];
        }
    }
    rank_row_off[R] = (int32_t)acc;
    int64_t *run = calloc((size_t)R, sizeof(int64_t));
    for (int s = 0; s < R; ++s) {
        for (int r = 0; r < R; ++r)
            run[r] = 0;
        for (int t = 0; t < T; ++t) {
            int64_t g = (int64_t)s * T + t;
            for (int r = 0; r < R; ++r) {
                if (!is_token_in_rank[g * R + r]) {
                    tok_row[g * R + r] = -1;
                    continue;
                }
                tok_row[g * R + r] = (int32_t)(rank_row_off[r] + rank_src_off[r * R + s] + run[r]);
                run[r] += 1;
            }
        }
    }
    free(cnt);
    free(run);
    return acc;
}

void orc_dispatch_dedup(const uint16_t *x, const int32_t *tok_row, const int32_t *topk_idx,
                        const float *topk_w, int64_t N, int R, int E, int H, int K, int fp8,
                        void *recv_x, float *recv_scale, int32_t *recv_src, int32_t *recv_topk_idx,
                        float *recv_topk_w)
{
    int L = E / R, nb = H / 128;
    uint8_t *q = fp8 ? malloc((size_t)H) : NULL;
    float *sc = fp8 ? malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1)) : NULL;
    for (int64_t g = 0; g < N; ++g) {
        const uint16_t *xr = x + g * H;
        if (fp8)
            orc_quant_fp8_row(xr, H, q, sc);
        for (int r = 0; r < R; ++r) {
            int64_t row = tok_row[g * R + r];
            if (row < 0)
                continue;
            recv_src[row] = (int32_t)g;
            for (int k = 0; k < K; ++k) {
                int e = topk_idx[g * K + k];
                int here = (e >= 0 && e < E && e / L == r);
                recv_topk_idx[row * K + k] = here ? e : -1;
                recv_topk_w[row * K + k] = here ? topk_w[g * K + k] : 0.0f;
            }
            if (fp8) {
                memcpy((uint8_t *)recv_x + row * H, q, (size_t)H);
                memcpy(recv_scale + row * nb, sc, sizeof(float) * (size_t)nb);
            } else {
                memcpy((uint16_t *)recv_x + row * H, xr, sizeof(uint16_t) * (size_t)H);
            }
        }
    }
    free(q);
    free(sc);
}

void orc_permute(const void *dedup_x, const float *dedup_scale, const int32_t *dedup_src,
                 const int32_t *dedup_topk_idx, const float *dedup_topk_w, int64_t D, const int32_t *dst_row,
                 int H, int K, int fp8, void *recv_x, float *recv_scale, int32_t *recv_src, float *recv_w)
{
    int nb = H / 128;
    for (int64_t d = 0; d < D; ++d) {
        int64_t g = dedup_src[d];
        for (int k = 0; k < K; ++k) {
            if (dedup_topk_idx[d * K + k] < 0)
                continue;
            int64_t row = dst_row[g * K + k];
            if (row < 0)
                continue;
            recv_src[row] = (int32_t)g;
            recv_w[row] = dedup_topk_w[d * K + k];
            if (fp8) {
                memcpy((uint8_t *)recv_x + row * H, (const uint8_t *)dedup_x + d * H, (size_t)H);
                memcpy(recv_scale + row * nb, dedup_scale + d * nb, sizeof(float) * (size_t)nb);
            } else {
                memcpy((uint16_t *)recv_x + row * H, (const uint16_t *)dedup_x + d * H,
                       sizeof(uint16_t) * (size_t)H);
            }
        }
    }
}

void orc_local_reduce(const void *y, const float *y_scale, const int32_t *dedup_src,
                      const int32_t *dedup_topk_idx, const float *dedup_topk_w, int64_t D,
                      const int32_t *dst_row, int H, int K, uint16_t *partial)
{
    int nb = H / 128;
    for (int64_t d = 0; d < D; ++d) {
        int64_t g = dedup_src[d];
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                if (dedup_topk_idx[d * K + k] < 0)
                    continue;
                int64_t row = dst_row[g * K + k];
                if (row < 0)
                    continue;
                float v;
                if (y_scale)
                    v = orc_e4m3_decode(((const uint8_t *)y)[row * H + h]) * y_scale[row * nb + h / 128];
                else
                    v = orc_bf16_to_f32(((const uint16_t *)y)[row * H + h]);
                acc = fmaf(dedup_topk_w[d * K + k], v, acc);
            }
            partial[d * H + h] = orc_f32_to_bf16(acc);
        }
    }
}

void orc_combine_dedup(const uint16_t *partial, const int32_t *tok_row, int64_t N, int R, int H, uint16_t *out)
{
    for (int64_t g = 0; g < N; ++g)
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int r = 0; r < R; ++r) {
                int64_t d = tok_row[g * R + r];
                if (d >= 0)
                    acc += orc_bf16_to_f32(partial[d * H + h]);
            }
            out[g * H + h] = orc_f32_to_bf16(acc);
        }
}

/* ------------------------------------------------------------------------ */
/* Dispatch                                                                  */
/* ------------------------------------------------------------------------ */

/* FP8 cast per 128-channel block (DeepEP overlap notes, §节点内通信: FP8 cuts
 * each element from 2 bytes to 1):
 *   amax  = max(max_h |x_h|, 1e-4)
 *   inv   = 448 / amax              (fp32, IEEE division)
 *   q_h   = e4m3(x_h * inv)         (fp32 product, then RNE, satfinite)
 *   scale = amax / 448              (fp32, IEEE division)
 * A receiver recovers x_h ~= e4m3_decode(q_h) * scale. */
void orc_quant_fp8_row(const uint16_t *x, int H, uint8_t *q, float *scale)
{
    for (int b = 0; b < H / 128; ++b) {
        float amax = 0.0f;
        for (int j = 0; j < 128; ++j) {
            float a = fabsf(orc_bf16_to_f32(x[b * 128 + j]));
            if (a > amax)
                amax = a;
        }
        if (amax < 1e-4f)
            amax = 1e-4f;
        float inv = 448.0f / amax;
        for (int j = 0; j < 128; ++j) {
            float v = orc_bf16_to_f32(x[b * 128 + j]) * inv;
            q[b * 128 + j] = orc_e4m3_encode(v);
        }
        scale[b] = amax / 448.0f;
    }
}

/* Dispatch (DeepEP summary, §工程化: all-to-all dispatch; DeepEP overlap
 * notes, §节点内通信: send only to target ranks). Each unmasked slot (g,k)
 * gets its own receive row dst_row[g,k]. That row holds token g's hidden
 * vector, its source id g and its routing weight. */
void orc_dispatch(const uint16_t *x, const int32_t *dst_row, const float *topk_w,
                  int64_t N, int H, int K, int fp8,
                  void *recv_x, float *recv_scale, int32_t *recv_src, float *recv_w)
{
    int nb = H / 128;
    uint8_t *q = fp8 ? malloc((size_t)H) : NULL;
    float *sc = fp8 ? malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1)) : NULL;
    for (int64_t g = 0; g < N; ++g) {
        const uint16_t *xr = x + g * H;
        if (fp8)
            orc_quant_fp8_row(xr, H, q, sc);
        for (int k = 0; k < K; ++k) {
            int64_t row = dst_row[g * K + k];
            if (row < 0)
                continue;
            recv_src[row] = (int32_t)g;
            recv_w[row] = topk_w[g * K + k];
            if (fp8) {
                memcpy((uint8_t *)recv_x + row * H, q, (size_t)H);
                memcpy(recv_scale + row * nb, sc, sizeof(float) * (size_t)nb);
            } else {
                memcpy((uint16_t *)recv_x + row * H, xr, sizeof(uint16_t) * (size_t)H);
            }
        }
    }
    free(q);
    free(sc);
}

void orc_identity_expert_fp8(const uint8_t *q, const float *scale, int64_t M, int H, uint16_t *y)
{
    int nb = H / 128;
    for (int64_t r = 0; r < M; ++r)
        for (int h = 0; h < H; ++h)
            y[r * H + h] = orc_f32_to_bf16(orc_e4m3_decode(q[r * H + h]) * scale[r * nb + h / 128]);
}

/* ------------------------------------------------------------------------ */
/* Combine                                                                   */
/* ------------------------------------------------------------------------ */

/* Combine (DeepEP summary, §工程化: all-to-all combine): gather the expert
 * outputs of token g's slots back into token order as a top-k weighted sum.
 * Accumulate in fp32, slot by slot in ascending k, with one fused
 * multiply-add per slot. Round once to bf16. A token whose slots are all
 * masked gives +0. */
void orc_combine(const void *y, const float *y_scale, const int32_t *dst_row,
                 const float *topk_w, int64_t N, int H, int K,
                 const int64_t *tokens, int64_t n_tokens, uint16_t *out)
{
    int nb = H / 128;
    int64_t count = tokens ? n_tokens : N;
    for (int64_t i = 0; i < count; ++i) {
        int64_t g = tokens ? tokens[i] : i;
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                int64_t row = dst_row[g * K + k];
                if (row < 0)
                    continue;
                float v;
                if (y_scale)
                    v = orc_e4m3_decode(((const uint8_t *)y)[row * H + h]) * y_scale[row * nb + h / 128];
                else
                    v = orc_bf16_to_f32(((const uint16_t *)y)[row * H + h]);
                acc = fmaf(topk_w[g * K + k], v, acc);
            }
            out[i * H + h] = orc_f32_to_bf16(acc);
        }
    }
}
