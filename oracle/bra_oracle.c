/*
 * Float64 CPU oracle for Bi-Level Routing Attention (BRA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path links,
 * loads or calls this file; only the tests, the smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code with the CUDA path.
 *
 * What it computes follows "BiFormer: Vision Transformer with Bi-Level
 * Routing Attention" (Zhu et al., CVPR 2023) as described on the blog page
 * "BiFormer Reshapes Visual Attention with Bi-Level Routing" (Part 2,
 * section 2.2 "The Overall BRA Flow" and the pseudocode that follows it) and
 * on the paperlayer.ai summary "BiFormer: Vision Transformer with Bi-Level
 * Routing Attention" (section 3 "Our Approach").  The steps are written out
 * plainly, in the pages' order, with no blocking or fusion:
 *
 *   0. linear projection: Q, K, V are the three channel chunks of one
 *      linear layer applied to every token of X (section 2.2 step 2 and
 *      pseudocode step 2; oracle_qkv_projection, used only by the fused
 *      projection path);
 *   1. region partition: the H x W map is cut into S x S regions of
 *      n = (H/S)(W/S) tokens (section 2.2 step 1);
 *   2. region-level query/key Q^r, K^r = per-region mean of Q and K
 *      (section 2.2 step 3, first bullet);
 *   3. region affinity A^r = Q^r (K^r)^T (section 2.2 step 3, second bullet);
 *   4. routing index I^r = row-wise top-k of A^r (section 2.2 step 3, third
 *      bullet);
 *   5. gather the K/V tokens of the k routed regions and run token-to-token
 *      softmax attention over their union (section 2.2 step 4).
 *
 * Readings where the pages are silent:
 *   - heads: C = heads * d, every head is routed and attended on its own
 *     (channels [h*d, (h+1)*d));
 *   - the softmax logits are scaled by 1/sqrt(d); A^r is not scaled;
 *   - region order and token order inside a region are row-major;
 *   - top-k ties go to the lower region index, and each I^r row lists its
 *     regions by (affinity descending, index ascending);
 *   - attention runs over the union of the routed tokens: a caller-given
 *     I^r row that lists a region twice attends to its tokens once;
 *   - the local-context term (section 2.2 step 4, third bullet, and the
 *     "+ dwconv(value)" of pseudocode step 7) is a separate function,
 *     oracle_local_context: a 5x5 depthwise filter over the H x W map with
 *     caller-given weights [C][5][5] and an optional bias [C] (the pages give
 *     neither), stride 1, zero padding 2, applied as a cross-correlation
 *     (the convention of deep-learning convolution layers).
 *
 * Layouts: Q, K, V, O are [B, H, W, C] channels-last float64; Q^r, K^r are
 * [B, heads, R, d]; A^r is [B, heads, R, R]; I^r is [B, heads, R, topk]
 * int32, with R = S*S.  Every function returns 0 on success and a negative
 * value for invalid sizes; it never reads memory it was not given.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_EINVAL (-1)
#define ORACLE_ENOMEM (-2)

static int check_shape(int B, int H, int W, int C, int heads, int S, int topk)
{
    if (B < 0 || H <= 0 || W <= 0 || C <= 0 || heads <= 0 || S <= 0) return ORACLE_EINVAL;
    if (H % S != 0 || W % S != 0 || C % heads != 0) return ORACLE_EINVAL;
    if (topk < 1 || topk > S * S) return ORACLE_EINVAL;
    return 0;
}

/* Linear token index (y, x) of the t-th token of region r, row-major. */
static void region_token(int H, int W, int S, int r, int t, int* y, int* x)
{
    int hs = H / S, ws = W / S;
    int ri = r / S, rj = r % S;
    *y = ri * hs + t / ws;
    *x = rj * ws + t % ws;
    (void)H; (void)W;
}

/* Step 2: per-region mean of one map, per head. */
int oracle_region_pool(const double* x, int B, int H, int W, int C, int heads, int S,
                       double* xr)
{
    if (check_shape(B, H, W, C, heads, S, 1)) return ORACLE_EINVAL;
    int R = S * S, d = C / heads, n = (H / S) * (W / S);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < heads; ++h)
            for (int r = 0; r < R; ++r)
                for (int c = 0; c < d; ++c) {
                    double sum = 0.0;
                    for (int t = 0; t < n; ++t) {
                        int y, xx;
                        region_token(H, W, S, r, t, &y, &xx);
                        sum += x[(((size_t)b * H + y) * W + xx) * C + (size_t)h * d + c];
                    }
                    xr[(((size_t)b * heads + h) * R + r) * d + c] = sum / (double)n;
                }
    return 0;
}

/* Step 3: A^r[r][r'] = <Q^r[r], K^r[r']>, no scaling. */
int oracle_region_affinity(const double* qr, const double* kr, int B, int heads, int R, int d,
                           double* a)
{
    if (B < 0 || heads <= 0 || R <= 0 || d <= 0) return ORACLE_EINVAL;
    for (int bh = 0; bh < B * heads; ++bh)
        for (int r = 0; r < R; ++r)
            for (int s = 0; s < R; ++s) {
                double dot = 0.0;
                for (int c = 0; c < d; ++c)
                    dot += qr[((size_t)bh * R + r) * d + c] * kr[((size_t)bh * R + s) * d + c];
                a[((size_t)bh * R + r) * R + s] = dot;
            }
    return 0;
}

/* Sort key of step 4: larger affinity first, then the lower region index. */
typedef struct { double value; int index; } route_entry;

static int route_cmp(const void* pa, const void* pb)
{
    const route_entry* a = (const route_entry*)pa;
    const route_entry* b = (const route_entry*)pb;
    if (a->value > b->value) return -1;
    if (a->value < b->value) return 1;
    return (a->index > b->index) - (a->index < b->index);
}

/* Step 4: I^r[r] = first topk entries of row r sorted by the key above. */
int oracle_topk_routing(const double* a, int B, int heads, int R, int topk, int32_t* idx)
{
    if (B < 0 || heads <= 0 || R <= 0 || topk < 1 || topk > R) return ORACLE_EINVAL;
    route_entry* row = (route_entry*)malloc(sizeof(route_entry) * (size_t)R);
    if (!row) return ORACLE_ENOMEM;
    for (int bh = 0; bh < B * heads; ++bh)
        for (int r = 0; r < R; ++r) {
            for (int s = 0; s < R; ++s) {
                row[s].value = a[((size_t)bh * R + r) * R + s];
                row[s].index = s;
            }
            qsort(row, (size_t)R, sizeof(route_entry), route_cmp);
            for (int m = 0; m < topk; ++m)
                idx[((size_t)bh * R + r) * topk + m] = row[m].index;
        }
    free(row);
    return 0;
}

/*
 * Step 5: for every query token of region r, attention over the
 * concatenation (in I^r order) of the tokens of its routed regions:
 *   s_j = <q, k_j> / sqrt(d);  w_j = exp(s_j - max s);  o = sum w_j v_j / sum w_j.
 * Two passes, float64.  Routing indices outside [0, R) are an error.
 */
int oracle_token_attention(const double* q, const double* k, const double* v,
                           int B, int H, int W, int C, int heads, int S, int topk,
                           const int32_t* idx, double* o)
{
    if (check_shape(B, H, W, C, heads, S, topk)) return ORACLE_EINVAL;
    int R = S * S, d = C / heads, n = (H / S) * (W / S), kn = topk * n;  /* kn: most keys a query can have */
    double scale = 1.0 / sqrt((double)d);
    double* s = (double*)malloc(sizeof(double) * (size_t)kn);
    size_t* key_off = (size_t*)malloc(sizeof(size_t) * (size_t)kn);
    if (!s || !key_off) { free(s); free(key_off); return ORACLE_ENOMEM; }
    int rc = 0;
    for (int b = 0; b < B && !rc; ++b)
        for (int h = 0; h < heads && !rc; ++h)
            for (int r = 0; r < R && !rc; ++r) {
                const int32_t* route = idx + (((size_t)b * heads + h) * R + r) * topk;
                /* gather: offsets of the routed key/value tokens.  The query
                 * attends over the union of its routed tokens, so a region
                 * listed more than once contributes its tokens once (its
                 * first listing); top-k never lists a region twice. */
                int nkeys = 0;
                for (int m = 0; m < topk; ++m) {
                    int rr = route[m];
                    if (rr < 0 || rr >= R) { rc = ORACLE_EINVAL; break; }
                    int listed_before = 0;
                    for (int mm = 0; mm < m; ++mm) listed_before |= route[mm] == rr;
                    if (listed_before) continue;
                    for (int t = 0; t < n; ++t) {
                        int y, x;
                        region_token(H, W, S, rr, t, &y, &x);
                        key_off[nkeys++] = (((size_t)b * H + y) * W + x) * C + (size_t)h * d;
                    }
                }
                if (rc) break;
                for (int t = 0; t < n; ++t) {
                    int y, x;
                    region_token(H, W, S, r, t, &y, &x);
                    size_t qoff = (((size_t)b * H + y) * W + x) * C + (size_t)h * d;
                    double mx = -INFINITY;
                    for (int j = 0; j < nkeys; ++j) {
                        double dot = 0.0;
                        for (int c = 0; c < d; ++c) dot += q[qoff + c] * k[key_off[j] + c];
                        s[j] = dot * scale;
                        if (s[j] > mx) mx = s[j];
                    }
                    double den = 0.0;
                    for (int j = 0; j < nkeys; ++j) {
                        s[j] = exp(s[j] - mx);
                        den += s[j];
                    }
                    for (int c = 0; c < d; ++c) {
                        double num = 0.0;
                        for (int j = 0; j < nkeys; ++j) num += s[j] * v[key_off[j] + c];
                        o[qoff + c] = num / den;
                    }
                }
            }
    free(s);
    free(key_off);
    return rc;
}

/* All steps in order.  ``a`` may be NULL when the affinities are not wanted. */
int oracle_bra_forward(const double* q, const double* k, const double* v,
                       int B, int H, int W, int C, int heads, int S, int topk,
                       double* o, int32_t* idx, double* a)
{
    int rc = check_shape(B, H, W, C, heads, S, topk);
    if (rc) return rc;
    int R = S * S, d = C / heads;
    size_t nr = (size_t)B * heads * R * d, na = (size_t)B * heads * R * R;
    double* qr = (double*)malloc(sizeof(double) * (nr ? nr : 1));
    double* kr = (double*)malloc(sizeof(double) * (nr ? nr : 1));
    double* aa = a ? a : (double*)malloc(sizeof(double) * (na ? na : 1));
    if (!qr || !kr || !aa) { rc = ORACLE_ENOMEM; goto done; }
    if ((rc = oracle_region_pool(q, B, H, W, C, heads, S, qr))) goto done;
    if ((rc = oracle_region_pool(k, B, H, W, C, heads, S, kr))) goto done;
    if ((rc = oracle_region_affinity(qr, kr, B, heads, R, d, aa))) goto done;
    if ((rc = oracle_topk_routing(aa, B, heads, R, topk, idx))) goto done;
    rc = oracle_token_attention(q, k, v, B, H, W, C, heads, S, topk, idx, o);
done:
    free(qr);
    free(kr);
    if (!a) free(aa);
    return rc;
}

/* Local context enhancement (section 2.2 step 4, third bullet; pseudocode
 * step 7 adds it to the attention output): for every channel c,
 *   out[b, y, x, c] = bias[c] + sum_{i, j = 0..4} w[c][i][j] * v[b, y + i - 2, x + j - 2, c]
 * with v = 0 outside the map.  ``bias`` may be NULL (no bias).  Plain loops,
 * taps in (i, j) row-major order. */
int oracle_local_context(const double* v, int B, int H, int W, int C, const double* w,
                         const double* bias, double* out)
{
    if (B < 0 || H <= 0 || W <= 0 || C <= 0) return ORACLE_EINVAL;
    for (int b = 0; b < B; ++b)
        for (int y = 0; y < H; ++y)
            for (int x = 0; x < W; ++x)
                for (int c = 0; c < C; ++c) {
                    double acc = bias ? bias[c] : 0.0;
                    for (int i = 0; i < 5; ++i) {
                        int yy = y + i - 2;
                        if (yy < 0 || yy >= H) continue;
                        for (int j = 0; j < 5; ++j) {
                            int xx = x + j - 2;
                            if (xx < 0 || xx >= W) continue;
                            acc += w[(size_t)c * 25 + i * 5 + j] *
                                   v[(((size_t)b * H + yy) * W + xx) * C + c];
                        }
                    }
                    out[(((size_t)b * H + y) * W + x) * C + c] = acc;
                }
    return 0;
}

/* Gradients of the token attention for a fixed routing (the backward of the
 * step in section 2.2 step 4; top-k has no gradient, so I^r is an input).
 * With s_j = <q_t, k_j> / sqrt(d), P = softmax(s), o_t = sum_j P_j v_j and an
 * incoming gradient g_t = dL/do_t, the chain rule gives
 *   dP_j = <g_t, v_j>,  D = sum_j P_j dP_j,  dS_j = P_j (dP_j - D),
 *   dq_t += sum_j dS_j k_j / sqrt(d),  dk_j += dS_j q_t / sqrt(d),  dv_j += P_j g_t.
 * The keys of a query are the tokens of its routed regions, a region listed
 * twice counted once (first listing), as the library's attention does.
 * dq, dk, dv are [B, H, W, C] float64, overwritten. */
int oracle_attention_backward(const double* q, const double* k, const double* v,
                              int B, int H, int W, int C, int heads, int S, int topk,
                              const int32_t* idx, const double* g,
                              double* dq, double* dk, double* dv)
{
    if (check_shape(B, H, W, C, heads, S, topk)) return ORACLE_EINVAL;
    int R = S * S, d = C / heads, n = (H / S) * (W / S), kn = topk * n;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);  /* the forward's logit scale */
    size_t total = (size_t)B * H * W * C;
    memset(dq, 0, sizeof(double) * total);
    memset(dk, 0, sizeof(double) * total);
    memset(dv, 0, sizeof(double) * total);
    double* p = (double*)malloc(sizeof(double) * (size_t)kn);
    double* dp = (double*)malloc(sizeof(double) * (size_t)kn);
    size_t* key_off = (size_t*)malloc(sizeof(size_t) * (size_t)kn);
    if (!p || !dp || !key_off) { free(p); free(dp); free(key_off); return ORACLE_ENOMEM; }
    int rc = 0;
    for (int b = 0; b < B && !rc; ++b)
        for (int h = 0; h < heads && !rc; ++h)
            for (int r = 0; r < R && !rc; ++r) {
                const int32_t* route = idx + (((size_t)b * heads + h) * R + r) * topk;
                int nk = 0;  /* keys of the distinct routed regions */
                for (int m = 0; m < topk; ++m) {
                    int region = route[m];
                    if (region < 0 || region >= R) { rc = ORACLE_EINVAL; break; }
                    int seen = 0;
                    for (int mm = 0; mm < m; ++mm) seen |= route[mm] == region;
                    if (seen) continue;
                    for (int t = 0; t < n; ++t) {
                        int y, x;
                        region_token(H, W, S, region, t, &y, &x);
                        key_off[nk++] = (((size_t)b * H + y) * W + x) * C + (size_t)h * d;
                    }
                }
                if (rc) break;
                for (int t = 0; t < n; ++t) {
                    int y, x;
                    region_token(H, W, S, r, t, &y, &x);
                    size_t qoff = (((size_t)b * H + y) * W + x) * C + (size_t)h * d;
                    double mx = -INFINITY;
                    for (int j = 0; j < nk; ++j) {
                        double dot = 0.0;
                        for (int c = 0; c < d; ++c) dot += q[qoff + c] * k[key_off[j] + c];
                        p[j] = dot * inv_sqrt_d;
                        if (p[j] > mx) mx = p[j];
                    }
                    double den = 0.0;
                    for (int j = 0; j < nk; ++j) {
                        p[j] = exp(p[j] - mx);
                        den += p[j];
                    }
                    double dsum = 0.0;
                    for (int j = 0; j < nk; ++j) {
                        p[j] /= den;
                        double dot = 0.0;
                        for (int c = 0; c < d; ++c) dot += g[qoff + c] * v[key_off[j] + c];
                        dp[j] = dot;
                        dsum += p[j] * dot;
                    }
                    for (int j = 0; j < nk; ++j) {
                        double ds = p[j] * (dp[j] - dsum);
                        for (int c = 0; c < d; ++c) {
                            dq[qoff + c] += ds * k[key_off[j] + c] * inv_sqrt_d;
                            dk[key_off[j] + c] += ds * q[qoff + c] * inv_sqrt_d;
                            dv[key_off[j] + c] += p[j] * g[qoff + c];
                        }
                    }
                }
            }
    free(p);
    free(dp);
    free(key_off);
    return rc;
}

/* Linear projection (section 2.2 step 2; pseudocode step 2 splits the
 * output of one linear layer into three equal chunks along the channel axis:
 * query, key, value).  For every token and output channel o in [0, 3C):
 *   y[o] = bias[o] + sum_{c < C} w[o][c] * x[c],
 * and q = y[0, C), k = y[C, 2C), v = y[2C, 3C).  ``w`` is [3C][C] (a linear
 * layer's [out][in] weight), ``bias`` is [3C] or NULL (no bias: the pages do
 * not say whether the layer has one).  x, q, k, v are [B, H, W, C] float64;
 * q, k, v are overwritten. */
int oracle_qkv_projection(const double* x, int B, int H, int W, int C, const double* w,
                          const double* bias, double* q, double* k, double* v)
{
    if (B < 0 || H <= 0 || W <= 0 || C <= 0) return ORACLE_EINVAL;
    size_t tokens = (size_t)B * H * W;
    for (size_t t = 0; t < tokens; ++t) {
        const double* xt = x + t * C;
        for (int o = 0; o < 3 * C; ++o) {
            double acc = bias ? bias[o] : 0.0;
            for (int c = 0; c < C; ++c) acc += w[(size_t)o * C + c] * xt[c];
            double* dst = o < C ? q : (o < 2 * C ? k : v);
            dst[t * C + o % C] = acc;
        }
    }
    return 0;
}
