/*
 * jano_oracle.c -- plain, slow, fp64 CPU oracle for the Jano hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Source of the method: "Jano: Adaptive Diffusion Generation with
 * Early-stage Convergence Awareness" (gist.science summaries of arXiv
 * 2603.00519, nl/fr/pt/zh/ko pages).  Each function names the passage it
 * follows.  The pages give no formulas; the readings used where they are
 * silent are stated at each function and are the same readings the GPU
 * library documents in its header.
 *
 * Every floating-point computation here is fp64 from the caller's fp32 or
 * BF16 inputs; no blocking, fusion or reordering beyond the definitions.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum {
    OR_OK = 0,
    OR_EINVAL = 1,
    OR_ESHAPE = 2,
    OR_ENONFINITE = 5,
    OR_EINDEX = 6,
    OR_ENOMEM = 9
};

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

/*
 * Block-wise complexity score (zh page, technical summary 2.1 "block-wise
 * complexity analyzer"; nl page, Methodologie 1 "Implementatie"; pt page,
 * Metodologia A).  The latent [C][F][H][W] is split into 3D blocks of
 * bf x bh x bw (frame x height x width); per block the score combines the
 * second-order difference of the latent over the warm-up steps with the
 * temporal (inter-frame) and spatial gradient magnitudes:
 *
 *   S_b = mean over k = 1..K-1 and p in P_b of
 *           |x_{k+1}(p) - 2 x_k(p) + x_{k-1}(p)|
 *         + w_t |D_f x_k(p)| + w_s sqrt(D_h x_k(p)^2 + D_w x_k(p)^2)
 *
 * P_b = every channel c and every latent element (f,h,w) inside block b
 * (edge blocks are partial and average over their real elements).
 * D_f, D_h, D_w are forward differences; a difference whose neighbour lies
 * outside the tensor is 0.  The neighbour may belong to the next block.
 * Layout: lat[k][c][f][h][w], w fastest, k = 0..K.
 */
int oracle_block_scores(const float *lat, int K, int C, int F, int H, int W,
                        int bf, int bh, int bw, double w_t, double w_s,
                        double *scores)
{
    if (!lat || !scores || K < 2 || C < 1 || F < 1 || H < 1 || W < 1 ||
        bf < 1 || bh < 1 || bw < 1)
        return OR_EINVAL;
    const int nBf = ceil_div(F, bf), nBh = ceil_div(H, bh), nBw = ceil_div(W, bw);
    const size_t nB = (size_t)nBf * nBh * nBw;
    const size_t plane = (size_t)H * W;
    const size_t vol = (size_t)F * plane;
    const size_t snap = (size_t)C * vol;

    double *sum = (double *)calloc(nB, sizeof(double));
    double *cnt = (double *)calloc(nB, sizeof(double));
    if (!sum || !cnt) { free(sum); free(cnt); return OR_ENOMEM; }

    for (int k = 1; k <= K - 1; ++k) {
        const float *xm = lat + (size_t)(k - 1) * snap;
        const float *x0 = lat + (size_t)k * snap;
        const float *xp = lat + (size_t)(k + 1) * snap;
        for (int c = 0; c < C; ++c) {
            for (int f = 0; f < F; ++f) {
                for (int h = 0; h < H; ++h) {
                    for (int w = 0; w < W; ++w) {
                        const size_t p = (size_t)c * vol + (size_t)f * plane + (size_t)h * W + w;
                        const double a = (double)x0[p];
                        const double d2 = (double)xp[p] - 2.0 * a + (double)xm[p];
                        const double df = (f + 1 < F) ? (double)x0[p + plane] - a : 0.0;
                        const double dh = (h + 1 < H) ? (double)x0[p + W] - a : 0.0;
                        const double dw = (w + 1 < W) ? (double)x0[p + 1] - a : 0.0;
                        const double term = fabs(d2) + w_t * fabs(df) + w_s * sqrt(dh * dh + dw * dw);
                        const size_t b = ((size_t)(f / bf) * nBh + (size_t)(h / bh)) * nBw + (size_t)(w / bw);
                        sum[b] += term;
                        cnt[b] += 1.0;
                    }
                }
            }
        }
    }
    for (size_t b = 0; b < nB; ++b)
        scores[b] = sum[b] / cnt[b];
    free(sum);
    free(cnt);
    return OR_OK;
}

/*
 * Three convergence levels (nl page, Methodologie 1 "Resultaat": Level 1
 * Static, Level 2 Moderate, Level 3 Active; zh page 2.2 item 1).  The pages
 * give no thresholds; the split is by quantile over blocks: order blocks by
 * the key (score ascending, block index ascending), the first n_S are
 * Static, the last n_A are Active, the rest Moderate, with
 *   n_X = floor(bp_X * B / 10000),  bp_X = round(frac_X * 10000)
 * in integer arithmetic.  Negative zero ranks as zero; a non-finite score
 * is an error.  The sort is a library routine (qsort).
 */
typedef struct { double s; int i; } or_key;

static int or_key_cmp(const void *pa, const void *pb)
{
    const or_key *a = (const or_key *)pa, *b = (const or_key *)pb;
    if (a->s < b->s) return -1;
    if (a->s > b->s) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

int oracle_level_counts(int B, float frac_active, float frac_static,
                        long long *n_active, long long *n_static)
{
    if (B < 1 || !(frac_active >= 0.0f && frac_active <= 1.0f) ||
        !(frac_static >= 0.0f && frac_static <= 1.0f))
        return OR_EINVAL;
    const long long bpA = llround((double)frac_active * 10000.0);
    const long long bpS = llround((double)frac_static * 10000.0);
    if (bpA + bpS > 10000) return OR_EINVAL;
    *n_active = bpA * (long long)B / 10000;
    *n_static = bpS * (long long)B / 10000;
    return OR_OK;
}

int oracle_classify(const float *scores, int B, float frac_active,
                    float frac_static, uint8_t *levels)
{
    if (!scores || !levels) return OR_EINVAL;
    long long nA, nS;
    int st = oracle_level_counts(B, frac_active, frac_static, &nA, &nS);
    if (st) return st;
    for (int i = 0; i < B; ++i)
        if (!isfinite(scores[i])) return OR_ENONFINITE;
    or_key *keys = (or_key *)malloc((size_t)B * sizeof(or_key));
    if (!keys) return OR_ENOMEM;
    for (int i = 0; i < B; ++i) {
        keys[i].s = (double)scores[i];   /* -0.0 == +0.0 under < and > */
        keys[i].i = i;
    }
    qsort(keys, (size_t)B, sizeof(or_key), or_key_cmp);
    for (long long r = 0; r < B; ++r) {
        uint8_t lv = 2;
        if (r < nS) lv = 1;
        else if (r >= (long long)B - nA) lv = 3;
        levels[keys[r].i] = lv;
    }
    free(keys);
    return OR_OK;
}

/*
 * Block -> token level map, then the interleaved schedule (nl page,
 * Methodologie 2: warm-up, interleaved generation with Level 1 rarely,
 * Level 2 intermittently, Level 3 every step, cool-down; zh page 2.2
 * item 2; fr page 2.B "Pipeline Intercalé").
 *
 * A token is a pf x ph x pw patch; token id t = (ft*TH + th)*TW + tw.  It
 * takes the level of the block holding its first latent element
 * (ft*pf, th*ph, tw*pw).  Step s (0..T-1) is full when s < warmup or
 * s >= T - cooldown.  Otherwise, with j = s - warmup, Level 3 is due,
 * Level 2 is due when (j+1) % period_moderate == 0 and Level 1 when
 * (j+1) % period_static == 0.  idx holds, step after step, the due tokens
 * in ascending id; offsets[s]..offsets[s+1] delimit step s.
 */
int oracle_build_schedule(const uint8_t *block_levels, int F, int H, int W,
                          int bf, int bh, int bw, int pf, int ph, int pw,
                          int T, int warmup, int cooldown, int pM, int pS,
                          int32_t *offsets, int32_t *idx, long long idx_cap,
                          uint8_t *token_levels)
{
    if (!block_levels || !offsets || !idx || F < 1 || H < 1 || W < 1 ||
        bf < 1 || bh < 1 || bw < 1 || pf < 1 || ph < 1 || pw < 1)
        return OR_EINVAL;
    if (F % pf || H % ph || W % pw) return OR_ESHAPE;
    if (T < 1 || warmup < 0 || cooldown < 0 || warmup + cooldown > T || pM < 1 || pS < 1)
        return OR_EINVAL;
    const int TF = F / pf, TH = H / ph, TW = W / pw;
    const long long NT = (long long)TF * TH * TW;
    if (idx_cap < NT * T) return OR_EINVAL;
    const int nBh = ceil_div(H, bh), nBw = ceil_div(W, bw);

    uint8_t *tl = token_levels ? token_levels : (uint8_t *)malloc((size_t)NT);
    if (!tl) return OR_ENOMEM;
    for (int ft = 0; ft < TF; ++ft)
        for (int th = 0; th < TH; ++th)
            for (int tw = 0; tw < TW; ++tw) {
                const int f = ft * pf, h = th * ph, w = tw * pw;
                const long long b = ((long long)(f / bf) * nBh + h / bh) * nBw + w / bw;
                const long long t = ((long long)ft * TH + th) * TW + tw;
                const uint8_t lv = block_levels[b];
                if (lv < 1 || lv > 3) {
                    if (!token_levels) free(tl);
                    return OR_EINVAL;
                }
                tl[t] = lv;
            }

    long long n = 0;
    offsets[0] = 0;
    for (int s = 0; s < T; ++s) {
        const int full = (s < warmup) || (s >= T - cooldown);
        const int j = s - warmup;
        const int due2 = full || ((j + 1) % pM == 0);
        const int due1 = full || ((j + 1) % pS == 0);
        for (long long t = 0; t < NT; ++t) {
            const uint8_t lv = tl[t];
            if (lv == 3 || (lv == 2 && due2) || (lv == 1 && due1))
                idx[n++] = (int32_t)t;
        }
        offsets[s + 1] = (int32_t)n;
    }
    if (!token_levels) free(tl);
    return OR_OK;
}

/*
 * KV-cache update (nl page, Methodologie 2 "KV Cache Mechanisme": the K/V
 * of frozen tokens are kept; zh page 2.2 item 3).  The cache keeps the
 * latest K/V row of every token in token order; the fresh rows of the due
 * tokens overwrite theirs: Kc[idx[i]] = K_act[i], Vc[idx[i]] = V_act[i].
 * Rows are row_elems BF16 values (heads * d), copied bit for bit.
 */
int oracle_kv_scatter(const uint16_t *k_act, const uint16_t *v_act,
                      const int32_t *idx, int n_act, int row_elems,
                      uint16_t *k_cache, uint16_t *v_cache, int n_tokens)
{
    if (n_act < 0 || row_elems < 1 || n_tokens < 1) return OR_EINVAL;
    for (int i = 0; i < n_act; ++i) {
        const int32_t t = idx[i];
        if (t < 0 || t >= n_tokens) return OR_EINDEX;
        for (int e = 0; e < row_elems; ++e) {
            k_cache[(size_t)t * row_elems + e] = k_act[(size_t)i * row_elems + e];
            v_cache[(size_t)t * row_elems + e] = v_act[(size_t)i * row_elems + e];
        }
    }
    return OR_OK;
}

static double bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Active-query attention over the whole cached K/V (nl page, Methodologie 2
 * "KV Cache Mechanisme": cached K/V are concatenated with the active
 * queries; attention is invariant to the order of keys/values; pt page
 * 2.B "Gerenciamento de KV Cache").  With the cache kept in token order:
 *
 *   O[idx[i], h, :] = sum_j softmax_j(scale * q_i,h . k_j,h) v_j,h
 *
 * over all N cached tokens j, no mask, no bias.  Inputs are BF16 bit
 * patterns decoded exactly to fp64; the row max, exp, sum and division are
 * fp64.  Only the requested active rows rows[0..n_rows) are computed;
 * out_rows is [n_rows][heads][d] fp64 (row r holds active row rows[r],
 * which the library writes to token idx[rows[r]]).
 */
int oracle_active_attention(const uint16_t *q_act, const uint16_t *k_cache,
                            const uint16_t *v_cache, int n_act, int n_tokens,
                            int heads, int d, double scale,
                            const int32_t *rows, int n_rows, double *out_rows)
{
    if (n_act < 0 || n_tokens < 1 || heads < 1 || d < 1 || n_rows < 0) return OR_EINVAL;
    double *s = (double *)malloc((size_t)n_tokens * sizeof(double));
    if (!s) return OR_ENOMEM;
    const size_t rs = (size_t)heads * d;
    for (int r = 0; r < n_rows; ++r) {
        const int i = rows[r];
        if (i < 0 || i >= n_act) { free(s); return OR_EINDEX; }
        for (int h = 0; h < heads; ++h) {
            const uint16_t *q = q_act + (size_t)i * rs + (size_t)h * d;
            double m = -INFINITY;
            for (int j = 0; j < n_tokens; ++j) {
                const uint16_t *k = k_cache + (size_t)j * rs + (size_t)h * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c)
                    dot += bf16_value(q[c]) * bf16_value(k[c]);
                s[j] = scale * dot;
                if (s[j] > m) m = s[j];
            }
            double z = 0.0;
            for (int j = 0; j < n_tokens; ++j) {
                s[j] = exp(s[j] - m);
                z += s[j];
            }
            double *o = out_rows + ((size_t)r * heads + h) * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int j = 0; j < n_tokens; ++j) {
                const uint16_t *v = v_cache + (size_t)j * rs + (size_t)h * d;
                for (int c = 0; c < d; ++c)
                    o[c] += s[j] * bf16_value(v[c]);
            }
            for (int c = 0; c < d; ++c) o[c] /= z;
        }
    }
    free(s);
    return OR_OK;
}

/*
 * Projections of the active tokens only (nl page, Methodologie 2 "KV Cache
 * Mechanisme": per step JANO activates only a subset of the tokens and
 * stores the K/V of the frozen ones, so the DiT block's linear maps run on
 * the active rows alone; zh page 2.2 item 3).  A linear map y = x W^T on the
 * rows of x picked by `gather` (row r reads x[gather[r]]; gather == NULL
 * reads x[r]):
 *
 *   out[r][j] = sum_c x[src(r)][c] * w[j][c],   r < m, j < n
 *
 * x is [n_x][k] and w [n][k] BF16 bit patterns (w in the usual [out][in]
 * layout of a linear layer), decoded exactly; the sums are fp64 in c order.
 * out is [m][n] fp64.  Where the rows land (a token-ordered buffer, the K/V
 * cache) is placement only and is checked separately by the tests.
 */
int oracle_gather_gemm(const uint16_t *x, int n_x, const int32_t *gather, int m,
                       const uint16_t *w, int n, int k, double *out)
{
    if (!x || !w || !out || n_x < 1 || m < 0 || n < 1 || k < 1) return OR_EINVAL;
    for (int r = 0; r < m; ++r) {
        const int src = gather ? gather[r] : r;
        if (src < 0 || src >= n_x) return OR_EINDEX;
        const uint16_t *xr = x + (size_t)src * k;
        for (int j = 0; j < n; ++j) {
            const uint16_t *wj = w + (size_t)j * k;
            double acc = 0.0;
            for (int c = 0; c < k; ++c)
                acc += bf16_value(xr[c]) * bf16_value(wj[c]);
            out[(size_t)r * n + j] = acc;
        }
    }
    return OR_OK;
}

/*
 * Random-masking ablation (ko page, section 4 "Ablation Study": random
 * masking at a similar speed-up gives clearly worse quality than Jano's
 * convergence-aware levels).  The ablation keeps Jano's level counts but
 * assigns the levels at random: block b gets the uniform score
 *
 *   u_b = (splitmix64 output number b+1 of the stream seeded with `seed`) >> 40, times 2^-24
 *
 * and the scores are classified exactly like the analyzer's (same counts,
 * ties by block index).  splitmix64 (Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", 2014): the state advances by the golden
 * gamma 0x9E3779B97F4A7C15 and each output is the state passed through the
 * 64-bit finaliser (xor-shift 30, multiply 0xBF58476D1CE4E5B9, xor-shift 27,
 * multiply 0x94D049BB133111EB, xor-shift 31).  Output number i (from 1) is
 * therefore a function of seed + i * gamma alone.
 */
void oracle_splitmix64(uint64_t seed, int n, uint64_t *out)
{
    uint64_t state = seed;
    for (int i = 0; i < n; ++i) {
        state += 0x9E3779B97F4A7C15ull;
        uint64_t z = state;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        out[i] = z ^ (z >> 31);
    }
}

int oracle_random_scores(int n, uint64_t seed, float *scores)
{
    if (n < 1 || !scores) return OR_EINVAL;
    uint64_t *r = (uint64_t *)malloc((size_t)n * sizeof(uint64_t));
    if (!r) return OR_ENOMEM;
    oracle_splitmix64(seed, n, r);
    for (int b = 0; b < n; ++b)
        scores[b] = (float)((double)(r[b] >> 40) / 16777216.0);   /* exact: 24-bit integer / 2^24 */
    free(r);
    return OR_OK;
}

/*
 * The literal reading of the score (nl page, Methodologie 1
 * "Implementatie": the analyzer computes the second-order differences of
 * the temporal and spatial gradients over the first steps).  Per element p
 * and step k = 1..K-1, with the forward gradients of snapshot j
 *
 *   G_f(j) = D_f x_j(p),  G_h(j) = D_h x_j(p),  G_w(j) = D_w x_j(p)
 *
 * (0 where the neighbour lies outside the tensor) and their second
 * difference over the steps, Delta2 G(k) = G(k+1) - 2 G(k) + G(k-1):
 *
 *   S_b = mean over k and p in P_b of
 *           w_t |Delta2 G_f(k)| + w_s sqrt(Delta2 G_h(k)^2 + Delta2 G_w(k)^2)
 *
 * Computed in that order (the gradients of the three snapshots first, then
 * their second difference), fp64.  Same blocks, layout and edge rules as
 * oracle_block_scores.
 */
static double or_grad(const float *x, size_t p, int on, size_t step)
{
    return on ? (double)x[p + step] - (double)x[p] : 0.0;
}

int oracle_block_scores_literal(const float *lat, int K, int C, int F, int H, int W,
                                int bf, int bh, int bw, double w_t, double w_s,
                                double *scores)
{
    if (!lat || !scores || K < 2 || C < 1 || F < 1 || H < 1 || W < 1 ||
        bf < 1 || bh < 1 || bw < 1)
        return OR_EINVAL;
    const int nBf = ceil_div(F, bf), nBh = ceil_div(H, bh), nBw = ceil_div(W, bw);
    const size_t nB = (size_t)nBf * nBh * nBw;
    const size_t plane = (size_t)H * W;
    const size_t vol = (size_t)F * plane;
    const size_t snap = (size_t)C * vol;

    double *sum = (double *)calloc(nB, sizeof(double));
    double *cnt = (double *)calloc(nB, sizeof(double));
    if (!sum || !cnt) { free(sum); free(cnt); return OR_ENOMEM; }

    for (int k = 1; k <= K - 1; ++k) {
        const float *xs[3] = {lat + (size_t)(k - 1) * snap, lat + (size_t)k * snap,
                              lat + (size_t)(k + 1) * snap};
        for (int c = 0; c < C; ++c)
            for (int f = 0; f < F; ++f)
                for (int h = 0; h < H; ++h)
                    for (int w = 0; w < W; ++w) {
                        const size_t p = (size_t)c * vol + (size_t)f * plane + (size_t)h * W + w;
                        double gf[3], gh[3], gw[3];
                        for (int j = 0; j < 3; ++j) {
                            gf[j] = or_grad(xs[j], p, f + 1 < F, plane);
                            gh[j] = or_grad(xs[j], p, h + 1 < H, (size_t)W);
                            gw[j] = or_grad(xs[j], p, w + 1 < W, 1);
                        }
                        const double d2f = gf[2] - 2.0 * gf[1] + gf[0];
                        const double d2h = gh[2] - 2.0 * gh[1] + gh[0];
                        const double d2w = gw[2] - 2.0 * gw[1] + gw[0];
                        const double term = w_t * fabs(d2f) + w_s * sqrt(d2h * d2h + d2w * d2w);
                        const size_t b = ((size_t)(f / bf) * nBh + (size_t)(h / bh)) * nBw + (size_t)(w / bw);
                        sum[b] += term;
                        cnt[b] += 1.0;
                    }
    }
    for (size_t b = 0; b < nB; ++b)
        scores[b] = sum[b] / cnt[b];
    free(sum);
    free(cnt);
    return OR_OK;
}

/*
 * Frequency-domain block complexity, the FFT baseline the analyzer is
 * compared with (zh page, technical summary 1 and 2.1: an FFT taken on the
 * early latent predicts convergence poorly; fr page 2.A).  The pages give
 * no formula; the reading is the energy of the high band of each block's
 * 3-D discrete Fourier transform, on one snapshot x[c][f][h][w]:
 *
 *   X_{c,b}(u) = sum over the block's own elements (f, h, w) of
 *                x[c][f0+f][h0+h][w0+w] exp(-2 pi i (u_f f/m_f + u_h h/m_h + u_w w/m_w))
 *   S_b = 1/C sum_c 1/n_b^2 sum_{u : max_a min(u_a, m_a - u_a) >= cutoff} |X_{c,b}(u)|^2
 *
 * m_a the block's extent along axis a inside the tensor (edge blocks are
 * smaller), n_b = m_f m_h m_w.  The DFT is taken by this definition, one
 * frequency at a time, in fp64 with the C library's cos and sin.
 */
static int or_fold(int u, int m) { return u < m - u ? u : m - u; }

int oracle_fft_scores(const float *x, int C, int F, int H, int W, int bf, int bh, int bw,
                      int cutoff, double *scores)
{
    if (!x || !scores || C < 1 || F < 1 || H < 1 || W < 1 || bf < 1 || bh < 1 || bw < 1 ||
        cutoff < 0)
        return OR_EINVAL;
    const int nBf = ceil_div(F, bf), nBh = ceil_div(H, bh), nBw = ceil_div(W, bw);
    const size_t plane = (size_t)H * W;
    const size_t vol = (size_t)F * plane;
    const double two_pi = 2.0 * acos(-1.0);
    for (int fb = 0; fb < nBf; ++fb)
        for (int hb = 0; hb < nBh; ++hb)
            for (int wb = 0; wb < nBw; ++wb) {
                const int f0 = fb * bf, h0 = hb * bh, w0 = wb * bw;
                const int mf = F - f0 < bf ? F - f0 : bf;
                const int mh = H - h0 < bh ? H - h0 : bh;
                const int mw = W - w0 < bw ? W - w0 : bw;
                const double n = (double)mf * mh * mw;
                double total = 0.0;
                for (int c = 0; c < C; ++c) {
                    double e = 0.0;
                    for (int uf = 0; uf < mf; ++uf)
                        for (int uh = 0; uh < mh; ++uh)
                            for (int uw = 0; uw < mw; ++uw) {
                                int k = or_fold(uf, mf);
                                if (or_fold(uh, mh) > k) k = or_fold(uh, mh);
                                if (or_fold(uw, mw) > k) k = or_fold(uw, mw);
                                if (k < cutoff) continue;
                                double re = 0.0, im = 0.0;
                                for (int f = 0; f < mf; ++f)
                                    for (int h = 0; h < mh; ++h)
                                        for (int w = 0; w < mw; ++w) {
                                            const double v = x[(size_t)c * vol + (size_t)(f0 + f) * plane +
                                                               (size_t)(h0 + h) * W + (w0 + w)];
                                            const double ph = two_pi * ((double)uf * f / mf +
                                                                        (double)uh * h / mh +
                                                                        (double)uw * w / mw);
                                            re += v * cos(ph);
                                            im -= v * sin(ph);
                                        }
                                e += re * re + im * im;
                            }
                    total += e / (n * n);
                }
                scores[((size_t)fb * nBh + hb) * nBw + wb] = total / C;
            }
    return OR_OK;
}
