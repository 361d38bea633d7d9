/*
 * jano.h -- C ABI of libjano, the B200 (sm_100a) library for the
 * data-parallel hot path of Jano ("Jano: Adaptive Diffusion Generation with
 * Early-stage Convergence Awareness", arXiv 2603.00519, as summarised on the
 * gist.science pages in nl/fr/pt/zh/ko).
 *
 * The hot path has two parts:
 *   1. the block-wise complexity analyzer and its three-level split
 *      (jano_block_scores, jano_classify) plus the interleaved token schedule
 *      built from it (jano_build_schedule);
 *   2. the per-step partial-token attention: fresh K/V of the due tokens are
 *      scattered into a persistent full-sequence cache (jano_kv_scatter) and
 *      only the due (active) queries attend over the whole cache
 *      (jano_active_attention, or jano_active_attention_split for due sets
 *      too small to fill the GPU), their outputs going back to their token
 *      rows.
 *
 * Conventions shared by every entry point
 *   - All pointers named *device* below are device pointers on the current
 *     CUDA device; `stream` is a cudaStream_t passed as void* (NULL = the
 *     legacy default stream).  Every launch is asynchronous on `stream`.
 *   - The caller owns every buffer.  The library allocates no device or host
 *     memory; scratch space, where an entry point needs some, is passed in by
 *     the caller and sized by a *_workspace_bytes query.
 *   - Argument errors are detected on the host before anything is launched
 *     and returned synchronously; nothing is written in that case.  A failed
 *     launch returns JANO_ECUDA.  Errors that only the device can see (an
 *     index out of range, a non-finite score, an invalid level) set a sticky
 *     per-device error word that jano_get_device_error() reads and clears.
 *     Kernels never trap: an offending element is skipped, and every wait
 *     inside a kernel is bounded in time.
 *   - Layouts are dense and row-major, the last index fastest.
 *   - Token order: a token is a pf x ph x pw patch of the latent, and token
 *     id t = (ft*TH + th)*TW + tw with TF=F/pf, TH=H/ph, TW=W/pw.  Q/K/V/O
 *     rows are [tokens][heads][d] BF16, one contiguous row of heads*d values
 *     per token; the KV cache is kept in token order.
 */
#ifndef JANO_H
#define JANO_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define JANO_API __attribute__((visibility("default")))
#else
#define JANO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    JANO_OK = 0,
    JANO_EINVAL = 1,        /* bad argument value or NULL pointer            */
    JANO_ESHAPE = 2,        /* inconsistent sizes (e.g. F not divisible by pf) */
    JANO_EALIGN = 3,        /* pointer not 16-byte aligned                    */
    JANO_EUNSUPPORTED = 4,  /* valid but not implemented (e.g. d not 64/128)  */
    JANO_ENONFINITE = 5,    /* device: a score was NaN or infinite            */
    JANO_EINDEX = 6,        /* device: an index or level out of range, or an
                               index list not strictly ascending             */
    JANO_ETIMEOUT = 7,      /* device: a bounded internal wait gave up (a bug) */
    JANO_ECUDA = 8          /* a CUDA runtime call or launch failed           */
} jano_status;

/* Latent geometry: latent dims (F frames, H rows, W columns), analyzer block
 * dims (bf, bh, bw) and token patch dims (pf, ph, pw), all in latent
 * elements.  Blocks at the far edges may be partial; F, H, W must be
 * multiples of pf, ph, pw. */
typedef struct {
    int F, H, W;
    int bf, bh, bw;
    int pf, ph, pw;
} jano_geom;

/* Interleaved schedule: T sampling steps; the first `warmup` and the last
 * `cooldown` are full steps; in between, Moderate tokens refresh every
 * `period_moderate` steps and Static tokens every `period_static` steps. */
typedef struct {
    int T, warmup, cooldown, period_moderate, period_static;
} jano_sched_cfg;

/* ------------------------------------------------------------------------
 * jano_block_scores -- block-wise complexity score.
 * Pages: zh technical summary 2.1 (3D frame x height x width blocks;
 * temporal and spatial gradients; second-order differences over the first K
 * steps, about 10% of sampling, combined into a per-block score); nl
 * technical summary, Methodologie 1 "Implementatie"; pt 2.A.
 *
 *   S_b = mean over k=1..K-1 and every (c,f,h,w) in block b of
 *         |x_{k+1} - 2 x_k + x_{k-1}| + w_temporal |D_f x_k|
 *                                     + w_spatial sqrt(D_h x_k^2 + D_w x_k^2)
 *
 * D_* are forward differences, 0 where the neighbour is outside the tensor
 * (it may lie in the next block); edge blocks average over their real
 * elements.  The usual weights are 0.5 and 0.5.
 *
 * lat     device fp32 [K+1][C][F][H][W], 16-byte aligned; W % 4 == 0.
 * K       index of the last snapshot (K+1 snapshots); K >= 2.
 * scores  device fp32 [nBf*nBh*nBw], nBx = ceil(X/bx), block id
 *         (bf_i*nBh + bh_i)*nBw + bw_i.  Deterministic (fixed reduction
 *         order, no atomics).
 * Patch dims in `g` are not used here.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_block_scores(const float *lat, int K, int C, const jano_geom *g,
                              float w_temporal, float w_spatial, float *scores,
                              void *stream);

/* ------------------------------------------------------------------------
 * jano_block_scores_literal -- the literal reading of the score: the
 * second-order differences over the steps of the temporal and spatial
 * gradients (nl technical summary, Methodologie 1 "Implementatie").
 *
 *   S_b = mean over k=1..K-1 and every (c,f,h,w) in block b of
 *         w_temporal |D2 D_f x_k| + w_spatial sqrt((D2 D_h x_k)^2 + (D2 D_w x_k)^2)
 *   D2 y_k = y_{k+1} - 2 y_k + y_{k-1}
 *
 * with the forward differences and edge rules of jano_block_scores.  It
 * differs from jano_block_scores (which adds |D2 x| to first-order
 * gradients) only in the formula; arguments, layout, limits and errors are
 * the same.  Deterministic.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_block_scores_literal(const float *lat, int K, int C, const jano_geom *g,
                                               float w_temporal, float w_spatial, float *scores,
                                               void *stream);

/* ------------------------------------------------------------------------
 * jano_classify -- three convergence levels (Level 1 Static, 2 Moderate,
 * 3 Active).  Pages: nl technical summary, Methodologie 1 "Resultaat";
 * zh 2.2 item 1; ko 2.B.
 *
 * Blocks are ordered by the key (score ascending, block index ascending;
 * -0 ranks as +0).  With bp_X = round(frac_X * 10000) and
 * n_X = floor(bp_X * n_blocks / 10000), the first n_S blocks are Static,
 * the last n_A Active, the rest Moderate.  frac_active + frac_static <= 1.
 *
 * scores  device fp32 [n_blocks] (any finite values).
 * levels  device uint8 [n_blocks], written with 1, 2 or 3.
 * A NaN or infinite score raises JANO_ENONFINITE on the device error word
 * and leaves `levels` unspecified.  One thread-block cluster (16 blocks
 * where the device runs clusters of that size, else 8); no scratch memory.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_classify(const float *scores, int n_blocks, float frac_active,
                          float frac_static, uint8_t *levels, void *stream);

/* ------------------------------------------------------------------------
 * jano_build_schedule -- block levels -> token levels -> per-step lists of
 * due tokens for all T steps (CSR).  Pages: nl technical summary,
 * Methodologie 2 (warm-up; Level 1 rarely, Level 2 intermittently, Level 3
 * every step; cool-down); zh 2.2 item 2; fr 2.B "Pipeline Intercalé".
 *
 * A token takes the level of the block holding its first latent element.
 * Step s is full when s < warmup or s >= T - cooldown; otherwise, with
 * j = s - warmup, Level 3 is due, Level 2 when (j+1) % period_moderate == 0
 * and Level 1 when (j+1) % period_static == 0.
 *
 * block_levels  device uint8 [n_blocks] (values 1..3; others raise EINDEX
 *               on the device error word and count as Static).
 * offsets       device int32 [T+1]: step s lists idx[offsets[s]..offsets[s+1]).
 * idx           device int32, capacity idx_capacity >= T * n_tokens; the due
 *               token ids of each step in ascending order.
 * token_levels  device uint8 [n_tokens] or NULL.
 * workspace     device scratch of jano_build_schedule_workspace_bytes(g)
 *               bytes, 16-byte aligned; its contents need not be initialised
 *               and are meaningless afterwards.
 * ---------------------------------------------------------------------- */
JANO_API size_t jano_build_schedule_workspace_bytes(const jano_geom *g);
JANO_API jano_status jano_build_schedule(const uint8_t *block_levels, const jano_geom *g,
                                const jano_sched_cfg *c, int32_t *offsets,
                                int32_t *idx, size_t idx_capacity,
                                uint8_t *token_levels, void *workspace,
                                size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * jano_build_schedule_noalloc -- jano_build_schedule for callers that cannot
 * allocate device memory.  The Jano pages have no counterpart: this is a
 * deployment convenience, not part of the method.
 *
 * Some callers cannot call cudaMalloc or any allocating routine where they
 * build the schedule: plug-ins handed fixed buffers by a host framework,
 * runtimes without a device allocator, hosts whose memory pool is owned by
 * another framework and forbids side allocations.  This variant takes the same inputs and outputs
 * as jano_build_schedule but no workspace: its scratch is a file-scope
 * __device__ array of 1 MiB inside the library, which every GPU that loads
 * the library holds until the process exits.  It allocates nothing.
 *
 * Limit: the scratch the geometry needs (jano_build_schedule_workspace_bytes,
 * align16(n_tokens) + align16(12 * ceil(n_tokens / 1024)) bytes) must not
 * exceed 1 MiB, which holds geometries of at most 1,036,416 tokens; larger
 * ones return JANO_EUNSUPPORTED before any CUDA call and launch nothing.
 * Other errors are those of jano_build_schedule.
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.
 * Sharing: every call on a device uses the same array and it keeps the last
 * call's contents (the builder needs no zeroed scratch).  Calls whose
 * launches overlap on the GPU (different streams, no ordering between them)
 * race on the array; order them on one stream or with events.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_build_schedule_noalloc(const uint8_t *block_levels, const jano_geom *g,
                                         const jano_sched_cfg *c, int32_t *offsets,
                                         int32_t *idx, size_t idx_capacity,
                                         uint8_t *token_levels, void *stream);

/* ------------------------------------------------------------------------
 * jano_kv_scatter -- write the fresh K/V rows of the due tokens into the
 * persistent full-sequence cache: k_cache[idx[i]] = k_act[i],
 * v_cache[idx[i]] = v_act[i], bit for bit, both in one pass.
 * Pages: nl technical summary, Methodologie 2 "KV Cache Mechanisme" (the
 * K/V of frozen tokens are kept and reused); zh 2.2 item 3; pt 2.B.
 *
 * k_act, v_act      device BF16 [n_act][heads][d].
 * idx               device int32 [n_act], strictly ascending ids in
 *                   [0, n_tokens) (what jano_build_schedule emits).  A row
 *                   whose id is out of range or not above the previous
 *                   row's id raises JANO_EINDEX on the device error word and
 *                   is skipped, so an adjacent duplicate never races; after
 *                   that error, which cache rows hold which values is
 *                   unspecified if the list was not ascending.
 * k_cache, v_cache  device BF16 [n_tokens][heads][d]; must not overlap the
 *                   act buffers.  All four 16-byte aligned; heads*d % 8 == 0.
 * n_act == 0 is a no-op.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_kv_scatter(const void *k_act, const void *v_act, const int32_t *idx,
                            int n_act, int heads, int d, void *k_cache,
                            void *v_cache, int n_tokens, void *stream);

/* ------------------------------------------------------------------------
 * jano_active_attention -- attention of only the active queries over the
 * whole cached K/V, outputs written back to their token rows:
 *   out[idx[i], h, :] = softmax_j(scale * q_act[i,h,:] . k_cache[j,h,:])
 *                       @ v_cache[:, h, :]        over all n_tokens j.
 * Pages: nl technical summary, Methodologie 2 "KV Cache Mechanisme" (cached
 * K/V concatenated with the active queries; no position restoration since
 * attention does not depend on the order of keys/values); ko 2.B; pt 2.B.
 * The cache is kept in token order, so no concatenation copy is made.
 *
 * q_act             device BF16 [n_act][heads][d] (the due tokens' queries,
 *                   in the order of idx).
 * k_cache, v_cache  device BF16 [n_tokens][heads][d].
 * idx               device int32 [n_act]: output row of each query,
 *                   strictly ascending in [0, n_tokens) (what
 *                   jano_build_schedule emits).  A row whose id is out of
 *                   range or not above the previous row's id raises
 *                   JANO_EINDEX and is not written.
 * out               device BF16 [n_tokens][heads][d]; only rows idx[] are
 *                   written.  May not alias the inputs.
 * d in {64, 128}; BF16 in, fp32 accumulate and softmax, BF16 out;
 * no mask, no bias; scale is normally 1/sqrt(d).  All pointers 16-byte
 * aligned.  n_act == 0 is a no-op.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_active_attention(const void *q_act, const void *k_cache,
                                  const void *v_cache, const int32_t *idx,
                                  int n_act, int n_tokens, int heads, int d,
                                  float scale, void *out, void *stream);

/* ------------------------------------------------------------------------
 * jano_active_attention_split -- jano_active_attention with each query
 * tile's keys cut into n_split ranges, one CTA per range, for due sets too
 * small to fill the GPU (same pages as jano_active_attention; splitting the
 * keys is valid because the softmax denominator and the weighted sum of V
 * are both sums over the keys).  Every range yields, per (query, head) row,
 * its unnormalised output O_s (fp32), its running maximum m_s (log2 domain)
 * and its sum l_s; a second pass merges them in split order:
 *   out[idx[i], h] = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,
 *   M = max_s m_s.
 * Arguments as jano_active_attention, plus:
 * n_split    1 .. min(ceil(n_tokens / 128), 65535); 1 behaves as jano_active_attention
 *            (workspace unused).
 * workspace  device buffer of ws_bytes >= jano_active_attention_workspace_bytes
 *            (n_act, heads, d, n_split), 16-byte aligned, owned by the
 *            caller; its contents are overwritten and need no zeroing.  The
 *            calls that share it must be ordered on one stream.
 * Errors: n_split out of range, or a NULL / too small workspace ->
 * JANO_EINVAL; a misaligned workspace -> JANO_EALIGN; the rest as
 * jano_active_attention.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_active_attention_split(const void *q_act, const void *k_cache,
                                        const void *v_cache, const int32_t *idx,
                                        int n_act, int n_tokens, int heads, int d,
                                        float scale, int n_split, void *workspace,
                                        size_t ws_bytes, void *out, void *stream);

/* Workspace bytes jano_active_attention_split needs (0 for n_split <= 1):
 * n_split * n_act * heads * d fp32 partial rows, rounded up to 256 bytes,
 * then n_split * n_act * heads (m, l) fp32 pairs. */
JANO_API size_t jano_active_attention_workspace_bytes(int n_act, int heads, int d, int n_split);

/* The key split with the shortest modelled time on the current device: with
 * C = ceil(n_act / 256) * heads CTAs per split, S SMs and nt = ceil(n_tokens
 * / 128) key tiles, the z (at most 16, at least 8 key tiles per CTA) that
 * minimises R(z) * (nt / z + 12), where R(z) counts floor(w) full rounds of
 * w = z C / S and a partial last round of fraction f as 0.7 + 0.3 f (the
 * constants are fitted to measured B200 sweeps).  Returns 1 when no split
 * pays (call jano_active_attention then), or 1 on any error. */
JANO_API int jano_active_attention_splits(int n_act, int n_tokens, int heads, int d);

/* The same choice for a device of sm_count SMs (host only, no device
 * query); 1 on invalid arguments. */
JANO_API int jano_active_attention_splits_on(int n_act, int n_tokens, int heads, int d, int sm_count);

/* ------------------------------------------------------------------------
 * jano_gather_gemm -- a linear layer on the active rows only, rows gathered
 * on the way in and optionally scattered on the way out.  Pages: nl
 * technical summary, Methodologie 2 "KV Cache Mechanisme" (per step only a
 * subset of the tokens is activated; the K/V of the frozen ones are kept),
 * so the DiT block's projections run on the active rows alone; zh 2.2
 * item 3.
 *
 *   for r < m:  out[dst(r)][j] = sum_c x[src(r)][c] * w[j][c]
 *   src(r) = gather ? gather[r] : r,   dst(r) = scatter ? scatter[r] : r
 *
 * x        device BF16 [n_x][k] (e.g. the hidden states of all tokens).
 * gather   device int32 [m] or NULL; values in [0, n_x).  Without it m <= n_x.
 * w        device BF16 [n][k]: a linear layer's weight in [out][in] layout.
 * scatter  device int32 [m] or NULL; strictly ascending values in
 *          [0, n_out).  Without it m <= n_out.
 * out      device BF16 [n_out][n]; rows not written keep their contents.
 * k % 8 == 0 and n % 8 == 0 (JANO_EUNSUPPORTED otherwise); x, w, out
 * 16-byte aligned.  BF16 in, fp32 accumulation on the tensor cores, BF16
 * out (round to nearest even).  An index out of range raises JANO_EINDEX on
 * the device error word: a bad gather index reads a row of zeros, a
 * scatter index out of range or not above the previous one drops the row.
 * m == 0 is a no-op.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_gather_gemm(const void *x, int n_x, const int32_t *gather, int m,
                                      const void *w, int n, int k, const int32_t *scatter,
                                      void *out, int n_out, void *stream);

/* ------------------------------------------------------------------------
 * jano_qkv_project -- the fused Q/K/V projection of the active tokens with
 * the KV-cache write (same passages as jano_gather_gemm, plus the KV cache
 * of Methodologie 2): with y_i = x[idx[i]] @ w_qkv^T,
 *
 *   q_act[i]        = y_i[0 .. hd)
 *   k_cache[idx[i]] = y_i[hd .. 2hd)
 *   v_cache[idx[i]] = y_i[2hd .. 3hd)
 *
 * so the fresh K/V rows go straight from the tensor cores into the
 * token-ordered cache: no K_act/V_act buffers and no separate
 * jano_kv_scatter.  hd = heads * d.
 *
 * x        device BF16 [n_tokens][k], the hidden states of all tokens.
 * idx      device int32 [n_act], the active tokens, strictly ascending in
 *          [0, n_tokens) (a K/V row whose id breaks that is dropped).
 * w_qkv    device BF16 [3*hd][k]: the Q rows, then the K rows, then the V rows.
 * q_act    device BF16 [n_act][hd]; k_cache, v_cache device BF16 [n_tokens][hd].
 * hd must be a multiple of 128 and k of 8 (JANO_EUNSUPPORTED otherwise);
 * pointers 16-byte aligned.  Errors as for jano_gather_gemm.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_qkv_project(const void *x, int n_tokens, const int32_t *idx, int n_act,
                                      const void *w_qkv, int hd, int k, void *q_act,
                                      void *k_cache, void *v_cache, void *stream);

/* ------------------------------------------------------------------------
 * jano_random_scores -- scores of the random-masking ablation.  Pages: ko
 * technical summary, section 4 "Ablation Study" (random masking at a
 * similar speed-up against Jano's convergence-aware levels).  Classifying
 * these scores with jano_classify gives a level map with the same level
 * counts as Jano's, assigned at random:
 *
 *   scores[b] = (r_{b+1} >> 40) * 2^-24,  r_i = output i of splitmix64 seeded with seed
 *
 * (splitmix64: Steele, Lea and Flood 2014; r_i is the 64-bit finaliser of
 * seed + i * 0x9E3779B97F4A7C15, so the map depends on the seed and the
 * block count only).  Uniform in [0, 1) with 24-bit resolution; ties, which
 * are rare, fall to the lower block index in jano_classify.
 *
 * scores  device fp32 [n_blocks].  n_blocks >= 1.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_random_scores(int n_blocks, uint64_t seed, float *scores, void *stream);

/* ------------------------------------------------------------------------
 * jano_fft_scores -- frequency-domain block complexity, the FFT baseline
 * the analyzer is compared with.  Pages: zh technical summary 1 (an FFT
 * complexity analysis cannot tell the patterns apart in the early,
 * noise-dominated steps) and 2.1 (FFT on the early latent: median
 * prediction accuracy 0.13-0.25 against the analyzer's 0.73); fr technical
 * summary 2.A.  The pages give no formula; this is its plainest form, on one
 * latent snapshot x (normally the last warm-up step's, x_K):
 *
 *   S_b = 1/C sum_c 1/n_b^2 sum_{u in U_hi} |X_{c,b}(u)|^2
 *
 * X_{c,b} is the 3-D DFT of block b of channel c over the block's own
 * m_f x m_h x m_w elements (edge blocks are smaller, n_b = m_f m_h m_w), and
 * U_hi holds the frequencies u whose folded index min(u_a, m_a - u_a)
 * reaches `cutoff` on at least one axis a.  By Parseval's theorem cutoff 0
 * gives the block's mean square and cutoff 1 its variance (all but the DC
 * bin); a cutoff above every folded index gives 0.  Blocks are ordered as in
 * jano_block_scores, so jano_classify takes these scores unchanged.
 *
 * x       device fp32 [C][F][H][W], one snapshot (4-byte aligned).
 * g       block geometry (bf, bh, bw); the patch fields are not read.
 *         bf * bh * bw <= 256 (JANO_EUNSUPPORTED beyond).
 * cutoff  >= 0.
 * scores  device fp32 [n_blocks].
 * Errors: JANO_EINVAL (NULL pointer, C < 1, cutoff < 0, bad geometry),
 * JANO_EUNSUPPORTED, JANO_ECUDA.  Deterministic: fixed summation order.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_fft_scores(const float *x, int C, const jano_geom *g, int cutoff,
                                     float *scores, void *stream);

/* ------------------------------------------------------------------------
 * jano_stream_sum -- one streaming pass over a float buffer: the read rate
 * that the analyzer's single pass over its latent history is compared with.
 * A calibration of the device, not a step of the method: the Jano pages have
 * no counterpart.  The kernel does the least work a full read can do (a
 * deep ring of 1-D bulk copies per CTA, the consumer threads adding the
 * floats), so its time is the launch, the ramp-up of the memory pipeline,
 * the stream itself and the tail, as for any one-pass kernel of that size.
 *
 * x          device fp32 [n], 16-byte aligned; n % 4 == 0 (n == 0 allowed).
 * partial    device fp32 [n_partial], 16-byte aligned: partial[i] is the sum
 *            (fp32, fixed order, deterministic) of the i-th contiguous share
 *            of x, shares of ceil(n / 4 / n_partial) float4s (the last ones
 *            may be shorter or empty, summing to 0).
 * n_partial  CTAs, 1..65535; the SM count gives one CTA per SM.
 * Errors: JANO_EINVAL (n < 0, n % 4, n_partial out of range, NULL),
 * JANO_EALIGN, JANO_ECUDA; a timed-out internal wait raises JANO_ETIMEOUT on
 * the device error word.
 * ---------------------------------------------------------------------- */
JANO_API jano_status jano_stream_sum(const float *x, long long n, float *partial, int n_partial,
                                     void *stream);

/* Synchronises `stream`, returns the first device-side error recorded on the
 * current device since the last call (JANO_OK if none) and clears it. */
JANO_API jano_status jano_get_device_error(void *stream);

/* Static English text for a status code. */
JANO_API const char *jano_status_str(jano_status s);

/* Library version, major*10000 + minor*100 + patch. */
JANO_API int jano_version(void);

#ifdef __cplusplus
}
#endif

#endif /* JANO_H */
