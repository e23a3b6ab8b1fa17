/*
 * CPU oracle for the M-FALCON masked attention (forward and gradients), the
 * KV pool write and the cross-stage rank decode.  TEST INFRASTRUCTURE ONLY: the tests, the smoke
 * check and the benchmark's CPU-baseline leg call it; the product path never
 * does.  It shares no code, header or constant with the CUDA library.
 *
 * Plain fp64 C, written for a reader checking it against the pages:
 *
 *   [notes]  UniPinRec reproduction notes (slinene.github.io, ai-papers-daily,
 *            "unipinrec-unified-retrieval-ranking-masked-action-kv-share"),
 *            sub-module details §3 "attention mask" and §6 "serving:
 *            cross-process KV sharing".
 *   [review] UniPinRec paper review (liuzhao09.github.io,
 *            "pinterest-unipinrec"), §2.2 joint objective and §2.4
 *            co-serving / cross-stage KV cache.
 *
 * Mask ([notes] §3; [review] §2.2): the past part of a sequence is standard
 * causal attention; every candidate sees all n past positions; candidates
 * never see one another.  Whether a candidate sees itself is not stated on
 * the pages; the reading used here is "yes" (flag cand_self=1), so every row
 * attends to at least one key.  cand_self=0 gives the stricter reading of
 * [review] §2.2 ("candidates attend only to past history"); a row with no key
 * at all then outputs 0.
 *
 *   past row      (i <  n_b):  allowed(i, j) = j <= i
 *   candidate row (i >= n_b):  allowed(i, j) = j < n_b  or  (cand_self and j == i)
 *
 * which for cand_self=1 is the single rule  (j == i) or (j < min(i, n_b)).
 *
 * Score and softmax (no scale is printed on the pages; 1/sqrt(D) is passed in):
 *   s_ij = scale * sum_d q_id k_jd,   O_i = sum_j e^{s_ij - m_i} v_j / sum_j e^{s_ij - m_i}
 * over allowed j, with m_i = max over allowed j.  Inputs are bfloat16 bit
 * patterns, widened exactly to double.
 *
 * Heads ([notes] §6 calls the pool's H "KV heads"): queries may have more
 * heads than keys and values, H = G * Hkv; query head h reads key/value head
 * h / G (grouped-query attention).  G = 1 is plain multi-head attention.
 *
 * Pool ([notes] §6; [review] §2.4): one preallocated tensor of shape
 * [L, S, H, n, D] (layer, slot, KV head, history length, head dim) for K and
 * one for V.  Rank decode of a request reads rows 0..n_r-1 of its slot at the
 * given layer and adds the candidate's own key (same mask: all past + self).
 *
 * Parallelism: OpenMP over independent (row, head) pairs only; each output is
 * computed by one straight loop in the order written above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* The M-FALCON mask for one segment with n_past past tokens (row i, key j are
 * positions inside the segment). */
static int allowed(int64_t i, int64_t j, int64_t n_past, int cand_self)
{
    if (i < n_past) return j <= i;            /* past row: causal incl. diagonal */
    if (j < n_past) return 1;                 /* candidate row: every past key   */
    return cand_self && j == i;               /* ... plus itself, no other cand. */
}

/* Segment that holds packed token t: the last b with cu[b] <= t. */
static int find_segment(const int32_t *cu, int B, int64_t t)
{
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if ((int64_t)cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/* Softmax attention of one query row over an explicit key list.
 * keys[j], vals[j] point at D bf16 values.  out receives D doubles. */
static void attend(const uint16_t *qrow, const uint16_t *const *keys,
                   const uint16_t *const *vals, int64_t nkeys, int D, double scale,
                   double *s, double *out, double *lse)
{
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (nkeys == 0) {
        if (lse) *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < nkeys; ++j) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += bf16_to_f64(qrow[d]) * bf16_to_f64(keys[j][d]);
        s[j] = dot * scale;
        if (s[j] > m) m = s[j];
    }
    double denom = 0.0;
    for (int64_t j = 0; j < nkeys; ++j) {
        double w = exp(s[j] - m);
        denom += w;
        for (int d = 0; d < D; ++d) out[d] += w * bf16_to_f64(vals[j][d]);
    }
    for (int d = 0; d < D; ++d) out[d] /= denom;
    if (lse) *lse = m + log(denom);
}

/*
 * Masked prefill attention over packed segments.
 *   q           : bf16 bits, [T, H, D] row-major, T = cu_seqlens[B]
 *   k, v        : bf16 bits, [T, Hkv, D]; query head h reads kv head h / (H / Hkv)
 *   cu_seqlens  : [B+1], segment b spans tokens cu[b] .. cu[b+1]-1
 *   past_lens   : [B], n_b <= cu[b+1]-cu[b]; the rest of segment b are candidates
 *   tokens      : packed token indices to evaluate (NULL = all T)
 *   out         : [ntok, H, D] doubles; lse: [ntok, H] natural-log sum-exp or NULL
 * Returns 0, or -1 on inconsistent arguments.
 */
int oracle_prefill_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *cu_seqlens, const int32_t *past_lens, int B, int H, int Hkv, int D,
                        double scale, int cand_self, const int64_t *tokens, int64_t ntok,
                        double *out, double *lse)
{
    if (B < 1 || H < 1 || D < 1 || Hkv < 1 || H % Hkv != 0) return -1;
    const int G = H / Hkv;
    int64_t T = cu_seqlens[B];
    int64_t max_len = 0;
    for (int b = 0; b < B; ++b) {
        int64_t len = (int64_t)cu_seqlens[b + 1] - cu_seqlens[b];
        if (len < 0 || past_lens[b] < 0 || past_lens[b] > len) return -1;
        if (len > max_len) max_len = len;
    }
    if (!tokens) ntok = T;
    for (int64_t r = 0; r < ntok; ++r) {
        int64_t t = tokens ? tokens[r] : r;
        if (t < 0 || t >= T) return -1;
    }
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(max_len + 1));
        const uint16_t **kp = (const uint16_t **)malloc(sizeof(void *) * (size_t)(max_len + 1));
        const uint16_t **vp = (const uint16_t **)malloc(sizeof(void *) * (size_t)(max_len + 1));
        if (!s || !kp || !vp) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t rh = 0; rh < ntok * H; ++rh) {
            if (bad) continue;
            int64_t r = rh / H;
            int h = (int)(rh % H);
            int64_t t = tokens ? tokens[r] : r;
            int b = find_segment(cu_seqlens, B, t);
            int64_t start = cu_seqlens[b], len = (int64_t)cu_seqlens[b + 1] - start;
            int64_t i = t - start, n_past = past_lens[b];
            int64_t nk = 0;
            for (int64_t j = 0; j < len; ++j) {
                if (!allowed(i, j, n_past, cand_self)) continue;
                kp[nk] = k + ((start + j) * Hkv + h / G) * (int64_t)D;
                vp[nk] = v + ((start + j) * Hkv + h / G) * (int64_t)D;
                ++nk;
            }
            attend(q + (t * H + h) * (int64_t)D, kp, vp, nk, D, scale, s,
                   out + (r * H + h) * (int64_t)D, lse ? lse + r * H + h : NULL);
        }
        free(s);
        free((void *)kp);
        free((void *)vp);
    }
    return bad ? -1 : 0;
}

/*
 * Rank decode over the cached pool ([review] §2.4, [notes] §6).
 *   qc             : candidate bf16 bits, [Tc, H, D], Tc = cu_c[R]
 *   kc, vc         : candidate bf16 bits, [Tc, Hkv, D]
 *   cu_c           : [R+1] candidate offsets of each request
 *   slot_ids       : [R] pool slot of each request
 *   past_lens      : [R] cached rows n_r of each request (n_r <= n_cap)
 *   pool_k, pool_v : bf16 bits, [L, S, Hkv, n_cap, D]; query head h reads kv head h / (H / Hkv)
 *   tokens         : candidate indices to evaluate (NULL = all Tc)
 * Candidate c of request r attends to pool rows 0..n_r-1 of slot_ids[r] at
 * `layer`, and (cand_self) to its own key/value.
 */
int oracle_decode_rows(const uint16_t *qc, const uint16_t *kc, const uint16_t *vc,
                       const int32_t *cu_c, const int32_t *slot_ids, const int32_t *past_lens,
                       int R, int H, int Hkv, int D, double scale, int cand_self,
                       const uint16_t *pool_k, const uint16_t *pool_v, int L, int S, int n_cap,
                       int layer, const int64_t *tokens, int64_t ntok, double *out, double *lse)
{
    if (R < 1 || H < 1 || D < 1 || layer < 0 || layer >= L || Hkv < 1 || H % Hkv != 0) return -1;
    const int G = H / Hkv;
    for (int r = 0; r < R; ++r) {
        if (cu_c[r + 1] < cu_c[r]) return -1;
        if (slot_ids[r] < 0 || slot_ids[r] >= S) return -1;
        if (past_lens[r] < 0 || past_lens[r] > n_cap) return -1;
    }
    int64_t Tc = cu_c[R];
    if (!tokens) ntok = Tc;
    for (int64_t x = 0; x < ntok; ++x) {
        int64_t t = tokens ? tokens[x] : x;
        if (t < 0 || t >= Tc) return -1;
    }
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(n_cap + 1));
        const uint16_t **kp = (const uint16_t **)malloc(sizeof(void *) * (size_t)(n_cap + 1));
        const uint16_t **vp = (const uint16_t **)malloc(sizeof(void *) * (size_t)(n_cap + 1));
        if (!s || !kp || !vp) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t xh = 0; xh < ntok * H; ++xh) {
            if (bad) continue;
            int64_t x = xh / H;
            int h = (int)(xh % H);
            int64_t t = tokens ? tokens[x] : x;
            int r = find_segment(cu_c, R, t);
            int64_t n_r = past_lens[r];
            int64_t row0 = (((int64_t)layer * S + slot_ids[r]) * Hkv + h / G) * (int64_t)n_cap;
            int64_t nk = 0;
            for (int64_t j = 0; j < n_r; ++j) {
                kp[nk] = pool_k + (row0 + j) * D;
                vp[nk] = pool_v + (row0 + j) * D;
                ++nk;
            }
            if (cand_self) {
                kp[nk] = kc + (t * Hkv + h / G) * (int64_t)D;
                vp[nk] = vc + (t * Hkv + h / G) * (int64_t)D;
                ++nk;
            }
            attend(qc + (t * H + h) * (int64_t)D, kp, vp, nk, D, scale, s,
                   out + (x * H + h) * (int64_t)D, lse ? lse + x * H + h : NULL);
        }
        free(s);
        free((void *)kp);
        free((void *)vp);
    }
    return bad ? -1 : 0;
}

/*
 * Gradients of the masked prefill attention.  [review] §2.2 trains the whole
 * sequence [past || candidates] in one forward pass under this mask (the
 * joint objective); the backward pass below is the plain chain rule of the
 * forward defined above, over the same allowed (i, j) pairs:
 *
 *   P_ij  = softmax_j over allowed j of s_ij,  s_ij = scale * q_i . k_j
 *   O_i   = sum_j P_ij v_j
 *   given dO (the gradient of the loss with respect to O):
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = dO_i . v_j
 *   dS_ij = P_ij (dP_ij - sum_l P_il dP_il)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 *
 * so a past key receives gradient from the later past rows and from every
 * candidate row; a candidate's own key and value only from its own row.
 * With grouped heads a key/value head's gradient sums the contributions of
 * its G query heads.  Inputs are doubles (bf16 inputs are widened exactly by
 * the caller); dq [T, H, D], dk and dv [T, Hkv, D] are written in full.
 * Parallel over (segment, kv head): every gradient element belongs to
 * exactly one of them.
 */
int oracle_prefill_bwd_f64(const double *q, const double *k, const double *v, const double *dout,
                           const int32_t *cu_seqlens, const int32_t *past_lens, int B, int H, int Hkv, int D,
                           double scale, int cand_self, double *dq, double *dk, double *dv)
{
    if (B < 1 || H < 1 || D < 1 || Hkv < 1 || H % Hkv != 0) return -1;
    const int G = H / Hkv;
    int64_t max_len = 0;
    for (int b = 0; b < B; ++b) {
        int64_t len = (int64_t)cu_seqlens[b + 1] - cu_seqlens[b];
        if (len < 0 || past_lens[b] < 0 || past_lens[b] > len) return -1;
        if (len > max_len) max_len = len;
    }
    int64_t T = cu_seqlens[B];
    memset(dq, 0, sizeof(double) * (size_t)(T * H * D));
    memset(dk, 0, sizeof(double) * (size_t)(T * Hkv * D));
    memset(dv, 0, sizeof(double) * (size_t)(T * Hkv * D));
    int bad = 0;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)(max_len + 1));
        double *dp = (double *)malloc(sizeof(double) * (size_t)(max_len + 1));
        int64_t *js = (int64_t *)malloc(sizeof(int64_t) * (size_t)(max_len + 1));
        if (!p || !dp || !js) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < (int64_t)B * Hkv; ++bh) {
            if (bad) continue;
            int b = (int)(bh / Hkv), hk = (int)(bh % Hkv);
            int64_t start = cu_seqlens[b], len = (int64_t)cu_seqlens[b + 1] - start, n_past = past_lens[b];
            for (int h = hk * G; h < (hk + 1) * G; ++h)
#define ROW(x, t) ((x) + (((start + (t)) * H + h) * (int64_t)D))
#define KROW(x, t) ((x) + (((start + (t)) * Hkv + hk) * (int64_t)D))
            for (int64_t i = 0; i < len; ++i) {
                int64_t nk = 0;
                for (int64_t j = 0; j < len; ++j)
                    if (allowed(i, j, n_past, cand_self)) js[nk++] = j;
                if (nk == 0) continue;              /* no key: O_i = 0 carries no gradient */
                /* forward of row i: P_ij */
                double m = -INFINITY;
                for (int64_t a = 0; a < nk; ++a) {
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += ROW(q, i)[d] * KROW(k, js[a])[d];
                    p[a] = dot * scale;
                    if (p[a] > m) m = p[a];
                }
                double den = 0.0;
                for (int64_t a = 0; a < nk; ++a) {
                    p[a] = exp(p[a] - m);
                    den += p[a];
                }
                for (int64_t a = 0; a < nk; ++a) p[a] /= den;
                /* dP_ij = dO_i . v_j and its P-weighted mean over the row */
                double dmean = 0.0;
                for (int64_t a = 0; a < nk; ++a) {
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += ROW(dout, i)[d] * KROW(v, js[a])[d];
                    dp[a] = dot;
                    dmean += p[a] * dot;
                }
                for (int64_t a = 0; a < nk; ++a) {
                    int64_t j = js[a];
                    double ds = p[a] * (dp[a] - dmean);
                    for (int d = 0; d < D; ++d) {
                        KROW(dv, j)[d] += p[a] * ROW(dout, i)[d];
                        ROW(dq, i)[d] += scale * ds * KROW(k, j)[d];
                        KROW(dk, j)[d] += scale * ds * ROW(q, i)[d];
                    }
                }
            }
#undef ROW
#undef KROW
        }
        free(p);
        free(dp);
        free(js);
    }
    return bad ? -1 : 0;
}

/* As oracle_prefill_bwd_f64 for bf16 inputs (bit patterns), widened exactly. */
int oracle_prefill_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                       const int32_t *cu_seqlens, const int32_t *past_lens, int B, int H, int Hkv, int D,
                       double scale, int cand_self, double *dq, double *dk, double *dv)
{
    if (B < 1 || H < 1 || D < 1 || Hkv < 1) return -1;
    size_t n = (size_t)cu_seqlens[B] * (size_t)H * (size_t)D;       /* q, dout */
    size_t m = (size_t)cu_seqlens[B] * (size_t)Hkv * (size_t)D;     /* k, v */
    double *w = (double *)malloc(sizeof(double) * (2 * n + 2 * m + 1));
    if (!w) return -1;
    for (size_t x = 0; x < n; ++x) {
        w[x] = bf16_to_f64(q[x]);
        w[n + x] = bf16_to_f64(dout[x]);
    }
    for (size_t x = 0; x < m; ++x) {
        w[2 * n + x] = bf16_to_f64(k[x]);
        w[2 * n + m + x] = bf16_to_f64(v[x]);
    }
    int rc = oracle_prefill_bwd_f64(w, w + 2 * n, w + 2 * n + m, w + n, cu_seqlens, past_lens, B, H, Hkv, D,
                                    scale, cand_self, dq, dk, dv);
    free(w);
    return rc;
}

/*
 * Pool write mirror: pool[layer, slot_ids[b], h, j, :] = K[cu[b] + j, h, :]
 * for every j < past_lens[b] (and the same for V).  A byte copy; nothing else
 * in the pool is touched.
 */
int oracle_pool_write(uint16_t *pool_k, uint16_t *pool_v, int L, int S, int H, int n_cap, int D,
                      int layer, const uint16_t *k, const uint16_t *v, const int32_t *cu_seqlens,
                      const int32_t *past_lens, const int32_t *slot_ids, int B)
{
    if (layer < 0 || layer >= L || B < 0) return -1;
    for (int b = 0; b < B; ++b) {
        if (slot_ids[b] < 0 || slot_ids[b] >= S) return -1;
        if (past_lens[b] < 0 || past_lens[b] > n_cap) return -1;
        if (past_lens[b] > cu_seqlens[b + 1] - cu_seqlens[b]) return -1;
    }
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            int64_t row0 = (((int64_t)layer * S + slot_ids[b]) * H + h) * (int64_t)n_cap;
            for (int64_t j = 0; j < past_lens[b]; ++j) {
                int64_t src = (((int64_t)cu_seqlens[b] + j) * H + h) * (int64_t)D;
                memcpy(pool_k + (row0 + j) * D, k + src, sizeof(uint16_t) * (size_t)D);
                memcpy(pool_v + (row0 + j) * D, v + src, sizeof(uint16_t) * (size_t)D);
            }
        }
    }
    return 0;
}

/*
 * E4M3 pool variant (an extrapolation: the pages apply FP8 E4M3 to linear
 * layers, [notes]/[review] FP8 sections; here the pool stores K and V in it).
 *
 * E4M3 ("fn" form): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 *   exponent field 0       subnormal  (-1)^s * m/8 * 2^-6    (m = 1..7)
 *   exponent field 1..15   normal     (-1)^s * (1 + m/8) * 2^(e-7)
 *   field 15 with m = 7 is NaN; there is no infinity; the largest finite
 *   magnitude is 1.75 * 2^8 = 448.
 *
 * Encoding (the reading used for the pool): round the real value to the
 * nearest E4M3 value, ties to the even mantissa, and clamp magnitudes that
 * round beyond 448 to 448 ("saturate to finite").  NaN encodes as 0x7F.
 */
uint8_t oracle_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a == 0.0) return sign;
    /* grid spacing of the binade holding a: 2^-9 below the smallest normal 2^-6 */
    int e;
    frexp(a, &e);                     /* a = f * 2^e, f in [0.5, 1): binade exponent e - 1 */
    int be = e - 1;
    if (be < -6) be = -6;             /* subnormal range shares the spacing of the first binade */
    double spacing = ldexp(1.0, be - 3);
    double q = nearbyint(a / spacing);   /* exact division by a power of two; ties to even */
    double val = q * spacing;
    if (val > 448.0) val = 448.0;
    /* re-derive the fields from the rounded value (rounding may carry into the next binade) */
    if (val < ldexp(1.0, -6)) {
        int m = (int)(val / ldexp(1.0, -9));
        return sign | (uint8_t)m;
    }
    frexp(val, &e);
    int ex = e - 1;
    int m = (int)(val / ldexp(1.0, ex - 3)) - 8;
    return sign | (uint8_t)(((ex + 7) << 3) | m);
}

double oracle_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40);   /* quiet NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/*
 * Pool write into an E4M3 pool: the same rows as oracle_pool_write, each
 * element stored as E4M3(k * inv_scale) with the product taken in float32
 * (the bfloat16 input widened exactly, one rounding of the product).
 */
int oracle_pool_write_e4m3(uint8_t *pool_k, uint8_t *pool_v, int L, int S, int H, int n_cap, int D,
                           int layer, const uint16_t *k, const uint16_t *v, const int32_t *cu_seqlens,
                           const int32_t *past_lens, const int32_t *slot_ids, int B, float inv_k, float inv_v)
{
    if (layer < 0 || layer >= L || B < 0) return -1;
    for (int b = 0; b < B; ++b) {
        if (slot_ids[b] < 0 || slot_ids[b] >= S) return -1;
        if (past_lens[b] < 0 || past_lens[b] > n_cap) return -1;
        if (past_lens[b] > cu_seqlens[b + 1] - cu_seqlens[b]) return -1;
    }
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            int64_t row0 = (((int64_t)layer * S + slot_ids[b]) * H + h) * (int64_t)n_cap;
            for (int64_t j = 0; j < past_lens[b]; ++j) {
                int64_t src = (((int64_t)cu_seqlens[b] + j) * H + h) * (int64_t)D;
                for (int d = 0; d < D; ++d) {
                    float kf = (float)bf16_to_f64(k[src + d]) * inv_k;
                    float vf = (float)bf16_to_f64(v[src + d]) * inv_v;
                    pool_k[(row0 + j) * D + d] = oracle_e4m3_encode(kf);
                    pool_v[(row0 + j) * D + d] = oracle_e4m3_encode(vf);
                }
            }
        }
    }
    return 0;
}

/*
 * What an attention kernel reads from an E4M3 pool: bfloat16(decode(c) * scale),
 * the product in float32, rounded to nearest even.  Elementwise over n codes.
 */
void oracle_e4m3_dequant_bf16(const uint8_t *codes, int64_t n, float scale, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) {
        float f = (float)oracle_e4m3_decode(codes[i]) * scale;
        out[i] = f32_to_bf16_rne(f);
    }
}
