/*
 * CPU oracle for the fully-integer attention forward (IntAttention,
 * arXiv 2511.21513, "Methodology" item 2: IndexSoftmax = clip, 32-entry exp
 * lookup, int32 sum, reciprocal by integer multiply + right shift; item 3:
 * Q.K^T and V.softmax stay in the integer domain, end-to-end INT8).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or constant generator with
 * the CUDA library: the parameter derivation below is written out here on
 * its own.
 *
 * It is deliberately plain: scalar loops, one query row at a time, no SIMD,
 * no blocking.  Threads only split independent rows.
 *
 * The exact integer definition (the pages give only the shape of the method;
 * every constant, rounding rule and width below is this build's reading):
 *
 *   Host parameters, IEEE double, per head h (per-tensor: every h uses entry 0)
 *     alpha = (s_q * s_k) / sqrt(d)           logit units per integer score
 *     r     = (alpha * 31) / c                LUT steps per integer score
 *     s     = 26; while (s > 1 && llround(r * 2^s) > 2^24) s--
 *     M     = llround(r * 2^s)                need 1 <= M <= 2^24 and M <= 2^s
 *     D     = ceil(61 * 2^(s-1) / M)          smallest gap whose index is 31
 *     LUT[i]= llround(32768 * exp(-i * c / 31)), i = 0..30;  LUT[31] = 0
 *     m_o   = s_v / (255 * s_o) = f * 2^e, f in [0.5, 1)
 *     Mo    = llround(f * 2^31) (2^31 -> 2^30, e+1);  so = 31 - e in [1, 62]
 *
 *   Per query row i of head (b, h)
 *     J     = { j < Lk : !causal or j <= i + (Lk - Lq) }
 *     S_j   = sum_t Q[i,t] * K[j,t]                       (exact int32)
 *     m     = max_{j in J} S_j
 *     idx_j = (min(m - S_j, D) * M + 2^(s-1)) >> s        in [0, 31]
 *     E_j   = LUT[idx_j]                                  (0 outside J)
 *     Z     = sum_j E_j                                   (int32)
 *     R     = floor((255 * 2^32 + floor(Z/2)) / Z)
 *     P_j   = floor((E_j * R + 2^31) / 2^32)              in [0, 255]
 *     acc_t = sum_j P_j * V[j,t]                          (int32)
 *     out_t = clamp(floor((acc_t * Mo + 2^(so-1)) / 2^so), -127, 127)
 *
 *   Zero-points (the forum page "IntAttention：面向边缘设备的纯整数注意力推理加速方案",
 *   section 动态量化策略: a dynamic scale and zero-point per layer).  K and V
 *   may be stored as u8 codes with a zero-point z per tensor or per head:
 *   code c stands for the integer c - z (real value s * (c - z)).  The
 *   definition above then reads K[j,t] = k_code - z_k and V[j,t] = v_code -
 *   z_v; Q stays symmetric int8.  oracle_forward_zp / oracle_decode_zp
 *   compute exactly that, literally.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_INVALID_ARG 1
#define ORC_PARAM_RANGE 3

typedef struct {
    int32_t M, s, D, Mo, so;
} oracle_head_params;

/* LUT of pseudo-exponentials: 2^15 * exp(-i*c/31), last entry forced to 0 so
 * that a clipped gap contributes nothing (the sparsity of the clip). */
int oracle_lut(double c, int32_t lut[32])
{
    if (!(c > 0.0) || !isfinite(c)) return ORC_PARAM_RANGE;
    for (int i = 0; i < 31; i++) {
        double x = 32768.0 * exp(-((double)i * c) / 31.0);
        lut[i] = (int32_t)llround(x);
    }
    lut[31] = 0;
    return ORC_OK;
}

/* Index multiplier/shift and clip for one head. */
int oracle_index_params(double s_q, double s_k, int d, double c,
                        int32_t *M_out, int32_t *s_out, int32_t *D_out)
{
    if (!(s_q > 0.0) || !(s_k > 0.0) || !(c > 0.0) || !isfinite(s_q) ||
        !isfinite(s_k) || !isfinite(c) || d <= 0)
        return ORC_PARAM_RANGE;
    double alpha = (s_q * s_k) / sqrt((double)d);
    double r = (alpha * 31.0) / c;
    int s = 26;
    while (s > 1 && llround(ldexp(r, s)) > (1LL << 24)) s--;
    long long M = llround(ldexp(r, s));
    if (M < 1 || M > (1LL << 24) || M > (1LL << s)) return ORC_PARAM_RANGE;
    long long num = 61LL * (1LL << (s - 1));
    long long D = (num + M - 1) / M;
    *M_out = (int32_t)M;
    *s_out = s;
    *D_out = (int32_t)D;
    return ORC_OK;
}

/* Requantisation multiplier/shift: acc * s_v / (255 * s_o) ~ acc * Mo / 2^so. */
int oracle_requant_params(double s_v, double s_o, int32_t *Mo_out, int32_t *so_out)
{
    if (!(s_v > 0.0) || !(s_o > 0.0) || !isfinite(s_v) || !isfinite(s_o))
        return ORC_PARAM_RANGE;
    double m_real = s_v / (255.0 * s_o);
    int e = 0;
    double f = frexp(m_real, &e);
    long long Mo = llround(f * 2147483648.0);
    if (Mo == (1LL << 31)) {
        Mo = 1LL << 30;
        e += 1;
    }
    int so = 31 - e;
    if (so < 1 || so > 62) return ORC_PARAM_RANGE;
    *Mo_out = (int32_t)Mo;
    *so_out = so;
    return ORC_OK;
}

/* Parameters of every head.  Scale arrays hold H entries when per_head != 0,
 * else one entry that all heads share. */
int oracle_params(int per_head, const float *s_q, const float *s_k,
                  const float *s_v, const float *s_o, int H, int d, float clip_c,
                  int32_t lut[32], oracle_head_params *out)
{
    if (H <= 0 || !s_q || !s_k || !s_v || !s_o || !out || !lut) return ORC_INVALID_ARG;
    int rc = oracle_lut((double)clip_c, lut);
    if (rc) return rc;
    for (int h = 0; h < H; h++) {
        int e = per_head ? h : 0;
        rc = oracle_index_params((double)s_q[e], (double)s_k[e], d, (double)clip_c,
                                 &out[h].M, &out[h].s, &out[h].D);
        if (rc) return rc;
        rc = oracle_requant_params((double)s_v[e], (double)s_o[e], &out[h].Mo, &out[h].so);
        if (rc) return rc;
    }
    return ORC_OK;
}

/* S_j = sum_t q[t] * k[j*d + t] for j < n. */
void oracle_scores(const int8_t *q, const int8_t *k, int n, int d, int32_t *S)
{
    for (int j = 0; j < n; j++) {
        int32_t acc = 0;
        for (int t = 0; t < d; t++) acc += (int32_t)q[t] * (int32_t)k[(size_t)j * d + t];
        S[j] = acc;
    }
}

/* One gap -> LUT index, written exactly as defined (64-bit, no wrap tricks). */
int32_t oracle_index(int64_t gap, int32_t M, int32_t s, int32_t D)
{
    int64_t g = gap < (int64_t)D ? gap : (int64_t)D;
    int64_t t = g * (int64_t)M + ((int64_t)1 << (s - 1));
    return (int32_t)(t >> s);
}

/* IndexSoftmax of one row of n valid scores -> u8 probabilities.  Also
 * returns the row max, Z and R for inspection by the tests. */
void oracle_index_softmax(const int32_t *S, int n, int32_t M, int32_t s, int32_t D,
                          const int32_t lut[32], uint8_t *P, int32_t *m_out,
                          int32_t *Z_out, uint32_t *R_out)
{
    int32_t m = S[0];
    for (int j = 1; j < n; j++)
        if (S[j] > m) m = S[j];
    int32_t Z = 0;
    for (int j = 0; j < n; j++) Z += lut[oracle_index((int64_t)m - S[j], M, s, D)];
    uint64_t R = ((255ULL << 32) + (uint64_t)(Z / 2)) / (uint64_t)Z;
    for (int j = 0; j < n; j++) {
        uint64_t E = (uint64_t)lut[oracle_index((int64_t)m - S[j], M, s, D)];
        P[j] = (uint8_t)((E * R + (1ULL << 31)) >> 32);
    }
    if (m_out) *m_out = m;
    if (Z_out) *Z_out = Z;
    if (R_out) *R_out = (uint32_t)R;
}

/* floor(x / 2^k) for any sign of x, written without relying on >> of
 * negative numbers. */
static int64_t floor_div_pow2(int64_t x, int k)
{
    int64_t p = (int64_t)1 << k;
    if (x >= 0) return x / p;
    return -((-x + p - 1) / p);
}

int8_t oracle_requant(int32_t acc, int32_t Mo, int32_t so)
{
    int64_t t = (int64_t)acc * (int64_t)Mo + ((int64_t)1 << (so - 1));
    int64_t y = floor_div_pow2(t, so);
    if (y > 127) y = 127;
    if (y < -127) y = -127;
    return (int8_t)y;
}

/* One full attention row: q (d), K/V rows (n valid rows of d), out (d). */
static void attention_row(const int8_t *q, const int8_t *k, const int8_t *v, int n,
                          int d, const oracle_head_params *p, const int32_t lut[32],
                          int32_t *S, uint8_t *P, int32_t *acc, int8_t *out)
{
    oracle_scores(q, k, n, d, S);
    oracle_index_softmax(S, n, p->M, p->s, p->D, lut, P, NULL, NULL, NULL);
    for (int t = 0; t < d; t++) acc[t] = 0;
    for (int j = 0; j < n; j++)
        for (int t = 0; t < d; t++) acc[t] += (int32_t)P[j] * (int32_t)v[(size_t)j * d + t];
    for (int t = 0; t < d; t++) out[t] = oracle_requant(acc[t], p->Mo, p->so);
}

/* One attention row whose K and / or V codes carry a zero-point: kz / vz
 * are u8 codes with zero-points zk / zv when k_u8 / v_u8, else int8 codes
 * (zero-point 0).  Written out on its own, element by element. */
static int32_t code_at(const void *base, int is_u8, size_t i)
{
    return is_u8 ? (int32_t)((const uint8_t *)base)[i] : (int32_t)((const int8_t *)base)[i];
}

static void attention_row_zp(const int8_t *q, const void *kz, int k_u8, int32_t zk,
                             const void *vz, int v_u8, int32_t zv, int n, int d,
                             const oracle_head_params *p, const int32_t lut[32], int32_t *S,
                             uint8_t *P, int32_t *acc, int8_t *out)
{
    for (int j = 0; j < n; j++) {
        int64_t dot = 0;
        for (int t = 0; t < d; t++)
            dot += (int64_t)q[t] * (int64_t)(code_at(kz, k_u8, (size_t)j * d + t) - zk);
        S[j] = (int32_t)dot;
    }
    oracle_index_softmax(S, n, p->M, p->s, p->D, lut, P, NULL, NULL, NULL);
    for (int t = 0; t < d; t++) acc[t] = 0;
    for (int j = 0; j < n; j++)
        for (int t = 0; t < d; t++)
            acc[t] += (int32_t)P[j] * (code_at(vz, v_u8, (size_t)j * d + t) - zv);
    for (int t = 0; t < d; t++) out[t] = oracle_requant(acc[t], p->Mo, p->so);
}

typedef struct {
    const int8_t *q, *k, *v;
    int8_t *out;
    int B, H, Lq, Lk, Lkv, d, causal;
    const oracle_head_params *hp;
    const int32_t *lut;
    const int32_t *rows; /* NULL: all rows; else nrows triples (b, h, i) */
    long long nrows;
    int tid, nthreads;
    /* zero-points per head (H entries), NULL: int8 codes, zero-point 0 */
    const int32_t *zk, *zv;
} job_t;

static void *run_rows(void *arg)
{
    job_t *J = (job_t *)arg;
    int32_t *S = (int32_t *)malloc(sizeof(int32_t) * (size_t)J->Lk);
    uint8_t *P = (uint8_t *)malloc((size_t)J->Lk);
    int32_t *acc = (int32_t *)malloc(sizeof(int32_t) * (size_t)J->d);
    long long total = J->rows ? J->nrows : (long long)J->B * J->H * J->Lq;
    for (long long r = J->tid; r < total; r += J->nthreads) {
        long long b, h, i;
        if (J->rows) {
            b = J->rows[3 * r];
            h = J->rows[3 * r + 1];
            i = J->rows[3 * r + 2];
        } else {
            i = r % J->Lq;
            h = (r / J->Lq) % J->H;
            b = r / ((long long)J->Lq * J->H);
        }
        size_t bh = (size_t)(b * J->H + h);
        int n = J->Lk;
        if (J->causal) {
            long long last = i + (J->Lk - J->Lq);
            n = (int)(last + 1 < J->Lk ? last + 1 : J->Lk);
        }
        const int8_t *qrow = J->q + (bh * J->Lq + (size_t)i) * J->d;
        const int8_t *kb = J->k + bh * (size_t)J->Lkv * J->d;
        const int8_t *vb = J->v + bh * (size_t)J->Lkv * J->d;
        int8_t *o = J->out + (J->rows ? (size_t)r * J->d : (bh * J->Lq + (size_t)i) * J->d);
        if (J->zk || J->zv) {
            /* K / V codes are one byte each either way: the same offsets */
            attention_row_zp(qrow, kb, J->zk != NULL, J->zk ? J->zk[h] : 0, vb, J->zv != NULL,
                             J->zv ? J->zv[h] : 0, n, J->d, &J->hp[h], J->lut, S, P, acc, o);
        } else {
            attention_row(qrow, kb, vb, n, J->d, &J->hp[h], J->lut, S, P, acc, o);
        }
    }
    free(S);
    free(P);
    free(acc);
    return NULL;
}

static int run_threads(job_t *base, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 512) nthreads = 512;
    pthread_t th[512];
    job_t jobs[512];
    for (int t = 0; t < nthreads; t++) {
        jobs[t] = *base;
        jobs[t].tid = t;
        jobs[t].nthreads = nthreads;
    }
    int started = 0;
    for (int t = 1; t < nthreads; t++) {
        if (pthread_create(&th[t], NULL, run_rows, &jobs[t]) != 0) break;
        started = t;
    }
    /* rows of threads that failed to start are taken by thread 0 */
    if (started + 1 < nthreads) {
        for (int t = started + 1; t < nthreads; t++) run_rows(&jobs[t]);
    }
    run_rows(&jobs[0]);
    for (int t = 1; t <= started; t++) pthread_join(th[t], NULL);
    return ORC_OK;
}

static int check_common(const int8_t *q, const int8_t *k, const int8_t *v, int8_t *out,
                        int B, int H, int Lq, int Lk, int d, int causal)
{
    if (!q || !k || !v || !out) return ORC_INVALID_ARG;
    if (B < 0 || H <= 0 || Lq <= 0 || Lk <= 0 || Lk > 65535 || d <= 0) return ORC_INVALID_ARG;
    if (causal && Lq > Lk) return ORC_INVALID_ARG;
    return ORC_OK;
}

/* Prefill: q [B,H,Lq,d], k/v [B,H,Lk,d], out [B,H,Lq,d], all contiguous. */
int oracle_forward(const int8_t *q, const int8_t *k, const int8_t *v, int per_head,
                   const float *s_q, const float *s_k, const float *s_v,
                   const float *s_o, int B, int H, int Lq, int Lk, int d, int causal,
                   float clip_c, int8_t *out, int nthreads)
{
    int rc = check_common(q, k, v, out, B, H, Lq, Lk, d, causal);
    if (rc) return rc;
    int32_t lut[32];
    oracle_head_params *hp = (oracle_head_params *)malloc(sizeof(oracle_head_params) * (size_t)H);
    rc = oracle_params(per_head, s_q, s_k, s_v, s_o, H, d, clip_c, lut, hp);
    if (rc == ORC_OK && B > 0) {
        job_t J = {q, k, v, out, B, H, Lq, Lk, Lk, d, causal, hp, lut, NULL, 0, 0, 1, NULL, NULL};
        rc = run_threads(&J, nthreads);
    }
    free(hp);
    return rc;
}

/* Selected rows only: rows = nrows triples (b, h, i); out [nrows, d]. */
int oracle_forward_rows(const int8_t *q, const int8_t *k, const int8_t *v, int per_head,
                        const float *s_q, const float *s_k, const float *s_v,
                        const float *s_o, int B, int H, int Lq, int Lk, int d,
                        int causal, float clip_c, const int32_t *rows, long long nrows,
                        int8_t *out, int nthreads)
{
    int rc = check_common(q, k, v, out, B, H, Lq, Lk, d, causal);
    if (rc) return rc;
    if (!rows || nrows < 0) return ORC_INVALID_ARG;
    for (long long r = 0; r < nrows; r++) {
        if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 ||
            rows[3 * r + 1] >= H || rows[3 * r + 2] < 0 || rows[3 * r + 2] >= Lq)
            return ORC_INVALID_ARG;
    }
    int32_t lut[32];
    oracle_head_params *hp = (oracle_head_params *)malloc(sizeof(oracle_head_params) * (size_t)H);
    rc = oracle_params(per_head, s_q, s_k, s_v, s_o, H, d, clip_c, lut, hp);
    if (rc == ORC_OK) {
        job_t J = {q, k, v, out, B, H, Lq, Lk, Lk, d, causal, hp, lut, rows, nrows, 0, 1, NULL, NULL};
        rc = run_threads(&J, nthreads);
    }
    free(hp);
    return rc;
}

/* Decode: one query per (b, h) against the first Lk rows of an int8 cache of
 * capacity Lmax rows: q [B,H,1,d], caches [B,H,Lmax,d], out [B,H,1,d]. */
int oracle_decode(const int8_t *q, const int8_t *k_cache, const int8_t *v_cache,
                  int per_head, const float *s_q, const float *s_k, const float *s_v,
                  const float *s_o, int B, int H, int Lk, int Lmax, int d, float clip_c,
                  int8_t *out, int nthreads)
{
    int rc = check_common(q, k_cache, v_cache, out, B, H, 1, Lk, d, 0);
    if (rc) return rc;
    if (Lmax < Lk) return ORC_INVALID_ARG;
    int32_t lut[32];
    oracle_head_params *hp = (oracle_head_params *)malloc(sizeof(oracle_head_params) * (size_t)H);
    rc = oracle_params(per_head, s_q, s_k, s_v, s_o, H, d, clip_c, lut, hp);
    if (rc == ORC_OK && B > 0) {
        job_t J = {q, k_cache, v_cache, out, B, H, 1, Lk, Lmax, d, 0, hp, lut, NULL, 0, 0, 1, NULL, NULL};
        rc = run_threads(&J, nthreads);
    }
    free(hp);
    return rc;
}

/* Zero-points of every head from a per-tensor (one entry) or per-head (H
 * entries) array; NULL stays NULL.  Each must be a u8 code, 0..255. */
static int expand_zero_points(const int32_t *z, int per_head, int H, int32_t **out)
{
    *out = NULL;
    if (!z) return ORC_OK;
    int32_t *e = (int32_t *)malloc(sizeof(int32_t) * (size_t)H);
    for (int h = 0; h < H; h++) {
        int32_t v = z[per_head ? h : 0];
        if (v < 0 || v > 255) {
            free(e);
            return ORC_INVALID_ARG;
        }
        e[h] = v;
    }
    *out = e;
    return ORC_OK;
}

/* Prefill with zero-points: k / v are u8 codes [B,H,Lk,d] when z_k / z_v is
 * given (per_head: H entries, else one), int8 codes otherwise. */
int oracle_forward_zp(const int8_t *q, const void *k, const void *v, const int32_t *z_k,
                      const int32_t *z_v, int per_head, const float *s_q, const float *s_k,
                      const float *s_v, const float *s_o, int B, int H, int Lq, int Lk, int d,
                      int causal, float clip_c, int8_t *out, int nthreads)
{
    int rc = check_common(q, (const int8_t *)k, (const int8_t *)v, out, B, H, Lq, Lk, d, causal);
    if (rc) return rc;
    int32_t *zk = NULL, *zv = NULL;
    rc = expand_zero_points(z_k, per_head, H, &zk);
    if (rc == ORC_OK) rc = expand_zero_points(z_v, per_head, H, &zv);
    int32_t lut[32];
    oracle_head_params *hp = (oracle_head_params *)malloc(sizeof(oracle_head_params) * (size_t)H);
    if (rc == ORC_OK) rc = oracle_params(per_head, s_q, s_k, s_v, s_o, H, d, clip_c, lut, hp);
    if (rc == ORC_OK && B > 0) {
        job_t J = {q, (const int8_t *)k, (const int8_t *)v, out, B, H, Lq, Lk, Lk, d, causal, hp, lut,
                   NULL, 0, 0, 1, zk, zv};
        rc = run_threads(&J, nthreads);
    }
    free(hp);
    free(zk);
    free(zv);
    return rc;
}

/* Decode with zero-points: caches [B,H,Lmax,d] of u8 codes where z_k / z_v is
 * given, int8 codes otherwise; the first Lk rows are attended. */
int oracle_decode_zp(const int8_t *q, const void *k_cache, const void *v_cache,
                     const int32_t *z_k, const int32_t *z_v, int per_head, const float *s_q,
                     const float *s_k, const float *s_v, const float *s_o, int B, int H, int Lk,
                     int Lmax, int d, float clip_c, int8_t *out, int nthreads)
{
    int rc = check_common(q, (const int8_t *)k_cache, (const int8_t *)v_cache, out, B, H, 1, Lk, d, 0);
    if (rc) return rc;
    if (Lmax < Lk) return ORC_INVALID_ARG;
    int32_t *zk = NULL, *zv = NULL;
    rc = expand_zero_points(z_k, per_head, H, &zk);
    if (rc == ORC_OK) rc = expand_zero_points(z_v, per_head, H, &zv);
    int32_t lut[32];
    oracle_head_params *hp = (oracle_head_params *)malloc(sizeof(oracle_head_params) * (size_t)H);
    if (rc == ORC_OK) rc = oracle_params(per_head, s_q, s_k, s_v, s_o, H, d, clip_c, lut, hp);
    if (rc == ORC_OK && B > 0) {
        job_t J = {q, (const int8_t *)k_cache, (const int8_t *)v_cache, out, B, H, 1, Lk, Lmax, d, 0,
                   hp, lut, NULL, 0, 0, 1, zk, zv};
        rc = run_threads(&J, nthreads);
    }
    free(hp);
    free(zk);
    free(zv);
    return rc;
}
