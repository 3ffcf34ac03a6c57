/*
 * CPU oracle for ADAMAS sparse decode attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the package's smoke check and the bench's CPU-baseline leg may
 * load this library.  It shares no code with the CUDA path.  It is plain, slow
 * and written to be checked by eye against the method's description in the
 * ADAMAS long-context sparse attention article (lnwmold.com/news/826806):
 *
 *   step 1  bf16 -> fp32 (exact: the bf16 bits are the top half of an fp32)
 *   step 2  Hadamard rotation (§2.1 "Hadamard transform"): y = H x / sqrt(d) with
 *           the Sylvester matrix H[i][j] = (-1)^popcount(i & j), evaluated as the
 *           divide-and-conquer butterfly the section mentions, in fp32, stage
 *           widths h = 1, 2, ..., d/2 in that order, (a, b) -> (a + b, a - b), then
 *           one multiply by C = RN_fp32(1 / sqrt(128)) (bit pattern 0x3DB504F3).
 *           Compiled with -ffp-contract=off so no FMA changes a rounding.
 *   step 3  dynamic bucketing (§2.2 "dynamic bucketing"): per 128-dim group
 *           m = max |y_i|, thresholds (-m/2, 0, +m/2); code 0 if y < -m/2,
 *           1 if y < 0, 2 if y < m/2, else 3.
 *   step 4  packing (§3.1 "memory compression"): four 2-bit codes per byte, first
 *           code in the top bits: byte j = c[4j]<<6 | c[4j+1]<<4 | c[4j+2]<<2 | c[4j+3].
 *   step 5  score (§2.3 "Manhattan distance"): D = sum_i |cq_i - ck_i| over the
 *           unpacked codes; a smaller D means a more relevant token (score = -D).
 *   step 6  select (§5.2 token budget): the k_eff = min(k, len) tokens of smallest
 *           D, ties to the lower token index, listed in (D, index) order; slots
 *           past k_eff hold -1.
 *   step 7  attention over the selected rows, in float64 from the bf16 values:
 *           s_r = q . K[idx_r] / sqrt(d), p = exp(s - max s), out = sum p V / sum p
 *           (the rotation leaves q . k unchanged, §2.1, so the exact dot product is
 *           taken on the original vectors).  No selected row: out = 0.
 *
 * Layouts: K, V [B][Hkv][Nmax][d] bf16 bits; codes [B][Hkv][Nmax][d/4] bytes;
 * q [B][Hq][d]; query head h reads kv head h / (Hq / Hkv).  d must be 128.
 * Functions return 0 on success and -1 on a bad argument.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define D128 128
#define CODE_BYTES (D128 / 4)

static float bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static float norm_constant(void)
{
    uint32_t u = 0x3DB504F3u; /* round-to-nearest fp32 of 1/sqrt(128) */
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* step 2: y = H x / sqrt(128), Sylvester order, in place */
static void fwht128(float *x)
{
    for (int h = 1; h < D128; h *= 2) {
        for (int i = 0; i < D128; i += 2 * h) {
            for (int j = i; j < i + h; ++j) {
                float a = x[j];
                float b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
        }
    }
    const float c = norm_constant();
    for (int j = 0; j < D128; ++j)
        x[j] = x[j] * c;
}

/* step 3: one 128-dim group */
static void bucket128(const float *y, uint8_t *code)
{
    float m = 0.0f;
    for (int i = 0; i < D128; ++i) {
        float a = fabsf(y[i]);
        if (a > m)
            m = a;
    }
    const float t0 = -0.5f * m;
    const float t1 = 0.0f;
    const float t2 = 0.5f * m;
    for (int i = 0; i < D128; ++i) {
        if (y[i] < t0)
            code[i] = 0;
        else if (y[i] < t1)
            code[i] = 1;
        else if (y[i] < t2)
            code[i] = 2;
        else
            code[i] = 3;
    }
}

/* step 4 */
static void pack128(const uint8_t *code, uint8_t *out)
{
    for (int j = 0; j < CODE_BYTES; ++j)
        out[j] = (uint8_t)((code[4 * j] << 6) | (code[4 * j + 1] << 4) | (code[4 * j + 2] << 2) |
                           code[4 * j + 3]);
}

static void unpack128(const uint8_t *packed, uint8_t *code)
{
    for (int j = 0; j < CODE_BYTES; ++j) {
        code[4 * j] = (packed[j] >> 6) & 3;
        code[4 * j + 1] = (packed[j] >> 4) & 3;
        code[4 * j + 2] = (packed[j] >> 2) & 3;
        code[4 * j + 3] = packed[j] & 3;
    }
}

/* ------------------------------------------------------------------ exported */

/* Rotated fp32 values of n bf16 vectors (steps 1-2). */
int oracle_rotate(const uint16_t *x, int64_t n, int d, float *y)
{
    if (d != D128 || n < 0 || (n > 0 && (!x || !y)))
        return -1;
    for (int64_t v = 0; v < n; ++v) {
        float *row = y + v * D128;
        for (int i = 0; i < D128; ++i)
            row[i] = bf16_to_float(x[v * D128 + i]);
        fwht128(row);
    }
    return 0;
}

/* Codes (steps 3-4) of n already-rotated fp32 vectors. */
int oracle_bucket_pack(const float *y, int64_t n, int d, uint8_t *packed)
{
    if (d != D128 || n < 0 || (n > 0 && (!y || !packed)))
        return -1;
    uint8_t code[D128];
    for (int64_t v = 0; v < n; ++v) {
        bucket128(y + v * D128, code);
        pack128(code, packed + v * CODE_BYTES);
    }
    return 0;
}

/* Packed codes of n bf16 vectors (steps 1-4). */
int oracle_encode(const uint16_t *x, int64_t n, int d, uint8_t *packed)
{
    if (d != D128 || n < 0 || (n > 0 && (!x || !packed)))
        return -1;
    float y[D128];
    uint8_t code[D128];
    for (int64_t v = 0; v < n; ++v) {
        for (int i = 0; i < D128; ++i)
            y[i] = bf16_to_float(x[v * D128 + i]);
        fwht128(y);
        bucket128(y, code);
        pack128(code, packed + v * CODE_BYTES);
    }
    return 0;
}

/* Step 5 for one query against n keys: D[t] = L1 distance of the unpacked codes. */
int oracle_distance(const uint8_t *qcode, const uint8_t *kcodes, int64_t n, int d, int32_t *D)
{
    if (d != D128 || n < 0 || !qcode || (n > 0 && (!kcodes || !D)))
        return -1;
    uint8_t cq[D128], ck[D128];
    unpack128(qcode, cq);
    for (int64_t t = 0; t < n; ++t) {
        unpack128(kcodes + t * CODE_BYTES, ck);
        int32_t s = 0;
        for (int i = 0; i < D128; ++i)
            s += abs((int)cq[i] - (int)ck[i]);
        D[t] = s;
    }
    return 0;
}

typedef struct {
    int32_t dist;
    int32_t tok;
} scored_t;

static int cmp_scored(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    if (a->dist != b->dist)
        return a->dist < b->dist ? -1 : 1;
    if (a->tok != b->tok)
        return a->tok < b->tok ? -1 : 1;
    return 0;
}

/* Step 6: idx[0..k) = tokens of smallest (D, index); -1 past min(k, n). */
int oracle_select(const int32_t *D, int64_t n, int64_t k, int32_t *idx)
{
    if (n < 0 || k < 0 || (n > 0 && !D) || (k > 0 && !idx) || n > INT32_MAX)
        return -1;
    scored_t *s = (scored_t *)malloc((size_t)(n > 0 ? n : 1) * sizeof *s);
    if (!s)
        return -1;
    for (int64_t t = 0; t < n; ++t) {
        s[t].dist = D[t];
        s[t].tok = (int32_t)t;
    }
    qsort(s, (size_t)n, sizeof *s, cmp_scored);
    int64_t keff = k < n ? k : n;
    for (int64_t r = 0; r < k; ++r)
        idx[r] = r < keff ? s[r].tok : -1;
    free(s);
    return 0;
}

/* Step 7: attention of one query over the rows idx[0..k) (entries < 0 are skipped). */
int oracle_attend(const uint16_t *q, const uint16_t *K, const uint16_t *V, const int32_t *idx,
                  int64_t k, int d, double *out)
{
    if (d != D128 || k < 0 || !q || !out || (k > 0 && (!K || !V || !idx)))
        return -1;
    double *s = (double *)malloc((size_t)(k > 0 ? k : 1) * sizeof *s);
    if (!s)
        return -1;
    const double scale = 1.0 / sqrt((double)D128);
    double smax = -INFINITY;
    int64_t used = 0;
    for (int64_t r = 0; r < k; ++r) {
        if (idx[r] < 0)
            continue;
        const uint16_t *kr = K + (int64_t)idx[r] * D128;
        double acc = 0.0;
        for (int i = 0; i < D128; ++i)
            acc += (double)bf16_to_float(q[i]) * (double)bf16_to_float(kr[i]);
        s[r] = acc * scale;
        if (s[r] > smax)
            smax = s[r];
        ++used;
    }
    for (int i = 0; i < D128; ++i)
        out[i] = 0.0;
    if (used == 0) {
        free(s);
        return 0;
    }
    double denom = 0.0;
    for (int64_t r = 0; r < k; ++r) {
        if (idx[r] < 0)
            continue;
        double p = exp(s[r] - smax);
        denom += p;
        const uint16_t *vr = V + (int64_t)idx[r] * D128;
        for (int i = 0; i < D128; ++i)
            out[i] += p * (double)bf16_to_float(vr[i]);
    }
    for (int i = 0; i < D128; ++i)
        out[i] /= denom;
    free(s);
    return 0;
}

/* ---------------------------------------------------------- whole decode step */

typedef struct {
    const uint16_t *q, *K, *V;
    const uint8_t *codes;
    const int32_t *seq_lens;
    int B, Hq, Hkv, budget;
    int64_t Nmax;
    double *out;
    int32_t *idx;
    int32_t *dist; /* optional [B][Hq][Nmax] */
    int first, stride;
    int status;
} step_job_t;

static void *step_worker(void *arg)
{
    step_job_t *j = (step_job_t *)arg;
    const int G = j->Hq / j->Hkv;
    int32_t *D = (int32_t *)malloc((size_t)(j->Nmax > 0 ? j->Nmax : 1) * sizeof(int32_t));
    if (!D) {
        j->status = -1;
        return NULL;
    }
    uint8_t qcode[CODE_BYTES];
    for (int bh = j->first; bh < j->B * j->Hq; bh += j->stride) {
        const int b = bh / j->Hq, h = bh % j->Hq, g = h / G;
        int64_t len = j->seq_lens[b];
        if (len < 0)
            len = 0;
        if (len > j->Nmax)
            len = j->Nmax;
        const uint16_t *qv = j->q + (int64_t)bh * D128;
        const int64_t kv_off = ((int64_t)b * j->Hkv + g) * j->Nmax;
        int32_t *idx = j->idx + (int64_t)bh * j->budget;
        if (oracle_encode(qv, 1, D128, qcode) ||
            oracle_distance(qcode, j->codes + kv_off * CODE_BYTES, len, D128, D) ||
            oracle_select(D, len, j->budget, idx) ||
            oracle_attend(qv, j->K + kv_off * D128, j->V + kv_off * D128, idx, j->budget, D128,
                          j->out + (int64_t)bh * D128)) {
            j->status = -1;
            break;
        }
        if (j->dist) {
            int32_t *dd = j->dist + (int64_t)bh * j->Nmax;
            for (int64_t t = 0; t < j->Nmax; ++t)
                dd[t] = t < len ? D[t] : -1;
        }
    }
    free(D);
    return NULL;
}

/*
 * One decode step for the whole batch (steps 1-7 per query head).  codes must be
 * the oracle's own encoding of K (oracle_encode).  out is float64 [B][Hq][128],
 * idx is int32 [B][Hq][budget], dist (may be NULL) receives int32 [B][Hq][Nmax]
 * distances with -1 past each sequence's length.  Sequence lengths are clamped
 * to [0, Nmax].  The (b, head) pairs are split over nthreads POSIX threads.
 */
int oracle_decode_step(const uint16_t *q, const uint16_t *K, const uint16_t *V, const uint8_t *codes,
                       const int32_t *seq_lens, int B, int Hq, int Hkv, int64_t Nmax, int d,
                       int budget, double *out, int32_t *idx, int32_t *dist, int nthreads)
{
    if (d != D128 || B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Nmax < 0 || budget < 0 ||
        !q || !K || !V || !codes || !seq_lens || !out || (budget > 0 && !idx))
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > 256)
        nthreads = 256;
    step_job_t jobs[256];
    pthread_t tid[256];
    int started[256];
    for (int i = 0; i < nthreads; ++i) {
        step_job_t j = {q, K, V, codes, seq_lens, B, Hq, Hkv, budget, Nmax, out, idx, dist, i,
                        nthreads, 0};
        jobs[i] = j;
        started[i] = (i > 0) && pthread_create(&tid[i], NULL, step_worker, &jobs[i]) == 0;
        if (i > 0 && !started[i])
            step_worker(&jobs[i]);
    }
    step_worker(&jobs[0]);
    int status = jobs[0].status;
    for (int i = 1; i < nthreads; ++i) {
        if (started[i])
            pthread_join(tid[i], NULL);
        if (jobs[i].status)
            status = jobs[i].status;
    }
    return status;
}
