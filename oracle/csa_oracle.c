/*
 * csa_oracle.c -- plain float64 CPU oracle for the hybrid CSA/HCA attention step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or helper with
 * the CUDA library; the two are compared on the same seeded input bits.
 *
 * Every function is written for clarity, not speed: straight loops in
 * float64, one query (or one compressed entry) at a time, with an optional
 * OpenMP loop over independent queries/entries that does not change any
 * arithmetic.  Inputs are the exact bf16 / u8 bit patterns the GPU consumes;
 * bf16 values are widened exactly to double.
 *
 * Sources (web pages describing DeepSeek-V4; no code is printed there for
 * any of these operations):
 *   [DSv4-KR]  "DeepSeek v4" (it.peoplentools.com), section
 *              "Compressed Sparse Attention" -> "압축된 Key-Value entry"
 *              (compressed entries) and "sparse selection용 Lightning
 *              Indexer" (indexer, top-k, sliding window); section
 *              "CSA와 HCA를 결합한 하이브리드 attention" (HCA: m' >> m).
 *   [DSv4-AN]  "DeepSeek-AI (2026) - ARXIV-2606.19348" (dmarx anthology
 *              record), "Key takeaways": two latent KV streams pooling
 *              overlapping 2m-token windows; RMSNorm on each query head and
 *              on the single compressed KV head.
 *   [DSv4-MAP] "DeepSeek-V4-Pro - Model techniques map" (inteligile.com),
 *              table "Checked in its code": rows "Grouped-query attention"
 *              (one KV head, 128 query heads), "Sliding-window attention"
 *              (window 128, current token included), "Indexer-selected sparse
 *              attention" (top-k 1024, 64 x 128 indexer heads, invalid slots
 *              -> -1), "QK normalization", "Learnable attention sink",
 *              "Partial RoPE", "Gated attention output" (rope-conjugate
 *              rotation of the output); list "inference quantization"
 *              -> "FP4 precision for the attention indexer", "FP8 KV-cache
 *              quantization".
 *   [DSv4-FP4] "DeepSeek V4 paper full version is out, FP4 QAT details and
 *              stability tricks [D]" (corsoro.com): the indexer QK path uses
 *              FP4 activations.
 * Where the pages leave a formula open the reading used here is the one
 * stated at each function (pooling logit order, compression-weight rows,
 * causal visibility, window rows, RoPE tables and pairing, FP4 and FP8 block
 * formats).
 *
 * Parity pins: every function below is pinned by tests/test_oracle_pins.py
 * against closed forms, brute force or an independent library routine.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* scalar helpers                                                      */
/* ------------------------------------------------------------------ */

/* bf16 is the top 16 bits of an IEEE binary32; widening is exact. */
static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------ */
/* 1. Compressed KV entries  [DSv4-KR "압축된 Key-Value entry"], [DSv4-AN]  */
/* ------------------------------------------------------------------ */
/*
 * Entry i (0 <= i < N = floor(T/m)) pools 2m token rows per channel c:
 *   rows j = 0..m-1   : stream B, token (i-1)*m + j   (the previous m tokens)
 *   rows j = m..2m-1  : stream A, token  i*m + (j-m)   (the newest m tokens)
 * with weights w_j[c] = softmax_j(logits[j][c]) over the 2m rows (a per-channel
 * softmax over 2m elements).  For i = 0 the B half is padded with logit -inf
 * and value 0, so the softmax runs over the A half only.  Optionally the
 * entry is RMS-normalised over its d channels:
 *   y[c] = x[c] / sqrt(mean_c(x^2) + eps) * g[c]     (g = 1 when gain is NULL)
 * Reading: the pages call the weights "compression weights + learnable
 * positional bias"; here the positional logits alone are the weights, they
 * do not depend on the input.
 *
 * Computes entries [i0, i0 + ni) of every sequence; out is [batch][ni][d].
 */
void orc_compress(const uint16_t *A, const uint16_t *B, const float *logits,
                  int batch, long long T, int d, int m,
                  int apply_rmsnorm, const float *gain, double eps,
                  long long i0, long long ni, double *out)
{
    const int two_m = 2 * m;
    double *w_full = (double *)malloc(sizeof(double) * (size_t)two_m * d);
    double *w_first = (double *)malloc(sizeof(double) * (size_t)m * d);

    for (int c = 0; c < d; ++c) {
        /* softmax over all 2m rows (entries i >= 1) */
        double mx = -INFINITY;
        for (int j = 0; j < two_m; ++j)
            if ((double)logits[(size_t)j * d + c] > mx) mx = logits[(size_t)j * d + c];
        double den = 0.0;
        for (int j = 0; j < two_m; ++j) den += exp((double)logits[(size_t)j * d + c] - mx);
        for (int j = 0; j < two_m; ++j)
            w_full[(size_t)j * d + c] = exp((double)logits[(size_t)j * d + c] - mx) / den;

        /* softmax over the A half only (entry 0: B logits are -inf) */
        double mx0 = -INFINITY;
        for (int j = m; j < two_m; ++j)
            if ((double)logits[(size_t)j * d + c] > mx0) mx0 = logits[(size_t)j * d + c];
        double den0 = 0.0;
        for (int j = m; j < two_m; ++j) den0 += exp((double)logits[(size_t)j * d + c] - mx0);
        for (int j = m; j < two_m; ++j)
            w_first[(size_t)(j - m) * d + c] = exp((double)logits[(size_t)j * d + c] - mx0) / den0;
    }

    const long long total = (long long)batch * ni;
#pragma omp parallel for schedule(static)
    for (long long job = 0; job < total; ++job) {
        const long long b = job / ni;
        const long long i = i0 + job % ni;
        const uint16_t *Ab = A + (size_t)b * T * d;
        const uint16_t *Bb = B + (size_t)b * T * d;
        double *o = out + (size_t)job * d;

        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            if (i == 0) {
                for (int j = 0; j < m; ++j)
                    acc += w_first[(size_t)j * d + c] * bf16_bits_to_double(Ab[(size_t)j * d + c]);
            } else {
                for (int j = 0; j < m; ++j)
                    acc += w_full[(size_t)j * d + c] *
                           bf16_bits_to_double(Bb[(size_t)((i - 1) * m + j) * d + c]);
                for (int j = 0; j < m; ++j)
                    acc += w_full[(size_t)(m + j) * d + c] *
                           bf16_bits_to_double(Ab[(size_t)(i * m + j) * d + c]);
            }
            o[c] = acc;
        }
        if (apply_rmsnorm) {
            double ms = 0.0;
            for (int c = 0; c < d; ++c) ms += o[c] * o[c];
            ms /= d;
            const double r = 1.0 / sqrt(ms + eps);
            for (int c = 0; c < d; ++c) o[c] = o[c] * r * (gain ? (double)gain[c] : 1.0);
        }
    }
    free(w_full);
    free(w_first);
}

/*
 * Compressed entries with input-dependent compression weights
 * [DSv4-KR "압축된 Key-Value entry"]: from the hidden states come, per token,
 * the two KV streams C_a (here A), C_b (here B) and two compression-weight
 * rows Z_a, Z_b; entry i combines its 2m rows with the weights plus the
 * learnable positional biases B_a, B_b under a per-channel softmax over the
 * 2m elements, and for i = 0 the previous block is padded with Z_b = -inf,
 * C_b = 0.  For channel c:
 *   l_j = Zb[(i-1)m + j][c] + bias[j][c]      (j = 0..m-1, previous block, i >= 1)
 *   l_j = Za[i*m + j-m][c]  + bias[j][c]      (j = m..2m-1, own block)
 *   C_i[c] = sum_j softmax_j(l)[j] * x_j[c]   (x_j the matching B or A row)
 * then the optional RMSNorm of orc_compress.
 * Readings: bias rows 0..m-1 are B_b and rows m..2m-1 are B_a (the order
 * orc_compress uses); Z_a and Z_b are bf16 like the streams; a NULL Za or Zb
 * contributes 0, so with both NULL this is orc_compress.
 *
 * Computes entries [i0, i0 + ni) of every sequence; out is [batch][ni][d].
 */
void orc_compress_dynamic(const uint16_t *A, const uint16_t *B, const uint16_t *Za, const uint16_t *Zb,
                          const float *bias, int batch, long long T, int d, int m,
                          int apply_rmsnorm, const float *gain, double eps,
                          long long i0, long long ni, double *out)
{
    const long long total = (long long)batch * ni;
#pragma omp parallel for schedule(static)
    for (long long job = 0; job < total; ++job) {
        const long long b = job / ni;
        const long long i = i0 + job % ni;
        const size_t seq = (size_t)b * T * d;
        double *o = out + (size_t)job * d;
        double *l = (double *)malloc(sizeof(double) * 2 * (size_t)m);
        double *x = (double *)malloc(sizeof(double) * 2 * (size_t)m);

        for (int c = 0; c < d; ++c) {
            /* the 2m (logit, value) pairs of this channel; entry 0 has only its own block */
            int n = 0;
            if (i > 0) {
                for (int j = 0; j < m; ++j) {
                    const size_t row = seq + (size_t)((i - 1) * m + j) * d + c;
                    l[n] = (Zb ? bf16_bits_to_double(Zb[row]) : 0.0) + (double)bias[(size_t)j * d + c];
                    x[n] = bf16_bits_to_double(B[row]);
                    ++n;
                }
            }
            for (int j = 0; j < m; ++j) {
                const size_t row = seq + (size_t)(i * m + j) * d + c;
                l[n] = (Za ? bf16_bits_to_double(Za[row]) : 0.0) + (double)bias[(size_t)(m + j) * d + c];
                x[n] = bf16_bits_to_double(A[row]);
                ++n;
            }
            double mx = -INFINITY;
            for (int j = 0; j < n; ++j)
                if (l[j] > mx) mx = l[j];
            double den = 0.0, acc = 0.0;
            for (int j = 0; j < n; ++j) {
                const double e = exp(l[j] - mx);
                den += e;
                acc += e * x[j];
            }
            o[c] = acc / den;
        }
        if (apply_rmsnorm) {
            double ms = 0.0;
            for (int c = 0; c < d; ++c) ms += o[c] * o[c];
            ms /= d;
            const double r = 1.0 / sqrt(ms + eps);
            for (int c = 0; c < d; ++c) o[c] = o[c] * r * (gain ? (double)gain[c] : 1.0);
        }
        free(l);
        free(x);
    }
}

/* RMSNorm of `rows` vectors of length d (used for the query heads).
 * [DSv4-AN]: an RMSNorm is applied to each query head before core attention. */
void orc_rmsnorm_bf16(const uint16_t *x, long long rows, int d, double eps,
                      const float *gain, double *out)
{
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; ++r) {
        double ms = 0.0;
        for (int c = 0; c < d; ++c) {
            double v = bf16_bits_to_double(x[(size_t)r * d + c]);
            ms += v * v;
        }
        ms /= d;
        double s = 1.0 / sqrt(ms + eps);
        for (int c = 0; c < d; ++c)
            out[(size_t)r * d + c] =
                bf16_bits_to_double(x[(size_t)r * d + c]) * s * (gain ? (double)gain[c] : 1.0);
    }
}

/* Number of compressed entries visible to a query at position t: an entry is
 * usable once all of its A tokens are at or before t, i.e. s < floor((t+1)/m)
 * (reading of the causal threshold of [DSv4-MAP] "Indexer-selected sparse
 * attention"), capped at N. */
static long long n_visible(long long t, int m, long long N)
{
    long long v = (t + 1) / m;
    if (v < 0) v = 0;
    if (v > N) v = N;
    return v;
}

long long orc_n_visible(long long t, int m, long long N) { return n_visible(t, m, N); }

/* ------------------------------------------------------------------ */
/* 2. Lightning indexer  [DSv4-KR "sparse selection용 Lightning Indexer"]  */
/* ------------------------------------------------------------------ */
/*
 *   S[q][s] = sum_h w[q][h] * max(0, q_I[q][h] . K_I[s])   for s < n_vis(t_q)
 *   S[q][s] = -inf                                          otherwise
 * One indexer key per compressed entry, shared by all indexer heads.
 * q_idx [batch][nq][H_I][d_I] bf16, w [batch][nq][H_I] fp32,
 * k_idx [batch][N][d_I] bf16, q_pos [batch][nq], scores [batch][nq][N].
 */
void orc_index(const uint16_t *q_idx, const float *w, const uint16_t *k_idx,
               const int *q_pos, int batch, int nq, long long N, int H_I, int d_I,
               int m, double *scores)
{
    const long long total = (long long)batch * nq;
    for (long long bq = 0; bq < total; ++bq) {
        const long long b = bq / nq;
        const long long nv = n_visible(q_pos[bq], m, N);
        const uint16_t *qq = q_idx + (size_t)bq * H_I * d_I;
        const float *ww = w + (size_t)bq * H_I;
        const uint16_t *kb = k_idx + (size_t)b * N * d_I;
        double *S = scores + (size_t)bq * N;
#pragma omp parallel for schedule(static)
        for (long long s = 0; s < N; ++s) {
            if (s >= nv) {
                S[s] = -INFINITY;
                continue;
            }
            double acc = 0.0;
            for (int h = 0; h < H_I; ++h) {
                double dot = 0.0;
                for (int j = 0; j < d_I; ++j)
                    dot += bf16_bits_to_double(qq[(size_t)h * d_I + j]) *
                           bf16_bits_to_double(kb[(size_t)s * d_I + j]);
                acc += (double)ww[h] * (dot > 0.0 ? dot : 0.0);
            }
            S[s] = acc;
        }
    }
}

/* ------------------------------------------------------------------ */
/* 3. Causal top-k  [DSv4-KR Lightning Indexer], [DSv4-MAP]            */
/* ------------------------------------------------------------------ */
/*
 * For each query: a full sort of the visible entries by (score descending,
 * index ascending), keeping the first min(k, n_vis).  The remaining slots are
 * -1 (an invalid slot, as in [DSv4-MAP]).  idx [batch][nq][k] lists the
 * chosen entries in that sorted order.
 */
typedef struct {
    double score;
    long long index;
} orc_scored_t;

static int cmp_scored(const void *pa, const void *pb)
{
    const orc_scored_t *a = (const orc_scored_t *)pa, *b = (const orc_scored_t *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->index < b->index) ? -1 : (a->index > b->index);
}

void orc_topk(const double *scores, const int *q_pos, int batch, int nq, long long N,
              int m, int k, int *idx)
{
    const long long total = (long long)batch * nq;
#pragma omp parallel for schedule(dynamic)
    for (long long bq = 0; bq < total; ++bq) {
        const long long nv = n_visible(q_pos[bq], m, N);
        orc_scored_t *v = (orc_scored_t *)malloc(sizeof(orc_scored_t) * (size_t)(nv > 0 ? nv : 1));
        for (long long s = 0; s < nv; ++s) {
            v[s].score = scores[(size_t)bq * N + s];
            v[s].index = s;
        }
        qsort(v, (size_t)nv, sizeof(orc_scored_t), cmp_scored);
        for (int i = 0; i < k; ++i)
            idx[(size_t)bq * k + i] = (i < nv) ? (int)v[i].index : -1;
        free(v);
    }
}

/* ------------------------------------------------------------------ */
/* 4. Core attention (MQA, K = V)  [DSv4-MAP], [DSv4-KR], [DSv4-AN]    */
/* ------------------------------------------------------------------ */
/*
 * For one query at position t with H heads of dim D and one shared KV head:
 *   qh_hat = RMSNorm(q_h)                 (eps, optional gain [D])
 *   J      = { kv[j] : j in the key list } U { A[u] : max(0,t-W+1) <= u <= t }
 *   o_h    = sum_{x in J} softmax_x(scale * qh_hat . x) * x
 * Keys and values are the same rows (one KV head).  Window rows are raw
 * stream-A rows (no RMSNorm); overlap with compressed entries is kept.
 */
/*
 * Partial rotary position embedding ([DSv4-MAP] "Partial RoPE": only the
 * trailing qk_rope_head_dim = 64 channels of each 512-channel head are
 * rotated, the leading "nope" channels are left as they are; the rotated
 * slice is x*cos + rotate_half(x)*sin, rotate_half taking the slice's two
 * halves (x1, x2) to (-x2, x1)).  For a row x of `width` channels at
 * position p, with n = width - rope_dim, r = rope_dim / 2 and
 * c_i = cos_t[p][i], s_i = sin_t[p][i] (i < r):
 *   y[n + i]     = x[n + i] * c_i - x[n + r + i] * s_i
 *   y[n + r + i] = x[n + r + i] * c_i + x[n + i] * s_i
 * (channel n+i is paired with n+r+i).  inverse != 0 rotates by the conjugate
 * (s_i -> -s_i), which undoes the rotation ([DSv4-MAP] "Gated attention
 * output": the attention output goes through a rope-conjugate rotation).
 * Reading: the cos / sin tables [positions][r] are the caller's (their
 * frequencies, YaRN scaling included, are not part of this step).
 */
static void rope_rotate(double *x, int width, int rope_dim, long long p, const float *cos_t,
                        const float *sin_t, int inverse)
{
    const int r = rope_dim / 2, n = width - rope_dim;
    for (int i = 0; i < r; ++i) {
        const double c = (double)cos_t[(size_t)p * r + i];
        const double sn = (double)sin_t[(size_t)p * r + i];
        const double s = inverse ? -sn : sn;
        const double x1 = x[n + i], x2 = x[n + r + i];
        x[n + i] = x1 * c - x2 * s;
        x[n + r + i] = x2 * c + x1 * s;
    }
}

/* rows x [rows][width] (float64) at positions pos[rows] -> out [rows][width] */
void orc_rope(const double *x, long long rows, int width, int rope_dim, const int *pos,
              const float *cos_t, const float *sin_t, int inverse, double *out)
{
    for (long long i = 0; i < rows; ++i) {
        memcpy(out + (size_t)i * width, x + (size_t)i * width, sizeof(double) * (size_t)width);
        rope_rotate(out + (size_t)i * width, width, rope_dim, pos[i], cos_t, sin_t, inverse);
    }
}

/*
 * One query, all H heads.  With rope_dim > 0 the RMS-normalised query head is
 * rotated at the query position t before the dot products, and each head's
 * output is rotated back by the conjugate at t (keys and window rows arrive
 * already rotated at their own positions: they are values too, K = V).
 */
static void attend_one(const uint16_t *q, const float *q_gain, const float *sinks, int H, int D,
                       double scale, double eps, const uint16_t *const *rows, long long nrows,
                       int rope_dim, const float *rope_cos, const float *rope_sin, long long t,
                       double *out)
{
    double *qh = (double *)malloc(sizeof(double) * (size_t)D);
    double *z = (double *)malloc(sizeof(double) * (size_t)(nrows > 0 ? nrows : 1));
    for (int h = 0; h < H; ++h) {
        double ms = 0.0;
        for (int c = 0; c < D; ++c) {
            double v = bf16_bits_to_double(q[(size_t)h * D + c]);
            ms += v * v;
        }
        ms /= D;
        const double r = 1.0 / sqrt(ms + eps);
        for (int c = 0; c < D; ++c)
            qh[c] = bf16_bits_to_double(q[(size_t)h * D + c]) * r * (q_gain ? (double)q_gain[c] : 1.0);
        if (rope_dim > 0) rope_rotate(qh, D, rope_dim, t, rope_cos, rope_sin, 0);

        double mx = -INFINITY;
        for (long long j = 0; j < nrows; ++j) {
            double dot = 0.0;
            for (int c = 0; c < D; ++c) dot += qh[c] * bf16_bits_to_double(rows[j][c]);
            z[j] = scale * dot;
            if (z[j] > mx) mx = z[j];
        }
        /* learnable sink ([DSv4-MAP] "Learnable attention sink"): one more
         * logit per head in the softmax denominator, with no value row */
        const double sink = sinks ? (double)sinks[h] : -INFINITY;
        if (sink > mx) mx = sink;
        double den = sinks && isfinite(mx) ? exp(sink - mx) : 0.0;
        for (long long j = 0; j < nrows; ++j) {
            z[j] = exp(z[j] - mx);
            den += z[j];
        }
        double *o = out + (size_t)h * D;
        for (int c = 0; c < D; ++c) o[c] = 0.0;
        for (long long j = 0; j < nrows && den > 0.0; ++j) {
            const double p = z[j] / den;
            for (int c = 0; c < D; ++c) o[c] += p * bf16_bits_to_double(rows[j][c]);
        }
        if (rope_dim > 0) rope_rotate(o, D, rope_dim, t, rope_cos, rope_sin, 1);
    }
    free(qh);
    free(z);
}

/* Window rows: stream-A rows of positions u in [max(0, t-W+1), t] that the
 * window buffer holds; win [batch][win_rows][D] holds positions
 * win_pos0 .. win_pos0 + win_rows - 1 (win_pos0 = 0, win_rows = T for a whole
 * stream; win_pos0 = t-W+1, win_rows = W for a decode window cache). */
static long long window_rows(const uint16_t *win, long long win_pos0, long long win_rows, int W,
                             long long b, long long t, int D, const uint16_t **rows)
{
    long long n = 0;
    for (long long u = t - W + 1; u <= t; ++u) {
        if (u < 0 || u < win_pos0 || u - win_pos0 >= win_rows) continue;
        rows[n++] = win + ((size_t)b * win_rows + (u - win_pos0)) * D;
    }
    return n;
}

/* CSA: key list = selected compressed entries (idx != -1 and 0 <= idx < N)
 * plus the sliding window.  q [batch][nq][H][D], kv [batch][N][D],
 * idx [batch][nq][k], win [batch][win_rows][D], out [batch][nq][H][D]. */
void orc_attend(const uint16_t *q, const float *q_gain, const float *sinks, const uint16_t *kv, long long N,
                const int *idx, int k, const uint16_t *win, long long win_pos0, long long win_rows, int W,
                const int *q_pos, int batch, int nq, int H, int D, double scale, double eps,
                int rope_dim, const float *rope_cos, const float *rope_sin, double *out)
{
    const long long total = (long long)batch * nq;
#pragma omp parallel for schedule(dynamic)
    for (long long bq = 0; bq < total; ++bq) {
        const long long b = bq / nq;
        const long long t = q_pos[bq];
        const uint16_t **rows = (const uint16_t **)malloc(sizeof(uint16_t *) * (size_t)(k + W));
        long long n = 0;
        for (int i = 0; i < k; ++i) {
            const long long j = idx[(size_t)bq * k + i];
            if (j < 0 || j >= N) continue;
            rows[n++] = kv + ((size_t)b * N + j) * D;
        }
        n += window_rows(win, win_pos0, win_rows, W, b, t, D, rows + n);
        attend_one(q + (size_t)bq * H * D, q_gain, sinks, H, D, scale, eps, rows, n,
                   rope_dim, rope_cos, rope_sin, t, out + (size_t)bq * H * D);
        free(rows);
    }
}

/* HCA: dense attention over every visible compressed entry (j < n_vis(t))
 * plus the sliding window; no indexer ([DSv4-KR] hybrid-attention section:
 * HCA compresses every m' >> m tokens and keeps attention dense). */
void orc_hca_attend(const uint16_t *q, const float *q_gain, const float *sinks, const uint16_t *kv, long long N,
                    int m, const uint16_t *win, long long win_pos0, long long win_rows, int W,
                    const int *q_pos,
                    int batch, int nq, int H, int D, double scale, double eps,
                    int rope_dim, const float *rope_cos, const float *rope_sin, double *out)
{
    const long long total = (long long)batch * nq;
#pragma omp parallel for schedule(dynamic)
    for (long long bq = 0; bq < total; ++bq) {
        const long long b = bq / nq;
        const long long t = q_pos[bq];
        const long long nv = n_visible(t, m, N);
        const uint16_t **rows = (const uint16_t **)malloc(sizeof(uint16_t *) * (size_t)(nv + W + 1));
        long long n = 0;
        for (long long j = 0; j < nv; ++j) rows[n++] = kv + ((size_t)b * N + j) * D;
        n += window_rows(win, win_pos0, win_rows, W, b, t, D, rows + n);
        attend_one(q + (size_t)bq * H * D, q_gain, sinks, H, D, scale, eps, rows, n,
                   rope_dim, rope_cos, rope_sin, t, out + (size_t)bq * H * D);
        free(rows);
    }
}

/* ------------------------------------------------------------------ */
/* 5. FP4 indexer activations  [DSv4-FP4], [DSv4-MAP]                  */
/* ------------------------------------------------------------------ */
/*
 * Block format (the pages name FP4 activations but not the format; the
 * reading used is e2m1 elements with one e4m3 scale per 16-element block):
 *   e2m1 code: bit 3 sign, magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} for codes 0..7
 *   e4m3 code: bit 7 sign, 4 exponent bits (bias 7), 3 mantissa bits,
 *              subnormals m * 2^-9, code 0x7F / 0xFF = NaN, max 448.
 * Quantisation of a block x_0..x_15:
 *   s = e4m3_RNE_satfinite( fp32(absmax / 6) )
 *   s == 0  -> all 16 codes 0
 *   else    -> q_j = e2m1_RNE_satfinite( fp32(x_j / s) )
 * A code whose magnitude rounds to 0 is stored as +0 (code 0).
 * Packing: byte j/2 holds element 2i in its low nibble, 2i+1 in its high one.
 */
double orc_e2m1_decode(unsigned code)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    const double v = mag[code & 7u];
    return (code & 8u) ? -v : v;
}

double orc_e4m3_decode(unsigned code)
{
    const unsigned e = (code >> 3) & 15u, mt = code & 7u;
    double v;
    if (e == 15u && mt == 7u) return NAN;
    if (e == 0u)
        v = ldexp((double)mt, -9);
    else
        v = ldexp(1.0 + mt / 8.0, (int)e - 7);
    return (code & 0x80u) ? -v : v;
}

/* Nearest representable magnitude by exhaustive search over the finite
 * codes, ties to the code with an even mantissa LSB (round-half-even); values
 * beyond the largest finite magnitude saturate to it. */
unsigned orc_e4m3_encode(float x)
{
    const double a = fabs((double)x);
    unsigned best = 0;
    double best_err = INFINITY;
    for (unsigned c = 0; c <= 0x7Eu; ++c) {
        const double err = fabs(orc_e4m3_decode(c) - a);
        if (err < best_err || (err == best_err && (c & 1u) == 0u)) {
            best = c;
            best_err = err;
        }
    }
    if (best != 0u && x < 0.0f) best |= 0x80u;
    return best;
}

unsigned orc_e2m1_encode(float x)
{
    const double a = fabs((double)x);
    unsigned best = 0;
    double best_err = INFINITY;
    for (unsigned c = 0; c <= 7u; ++c) {
        const double err = fabs(orc_e2m1_decode(c) - a);
        if (err < best_err || (err == best_err && (c & 1u) == 0u)) {
            best = c;
            best_err = err;
        }
    }
    if (best != 0u && x < 0.0f) best |= 8u;
    return best;
}

void orc_quantize_fp4(const uint16_t *x, long long rows, int d, uint8_t *packed, uint8_t *scales)
{
    const int nblk = d / 16;
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; ++r) {
        for (int blk = 0; blk < nblk; ++blk) {
            float xs[16];
            float amax = 0.0f;
            for (int j = 0; j < 16; ++j) {
                xs[j] = (float)bf16_bits_to_double(x[(size_t)r * d + blk * 16 + j]);
                if (fabsf(xs[j]) > amax) amax = fabsf(xs[j]);
            }
            const float s_in = amax / 6.0f; /* IEEE binary32 division */
            const unsigned sc = orc_e4m3_encode(s_in);
            const float s = (float)orc_e4m3_decode(sc);
            scales[(size_t)r * nblk + blk] = (uint8_t)sc;
            for (int j = 0; j < 16; j += 2) {
                unsigned lo = 0, hi = 0;
                if (s != 0.0f) {
                    lo = orc_e2m1_encode(xs[j] / s);     /* IEEE binary32 division */
                    hi = orc_e2m1_encode(xs[j + 1] / s);
                }
                packed[(size_t)r * (d / 2) + blk * 8 + j / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* Dequantised value of element j of a row: e2m1(code) * e4m3(scale of block j/16). */
static double fp4_value(const uint8_t *packed_row, const uint8_t *scale_row, int j)
{
    const unsigned byte = packed_row[j / 2];
    const unsigned code = (j & 1) ? (byte >> 4) : (byte & 15u);
    return orc_e2m1_decode(code) * orc_e4m3_decode(scale_row[j / 16]);
}

void orc_dequantize_fp4(const uint8_t *packed, const uint8_t *scales, long long rows, int d,
                        double *out)
{
    for (long long r = 0; r < rows; ++r)
        for (int j = 0; j < d; ++j)
            out[(size_t)r * d + j] =
                fp4_value(packed + (size_t)r * (d / 2), scales + (size_t)r * (d / 16), j);
}

/* The indexer score of section 2 on dequantised FP4 operands, in float64:
 * q4 [batch][nq][H_I][d_I/2], q4s [batch][nq][H_I][d_I/16],
 * k4 [batch][N][d_I/2],       k4s [batch][N][d_I/16]. */
#define ORC_MAX_DI 1024

int orc_index_fp4(const uint8_t *q4, const uint8_t *q4s, const float *w, const uint8_t *k4,
                   const uint8_t *k4s, const int *q_pos, int batch, int nq, long long N, int H_I,
                   int d_I, int m, double *scores)
{
    const long long total = (long long)batch * nq;
    if (d_I > ORC_MAX_DI || d_I % 16 != 0) return -1;
    double *qd = (double *)malloc(sizeof(double) * (size_t)H_I * d_I);
    for (long long bq = 0; bq < total; ++bq) {
        const long long b = bq / nq;
        const long long nv = n_visible(q_pos[bq], m, N);
        for (int h = 0; h < H_I; ++h)
            for (int j = 0; j < d_I; ++j)
                qd[(size_t)h * d_I + j] =
                    fp4_value(q4 + ((size_t)bq * H_I + h) * (d_I / 2),
                              q4s + ((size_t)bq * H_I + h) * (d_I / 16), j);
        const float *ww = w + (size_t)bq * H_I;
        double *S = scores + (size_t)bq * N;
#pragma omp parallel for schedule(static)
        for (long long s = 0; s < N; ++s) {
            if (s >= nv) {
                S[s] = -INFINITY;
                continue;
            }
            const uint8_t *kr = k4 + ((size_t)b * N + s) * (d_I / 2);
            const uint8_t *ks = k4s + ((size_t)b * N + s) * (d_I / 16);
            double kd[ORC_MAX_DI];
            for (int j = 0; j < d_I; ++j) kd[j] = fp4_value(kr, ks, j);
            double acc = 0.0;
            for (int h = 0; h < H_I; ++h) {
                double dot = 0.0;
                for (int j = 0; j < d_I; ++j) dot += qd[(size_t)h * d_I + j] * kd[j];
                acc += (double)ww[h] * (dot > 0.0 ? dot : 0.0);
            }
            S[s] = acc;
        }
    }
    free(qd);
    return 0;
}

/* ------------------------------------------------------------------ */
/* 6. FP8 KV cache  [DSv4-MAP] list "inference quantization"            */
/* ------------------------------------------------------------------ */
/*
 * The pages list "FP8 KV-cache quantization" and give no format.  Reading:
 * each KV row (a compressed entry or a window row, d channels) is stored as
 * e4m3 codes with one power-of-two scale per block of `block` channels, the
 * scale kept as an unsigned 8-bit exponent (UE8M0: s = 2^(e - 127)).  s is the
 * smallest power of two with absmax(block) / s <= 448 (the largest finite
 * e4m3 magnitude), its exponent k kept in [-124, 119]; the codes are
 * e4m3_RNE(x / s), the division by a power of two being exact; an all-zero
 * block has e = 127 and zero codes.  With s a power of two, 3 mantissa bits
 * per code and k in that range (the smallest code times s is at least bf16's
 * smallest subnormal 2^-133, 448 * s stays below bf16's largest value), every
 * dequantised value code * s is a bf16 number exactly, so attention over the
 * FP8 cache is the attention of section 4 over those bf16 rows.  (Blocks whose
 * absmax exceeds 448 * 2^119 saturate.)
 */
void orc_quantize_fp8_kv(const uint16_t *x, long long rows, int d, int block, uint8_t *codes,
                         uint8_t *exps)
{
    const int nblk = d / block;
    for (long long r = 0; r < rows; ++r) {
        for (int blk = 0; blk < nblk; ++blk) {
            const uint16_t *xs = x + (size_t)r * d + (size_t)blk * block;
            double amax = 0.0;
            for (int j = 0; j < block; ++j) {
                const double a = fabs(bf16_bits_to_double(xs[j]));
                if (a > amax) amax = a;
            }
            int k = 0;  /* s = 2^k */
            if (amax > 0.0) {
                k = (int)ceil(log2(amax / 448.0));
                while (ldexp(amax, -k) > 448.0) ++k;          /* guard the log2 rounding */
                while (ldexp(amax, -(k - 1)) <= 448.0) --k;   /* smallest such k */
                if (k < -124) k = -124;   /* 2^-9 * 2^k stays a bf16 number (>= 2^-133) */
                if (k > 119) k = 119;     /* 448 * 2^k stays finite in bf16 */
            }
            exps[(size_t)r * nblk + blk] = (uint8_t)(k + 127);
            for (int j = 0; j < block; ++j)
                codes[(size_t)r * d + (size_t)blk * block + j] =
                    (uint8_t)orc_e4m3_encode((float)ldexp(bf16_bits_to_double(xs[j]), -k));
        }
    }
}

/* code * 2^(e - 127) per element -> float64 [rows][d] */
void orc_dequantize_fp8_kv(const uint8_t *codes, const uint8_t *exps, long long rows, int d, int block,
                           double *out)
{
    const int nblk = d / block;
    for (long long r = 0; r < rows; ++r)
        for (int j = 0; j < d; ++j)
            out[(size_t)r * d + j] = ldexp(orc_e4m3_decode(codes[(size_t)r * d + j]),
                                           (int)exps[(size_t)r * nblk + j / block] - 127);
}
