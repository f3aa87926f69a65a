/*
 * CPU ORACLE for packed variable-length attention forward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it. It shares no code, header or constant with the
 * CUDA library.
 *
 * What it computes (written out from the definition, slowly and in fp64):
 *
 *   The packed stream holds B sequences back to back. Sequence i owns query
 *   rows [cu_q[i], cu_q[i+1]) and key rows [cu_k[i], cu_k[i+1]), and attends
 *   only to itself (page "pack the GenRec training forward through
 *   FlashAttention-2", opening summary and Test plan: packed stream with
 *   explicit cumulative boundaries, row isolation). Query head h reads
 *   key/value head kvh = floor(h / (Hq / Hkv)) (page "avoid decoding kernel
 *   selection for short GQA", Verification: 32 query heads over 8 K/V heads).
 *   For local query row r and local key c of sequence i:
 *
 *     s(r,c) = scale * sum_d Q[cu_q[i]+r, h, d] * K[cu_k[i]+c, kvh, d]
 *              + bias_key[cu_k[i]+c, h]                       (if given)
 *              + bias_pair[i*sb + h*sh + r*sr + c*sc]          (if given)
 *
 *   Per-key bias and the per-pair grid addressed per sequence through its
 *   leading stride: GiGL pull request 858, Approach. The bias is added after
 *   scaling, as SDPA does with a float mask; SDPA is the reference that page
 *   tests against (Verification).
 *
 *   visible(r,c) = !causal || c <= r + (Lk - Lq)      (bottom-right causal;
 *   with q_len = 1 it is the same as non-causal, which the page "Integrate
 *   Flash Dynamic Mask Attention (FDMA) Into Transformers-Style Attention
 *   Flow", Key Implementation Points, Causality Handling, relies on.)
 *
 *   LSE(r) = log sum_{visible c} exp(s(r,c))           natural log
 *   O(r,:) = sum_{visible c} exp(s(r,c) - LSE(r)) * V[cu_k[i]+c, kvh, :]
 *
 *   A row with no visible key, or whose visible scores are all -inf, has an
 *   empty softmax: LSE = -inf and O = 0 (reading of a case the pages leave
 *   open; never NaN).
 *
 * The max-subtraction inside the sum is the usual exact rewrite
 * log sum exp(s) = m + log sum exp(s - m) and changes nothing but rounding.
 *
 * Element types: Q/K/V may be given as bf16 bit patterns (uint16), fp32 or
 * fp64; biases as fp32 or fp64. Every value is widened exactly to double.
 * Outputs are fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_BF16 = 0, ORACLE_F32 = 1, ORACLE_F64 = 2 };

/* Widen one element to double. bf16 is the upper half of an IEEE fp32. */
static double load_elem(const void* base, int64_t idx, int dtype) {
  if (dtype == ORACLE_BF16) {
    uint32_t bits = ((uint32_t)((const uint16_t*)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  if (dtype == ORACLE_F32) return (double)((const float*)base)[idx];
  return ((const double*)base)[idx];
}

typedef struct {
  const void *q, *k, *v;
  int qkv_dtype;
  const int32_t *cu_q, *cu_k;
  int batch, n_heads, n_kv_heads, head_dim;
  double scale;
  int causal;
  const void* bias_key; /* [Tk, Hq] or NULL */
  const void* bias_pair; /* strided grid or NULL */
  int bias_dtype;
  int64_t sb, sh, sr, sc;
} problem_t;

/* Score s(r,c) of the definition, for sequence i, head h. */
static double score(const problem_t* p, int i, int h, int r, int c) {
  const int G = p->n_heads / p->n_kv_heads;
  const int kvh = h / G;
  const int D = p->head_dim;
  const int64_t qrow = (int64_t)p->cu_q[i] + r;
  const int64_t krow = (int64_t)p->cu_k[i] + c;
  double dot = 0.0;
  for (int d = 0; d < D; ++d) {
    double qv = load_elem(p->q, (qrow * p->n_heads + h) * D + d, p->qkv_dtype);
    double kv = load_elem(p->k, (krow * p->n_kv_heads + kvh) * D + d, p->qkv_dtype);
    dot += qv * kv;
  }
  double s = p->scale * dot;
  if (p->bias_key) s += load_elem(p->bias_key, krow * p->n_heads + h, p->bias_dtype);
  if (p->bias_pair)
    s += load_elem(p->bias_pair,
                   (int64_t)i * p->sb + (int64_t)h * p->sh + (int64_t)r * p->sr + (int64_t)c * p->sc,
                   p->bias_dtype);
  return s;
}

static int is_visible(const problem_t* p, int i, int r, int c) {
  const int Lq = p->cu_q[i + 1] - p->cu_q[i];
  const int Lk = p->cu_k[i + 1] - p->cu_k[i];
  return !p->causal || c <= r + (Lk - Lq);
}

/* One output row: O(r,:) into out_row[0..D), LSE into *lse_out.
 * scratch holds at least Lk doubles. */
static void attention_row(const problem_t* p, int i, int h, int r, double* scratch,
                          double* out_row, double* lse_out) {
  const int Lk = p->cu_k[i + 1] - p->cu_k[i];
  const int G = p->n_heads / p->n_kv_heads;
  const int kvh = h / G;
  const int D = p->head_dim;
  double m = -INFINITY;
  for (int c = 0; c < Lk; ++c) {
    if (!is_visible(p, i, r, c)) continue;
    scratch[c] = score(p, i, h, r, c);
    if (scratch[c] > m) m = scratch[c];
  }
  for (int d = 0; d < D; ++d) out_row[d] = 0.0;
  if (m == -INFINITY) { /* empty softmax */
    *lse_out = -INFINITY;
    return;
  }
  double sum = 0.0;
  for (int c = 0; c < Lk; ++c)
    if (is_visible(p, i, r, c)) sum += exp(scratch[c] - m);
  const double lse = m + log(sum);
  for (int c = 0; c < Lk; ++c) {
    if (!is_visible(p, i, r, c)) continue;
    const double w = exp(scratch[c] - lse);
    const int64_t krow = (int64_t)p->cu_k[i] + c;
    for (int d = 0; d < D; ++d)
      out_row[d] += w * load_elem(p->v, (krow * p->n_kv_heads + kvh) * D + d, p->qkv_dtype);
  }
  *lse_out = lse;
}

static int check_problem(const problem_t* p) {
  if (p->batch < 0 || p->n_heads <= 0 || p->n_kv_heads <= 0 || p->head_dim <= 0) return 1;
  if (p->n_heads % p->n_kv_heads != 0) return 2;
  if (p->cu_q[0] != 0 || p->cu_k[0] != 0) return 3;
  for (int i = 0; i < p->batch; ++i)
    if (p->cu_q[i + 1] < p->cu_q[i] || p->cu_k[i + 1] < p->cu_k[i]) return 3;
  return 0;
}

static int max_key_len(const problem_t* p) {
  int mx = 0;
  for (int i = 0; i < p->batch; ++i) {
    int L = p->cu_k[i + 1] - p->cu_k[i];
    if (L > mx) mx = L;
  }
  return mx;
}

/* Full forward. out: [Tq, Hq, D] fp64; lse: [Hq, Tq] fp64 with Tq = cu_q[B].
 * Returns 0, or a positive code for malformed arguments. */
int oracle_varlen_attn_fwd(const void* q, const void* k, const void* v, int qkv_dtype,
                           const int32_t* cu_q, const int32_t* cu_k, int batch, int n_heads,
                           int n_kv_heads, int head_dim, double scale, int causal,
                           const void* bias_key, const void* bias_pair, int bias_dtype, int64_t sb,
                           int64_t sh, int64_t sr, int64_t sc, double* out, double* lse,
                           int n_threads) {
  problem_t p = {q, k, v, qkv_dtype, cu_q, cu_k, batch, n_heads, n_kv_heads, head_dim,
                 scale, causal, bias_key, bias_pair, bias_dtype, sb, sh, sr, sc};
  int err = check_problem(&p);
  if (err) return err;
  const int64_t Tq = cu_q[batch];
  const int maxLk = max_key_len(&p);
  const int D = head_dim;
  (void)n_threads;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
  {
    double* scratch = (double*)malloc(sizeof(double) * (size_t)(maxLk > 0 ? maxLk : 1));
#pragma omp for collapse(2) schedule(dynamic, 1)
    for (int i = 0; i < batch; ++i) {
      for (int h = 0; h < n_heads; ++h) {
        const int Lq = cu_q[i + 1] - cu_q[i];
        for (int r = 0; r < Lq; ++r) {
          const int64_t row = (int64_t)cu_q[i] + r;
          attention_row(&p, i, h, r, scratch, out + (row * n_heads + h) * D,
                        lse + (int64_t)h * Tq + row);
        }
      }
    }
    free(scratch);
  }
  return 0;
}

/* Selected rows only: for each sample n, sequence seq[n], head head[n], local
 * query row row[n]; writes out_rows[n*D .. n*D+D) and lse_rows[n]. */
int oracle_varlen_attn_rows(const void* q, const void* k, const void* v, int qkv_dtype,
                            const int32_t* cu_q, const int32_t* cu_k, int batch, int n_heads,
                            int n_kv_heads, int head_dim, double scale, int causal,
                            const void* bias_key, const void* bias_pair, int bias_dtype,
                            int64_t sb, int64_t sh, int64_t sr, int64_t sc, int64_t n_samples,
                            const int32_t* seq, const int32_t* head, const int32_t* row,
                            double* out_rows, double* lse_rows, int n_threads) {
  problem_t p = {q, k, v, qkv_dtype, cu_q, cu_k, batch, n_heads, n_kv_heads, head_dim,
                 scale, causal, bias_key, bias_pair, bias_dtype, sb, sh, sr, sc};
  int err = check_problem(&p);
  if (err) return err;
  for (int64_t n = 0; n < n_samples; ++n) {
    if (seq[n] < 0 || seq[n] >= batch || head[n] < 0 || head[n] >= n_heads) return 4;
    if (row[n] < 0 || row[n] >= cu_q[seq[n] + 1] - cu_q[seq[n]]) return 4;
  }
  const int maxLk = max_key_len(&p);
  (void)n_threads;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
  {
    double* scratch = (double*)malloc(sizeof(double) * (size_t)(maxLk > 0 ? maxLk : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t n = 0; n < n_samples; ++n)
      attention_row(&p, seq[n], head[n], row[n], scratch, out_rows + n * head_dim, lse_rows + n);
    free(scratch);
  }
  return 0;
}

/* Softmax probabilities of one (sequence, head): probs[r*Lk + c] =
 * exp(s(r,c) - LSE(r)) for visible c, else 0. For small inputs only. */
int oracle_varlen_attn_probs(const void* q, const void* k, const void* v, int qkv_dtype,
                             const int32_t* cu_q, const int32_t* cu_k, int batch, int n_heads,
                             int n_kv_heads, int head_dim, double scale, int causal,
                             const void* bias_key, const void* bias_pair, int bias_dtype,
                             int64_t sb, int64_t sh, int64_t sr, int64_t sc, int i, int h,
                             double* probs) {
  problem_t p = {q, k, v, qkv_dtype, cu_q, cu_k, batch, n_heads, n_kv_heads, head_dim,
                 scale, causal, bias_key, bias_pair, bias_dtype, sb, sh, sr, sc};
  int err = check_problem(&p);
  if (err) return err;
  if (i < 0 || i >= batch || h < 0 || h >= n_heads) return 4;
  const int Lq = cu_q[i + 1] - cu_q[i];
  const int Lk = cu_k[i + 1] - cu_k[i];
  double* scratch = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
  double* orow = (double*)malloc(sizeof(double) * (size_t)head_dim);
  for (int r = 0; r < Lq; ++r) {
    double lse;
    attention_row(&p, i, h, r, scratch, orow, &lse);
    for (int c = 0; c < Lk; ++c) {
      double w = 0.0;
      if (lse != -INFINITY && is_visible(&p, i, r, c)) w = exp(score(&p, i, h, r, c) - lse);
      probs[(int64_t)r * Lk + c] = w;
    }
  }
  free(scratch);
  free(orow);
  return 0;
}
