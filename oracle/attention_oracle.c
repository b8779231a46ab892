/*
 * attention_oracle.c -- plain, slow, fp64 CPU oracle for exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * with the CUDA library, and it does not include any of the library's files.
 *
 * Source cited throughout as [MM]: the marketmaker.cc blog post (Indonesian
 * edition) "Apakah Konteks Sehari Penuh Mengalahkan Konteks Sepuluh Menit?
 * Perhatian Kilat dan Pertanyaan Panjang Urutan", cited by section heading.
 *
 * What it computes ([MM] "Mengapa perhatian terikat pada memori" and the
 * explicit three-line PyTorch path in "Integrasinya delapan baris"):
 *
 *     S = scale * Q K^T          (scale = 1/sqrt(d_k) in every workload)
 *     S[i, j] = -inf  if causal and key j lies in the future of query i (j > i)
 *     O = softmax_rows(S) V
 *     lse[i] = log(sum_j exp(S[i, j]))     -- natural log over the scaled,
 *                                             masked scores; this is the
 *                                             (m, l) pair that section
 *                                             "Backward pass" says is kept,
 *                                             folded into one number m + ln l.
 *
 * The softmax is the plain two-pass, max-subtracted form (pass 1 finds the
 * row maximum m, pass 2 sums exp(s - m)); the score row is materialised in
 * full before either pass.  All arithmetic is IEEE double via libm exp/log,
 * summed in ascending key order.  Build without -ffast-math.
 *
 * A second, deliberately different implementation follows the blocked
 * algorithm of [MM] "Algoritma Flash Attention" step by step (per-block local
 * max and sum, running statistics, output rescaled and renormalised at every
 * block).  It exists only so that the two-pass oracle can be cross-checked
 * against the pages' own algorithm; it calls none of the two-pass helpers.
 *
 * The backward pass ([MM] "Backward pass: menghitung ulang, bukan
 * menyimpan") is the gradient of the same definition, written out from the
 * calculus (the pages give no formulas): for an upstream gradient dO,
 *     dV = P^T dO,   dP = dO V^T,   D_i = sum_j P_ij dP_ij,
 *     dS = P * (dP - D) (elementwise, D broadcast along the row),
 *     dQ = scale * dS K,   dK = scale * dS^T Q.
 * Masked entries have P = 0 and so dS = 0.  The oracle recomputes P from
 * the scores with its own two-pass softmax, exactly as the forward does.
 *
 * Decode (few new queries against a long key/value sequence; the
 * briefgpt.xyz summary page of FlashAttention-2, arXiv 2307.08691, entry
 * "LeanAttention": the decode phase of long contexts): the queries are
 * the last Nq positions of an Nk-long sequence, so with the causal mask
 * query i sees keys 0 .. Nk - Nq + i.  Same definition otherwise.
 *
 * Layout conventions: Q, K, V, O are contiguous row-major [B, H, N, d];
 * lse is contiguous [B, H, N].  bf16 inputs are passed as their raw 16-bit
 * patterns and widened exactly to double (bf16 -> fp32 is exact, fp32 ->
 * fp64 is exact).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EBADARG 1
#define ORACLE_ENOMEM 2

/* Exact widening of a bfloat16 bit pattern: the pattern is the top half of
 * an IEEE binary32 value. */
static double bf16_bits_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Number of keys visible to query i: all N keys, or keys 0..i when causal
 * ([MM] "Causal masking adalah tempat perdagangan mendapat diskon": a query
 * may not attend to the future; the explicit path masks with -inf, so key i
 * itself stays visible). */
static int64_t visible_keys(int64_t i, int64_t N, int causal) {
  return causal ? (i + 1) : N;
}

/* The softmax-and-weighted-sum step on one materialised score row.
 * s[0..n) are finite scores of the visible keys; V points at n rows of d.
 * Writes o[0..d) and *lse.  p (n doubles, may be NULL) receives the softmax
 * probabilities when the caller wants to inspect them. */
static void attend_row(const double *s, int64_t n, const double *V, int64_t d,
                       double *o, double *lse, double *p) {
  /* pass 1: row maximum */
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j)
    if (s[j] > m) m = s[j];
  /* pass 2: exponentials and their sum */
  double l = 0.0;
  for (int64_t t = 0; t < d; ++t) o[t] = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    double e = exp(s[j] - m);
    l += e;
    for (int64_t t = 0; t < d; ++t) o[t] += e * V[j * d + t];
  }
  for (int64_t t = 0; t < d; ++t) o[t] /= l;
  *lse = m + log(l);
  if (p)
    for (int64_t j = 0; j < n; ++j) p[j] = exp(s[j] - m) / l;
}

/* ------------------------------------------------------------------------ */
/* Public entry points (ctypes).                                            */
/* ------------------------------------------------------------------------ */

/* Softmax of one score row; the pin "every row of probabilities sums to 1"
 * reads this.  No values are involved: the value width passed down is 0. */
int oracle_softmax_row(const double *s, int64_t n, double *p) {
  if (!s || !p || n < 1) return ORACLE_EBADARG;
  double v_dummy = 0.0, o_dummy = 0.0, lse = 0.0;
  attend_row(s, n, &v_dummy, 0, &o_dummy, &lse, p);
  return ORACLE_OK;
}

/* Attention given an already-materialised score matrix S [rows, n_keys] and
 * V [n_keys, d]: O[rows, d] = softmax_rows(S) V, lse[rows].  Entries of S
 * equal to -inf are masked keys and are dropped before the two passes. */
int oracle_attend_scores(const double *S, const double *V, int64_t rows,
                         int64_t n_keys, int64_t d, double *O, double *lse) {
  if (!S || !V || !O || !lse || rows < 0 || n_keys < 1 || d < 1)
    return ORACLE_EBADARG;
  double *s = (double *)malloc(sizeof(double) * (size_t)n_keys);
  double *vv = (double *)malloc(sizeof(double) * (size_t)(n_keys * d));
  if (!s || !vv) { free(s); free(vv); return ORACLE_ENOMEM; }
  for (int64_t i = 0; i < rows; ++i) {
    int64_t n = 0;
    for (int64_t j = 0; j < n_keys; ++j) {
      double x = S[i * n_keys + j];
      if (x == -INFINITY) continue;
      s[n] = x;
      memcpy(vv + n * d, V + j * d, sizeof(double) * (size_t)d);
      ++n;
    }
    if (n == 0) { free(s); free(vv); return ORACLE_EBADARG; }
    attend_row(s, n, vv, d, O + i * d, lse + i, NULL);
  }
  free(s);
  free(vv);
  return ORACLE_OK;
}

/* Full attention over fp64 inputs: the definition, one (b, h, i) row at a
 * time.  For each row the whole score row is materialised, then the two
 * softmax passes run over it.  OpenMP parallel over rows. */
int oracle_attention_f64(const double *Q, const double *K, const double *V,
                         double *O, double *lse, int64_t B, int64_t H,
                         int64_t N, int64_t d, int causal, double scale,
                         int nthreads) {
  if (!Q || !K || !V || !O || !lse || B < 0 || H < 0 || N < 0 || d < 1)
    return ORACLE_EBADARG;
  const int64_t rows = B * H * N;
  if (rows == 0) return ORACLE_OK;
  int err = ORACLE_OK;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    if (!s) {
#pragma omp atomic write
      err = ORACLE_ENOMEM;
    }
#pragma omp for schedule(dynamic, 16)
    for (int64_t r = 0; r < rows; ++r) {
      if (!s) continue;
      const int64_t bh = r / N, i = r % N;
      const double *Kh = K + bh * N * d, *Vh = V + bh * N * d;
      const double *qi = Q + r * d;
      const int64_t n = visible_keys(i, N, causal);
      for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t t = 0; t < d; ++t) acc += qi[t] * Kh[j * d + t];
        s[j] = scale * acc;
      }
      attend_row(s, n, Vh, d, O + r * d, lse + r, NULL);
    }
    free(s);
  }
  return err;
}

/* ------------------------------------------------------------------------ */
/* Decode: few queries against a long key/value sequence.                   */
/* ------------------------------------------------------------------------ */

/* Keys visible to query i of Nq new queries appended to a sequence whose
 * keys are 0..Nk-1 (the queries are the last Nq positions, Nq <= Nk):
 * query i sits at position Nk - Nq + i and, with the causal mask, sees keys
 * 0 .. Nk - Nq + i ([MM] "Causal masking ...": no key in a query's future;
 * the "bottom-right" alignment, the only one under which the new tokens are
 * the latest positions).  Without the mask every key is visible. */
static int64_t decode_visible_keys(int64_t i, int64_t Nq, int64_t Nk, int causal) {
  return causal ? (Nk - Nq + i + 1) : Nk;
}

/* Decode attention over fp64 inputs: Q [BH, Nq, d], K and V [BH, Nk, d],
 * O [BH, Nq, d], lse [BH, Nq]; the same definition as oracle_attention_f64
 * (whole score row, two softmax passes) with the visibility rule above.
 * OpenMP over rows. */
int oracle_attention_decode_f64(const double *Q, const double *K,
                                const double *V, double *O, double *lse,
                                int64_t BH, int64_t Nq, int64_t Nk, int64_t d,
                                int causal, double scale, int nthreads) {
  if (!Q || !K || !V || !O || !lse || BH < 0 || Nq < 0 || Nk < 1 || d < 1 ||
      (causal && Nq > Nk))
    return ORACLE_EBADARG;
  const int64_t rows = BH * Nq;
  if (rows == 0) return ORACLE_OK;
  int err = ORACLE_OK;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)Nk);
    if (!s) {
#pragma omp atomic write
      err = ORACLE_ENOMEM;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
      if (!s) continue;
      const int64_t bh = r / Nq, i = r % Nq;
      const double *Kh = K + bh * Nk * d, *Vh = V + bh * Nk * d;
      const double *qi = Q + r * d;
      const int64_t n = decode_visible_keys(i, Nq, Nk, causal);
      for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t t = 0; t < d; ++t) acc += qi[t] * Kh[j * d + t];
        s[j] = scale * acc;
      }
      attend_row(s, n, Vh, d, O + r * d, lse + r, NULL);
    }
    free(s);
  }
  return err;
}

/* The same on bf16 bit patterns for selected rows (flat index bh * Nq + i),
 * widening key and value rows on the fly (full-size checks without an fp64
 * copy of the key/value sequence).  O_out [nrows, d], lse_out [nrows]. */
int oracle_attention_decode_rows_bf16(const uint16_t *Q, const uint16_t *K,
                                      const uint16_t *V, int64_t BH, int64_t Nq,
                                      int64_t Nk, int64_t d, int causal,
                                      double scale, const int64_t *rows,
                                      int64_t nrows, double *O_out,
                                      double *lse_out, int nthreads) {
  if (!Q || !K || !V || !rows || !O_out || !lse_out || BH < 1 || Nq < 1 ||
      Nk < 1 || d < 1 || (causal && Nq > Nk))
    return ORACLE_EBADARG;
  for (int64_t k = 0; k < nrows; ++k)
    if (rows[k] < 0 || rows[k] >= BH * Nq) return ORACLE_EBADARG;
  int err = ORACLE_OK;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)Nk);
    double *vv = (double *)malloc(sizeof(double) * (size_t)(Nk * d));
    double *qi = (double *)malloc(sizeof(double) * (size_t)d);
    if (!s || !vv || !qi) {
#pragma omp atomic write
      err = ORACLE_ENOMEM;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t k = 0; k < nrows; ++k) {
      if (!s || !vv || !qi) continue;
      const int64_t r = rows[k], bh = r / Nq, i = r % Nq;
      const uint16_t *Kh = K + bh * Nk * d, *Vh = V + bh * Nk * d;
      for (int64_t t = 0; t < d; ++t) qi[t] = bf16_bits_to_double(Q[r * d + t]);
      const int64_t n = decode_visible_keys(i, Nq, Nk, causal);
      for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t t = 0; t < d; ++t)
          acc += qi[t] * bf16_bits_to_double(Kh[j * d + t]);
        s[j] = scale * acc;
        for (int64_t t = 0; t < d; ++t) vv[j * d + t] = bf16_bits_to_double(Vh[j * d + t]);
      }
      attend_row(s, n, vv, d, O_out + k * d, lse_out + k, NULL);
    }
    free(s); free(vv); free(qi);
  }
  return err;
}

/* Attention on selected rows of bf16 inputs (raw bit patterns).  rows[k] is
 * a flat row index bh * N + i; O_out is [nrows, d] fp64, lse_out [nrows].
 * The key and value rows a query needs are widened to fp64 on the fly, so
 * full-size workloads can be checked row by row without an fp64 copy. */
int oracle_attention_rows_bf16(const uint16_t *Q, const uint16_t *K,
                               const uint16_t *V, int64_t B, int64_t H,
                               int64_t N, int64_t d, int causal, double scale,
                               const int64_t *rows, int64_t nrows,
                               double *O_out, double *lse_out, int nthreads) {
  if (!Q || !K || !V || !rows || !O_out || !lse_out || B < 0 || H < 0 ||
      N < 1 || d < 1 || nrows < 0)
    return ORACLE_EBADARG;
  for (int64_t k = 0; k < nrows; ++k)
    if (rows[k] < 0 || rows[k] >= B * H * N) return ORACLE_EBADARG;
  int err = ORACLE_OK;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *qi = (double *)malloc(sizeof(double) * (size_t)d);
    double *vv = (double *)malloc(sizeof(double) * (size_t)(N * d));
    if (!s || !qi || !vv) {
#pragma omp atomic write
      err = ORACLE_ENOMEM;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t k = 0; k < nrows; ++k) {
      if (!s || !qi || !vv) continue;
      const int64_t r = rows[k];
      const int64_t bh = r / N, i = r % N;
      const uint16_t *Kh = K + bh * N * d, *Vh = V + bh * N * d;
      for (int64_t t = 0; t < d; ++t) qi[t] = bf16_bits_to_double(Q[r * d + t]);
      const int64_t n = visible_keys(i, N, causal);
      for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t t = 0; t < d; ++t)
          acc += qi[t] * bf16_bits_to_double(Kh[j * d + t]);
        s[j] = scale * acc;
        for (int64_t t = 0; t < d; ++t)
          vv[j * d + t] = bf16_bits_to_double(Vh[j * d + t]);
      }
      attend_row(s, n, vv, d, O_out + k * d, lse_out + k, NULL);
    }
    free(s);
    free(qi);
    free(vv);
  }
  return err;
}

/* ------------------------------------------------------------------------ */
/* Block-sparse attention.                                                  */
/* ------------------------------------------------------------------------ */

/* The block-sparse extension of the tiled method (briefgpt.xyz summary page
 * of FlashAttention-2, arXiv 2307.08691, FlashAttention entry): scores of
 * the (query block, key block) pairs a mask leaves out are -inf, so those
 * keys drop out of the row; the rest is the definition above.  Blocks are
 * 128 rows of queries by 128 keys; mask is row-major [T, T] bytes, T =
 * ceil(N / 128), nonzero = kept; one mask for every head (mask_per_head = 0)
 * or one per head in [B, H] order.  With the causal mask, key j > i is also
 * dropped.  A row with no key left has no softmax; the reading taken is
 * O = 0 and lse = -inf.  Selected rows (flat bh * N + i) of bf16 bit
 * patterns, widened exactly, as in oracle_attention_rows_bf16. */
int oracle_attention_block_sparse_rows_bf16(
    const uint16_t *Q, const uint16_t *K, const uint16_t *V, int64_t B,
    int64_t H, int64_t N, int64_t d, int causal, double scale,
    const uint8_t *mask, int mask_per_head, const int64_t *rows, int64_t nrows,
    double *O_out, double *lse_out, int nthreads) {
  if (!Q || !K || !V || !mask || !rows || !O_out || !lse_out || B < 0 ||
      H < 0 || N < 1 || d < 1 || nrows < 0)
    return ORACLE_EBADARG;
  for (int64_t a = 0; a < nrows; ++a)
    if (rows[a] < 0 || rows[a] >= B * H * N) return ORACLE_EBADARG;
  const int64_t T = (N + 127) / 128;
  int err = ORACLE_OK;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *qi = (double *)malloc(sizeof(double) * (size_t)d);
    double *vv = (double *)malloc(sizeof(double) * (size_t)(N * d));
    if (!s || !qi || !vv) {
#pragma omp atomic write
      err = ORACLE_ENOMEM;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t a = 0; a < nrows; ++a) {
      if (!s || !qi || !vv) continue;
      const int64_t r = rows[a], bh = r / N, i = r % N;
      const uint16_t *Kh = K + bh * N * d, *Vh = V + bh * N * d;
      const uint8_t *mrow = mask + (mask_per_head ? bh * T * T : 0) + (i / 128) * T;
      for (int64_t t = 0; t < d; ++t) qi[t] = bf16_bits_to_double(Q[r * d + t]);
      /* the kept keys of row i, in ascending order */
      int64_t n = 0;
      const int64_t jend = visible_keys(i, N, causal);
      for (int64_t j = 0; j < jend; ++j) {
        if (mrow[j / 128] == 0) continue;
        double acc = 0.0;
        for (int64_t t = 0; t < d; ++t)
          acc += qi[t] * bf16_bits_to_double(Kh[j * d + t]);
        s[n] = scale * acc;
        for (int64_t t = 0; t < d; ++t)
          vv[n * d + t] = bf16_bits_to_double(Vh[j * d + t]);
        ++n;
      }
      if (n == 0) {
        for (int64_t t = 0; t < d; ++t) O_out[a * d + t] = 0.0;
        lse_out[a] = -INFINITY;
        continue;
      }
      attend_row(s, n, vv, d, O_out + a * d, lse_out + a, NULL);
    }
    free(s);
    free(qi);
    free(vv);
  }
  return err;
}

/* ------------------------------------------------------------------------ */
/* The pages' blocked algorithm, as a second opinion on the oracle.         */
/* ------------------------------------------------------------------------ */

/* [MM] "Algoritma Flash Attention": Q is cut into blocks of Br rows and K, V
 * into blocks of Bc rows.  For every query block the output O_i starts at 0,
 * the running maximum m_i at -inf and the running sum l_i at 0.  For every
 * key/value block: form the block of scores, take its row maximum m_ij,
 * exponentiate against that local maximum to get P_ij, take its row sum
 * l_ij, then merge into the running statistics with
 *     m_new = max(m_i, m_ij)
 *     l_new = l_i e^(m_i - m_new) + l_ij e^(m_ij - m_new)
 * and replace O_i by the renormalised mix of the old output (weight
 * l_i e^(m_i - m_new) / l_new) and P_ij V_j (weight e^(m_ij - m_new) / l_new).
 * [MM] "Pengulangan softmax online" says this equals the two-pass softmax in
 * exact arithmetic.  lse is m_i + ln l_i after the last block.
 *
 * Reading where the pages are silent: with a causal mask a row of a block
 * can be entirely masked (all keys in its future).  Such a row has no local
 * maximum; it contributes nothing and its running statistics are left as
 * they were.  Blocks whose keys all lie in every query's future are skipped
 * outright ([MM] "Causal masking ...").  Works on fp64 inputs. */
int oracle_attention_blocked_f64(const double *Q, const double *K,
                                 const double *V, double *O, double *lse,
                                 int64_t B, int64_t H, int64_t N, int64_t d,
                                 int causal, double scale, int64_t Br,
                                 int64_t Bc) {
  if (!Q || !K || !V || !O || !lse || B < 0 || H < 0 || N < 0 || d < 1 ||
      Br < 1 || Bc < 1)
    return ORACLE_EBADARG;
  double *Sij = (double *)malloc(sizeof(double) * (size_t)(Br * Bc));
  double *PV = (double *)malloc(sizeof(double) * (size_t)(Br * d));
  double *mi = (double *)malloc(sizeof(double) * (size_t)Br);
  double *li = (double *)malloc(sizeof(double) * (size_t)Br);
  if (!Sij || !PV || !mi || !li) {
    free(Sij); free(PV); free(mi); free(li);
    return ORACLE_ENOMEM;
  }
  for (int64_t bh = 0; bh < B * H; ++bh) {
    const double *Qh = Q + bh * N * d, *Kh = K + bh * N * d,
                 *Vh = V + bh * N * d;
    double *Oh = O + bh * N * d, *lh = lse + bh * N;
    for (int64_t q0 = 0; q0 < N; q0 += Br) {
      const int64_t nr = (N - q0 < Br) ? (N - q0) : Br;
      for (int64_t r = 0; r < nr; ++r) {
        mi[r] = -INFINITY;
        li[r] = 0.0;
        for (int64_t t = 0; t < d; ++t) Oh[(q0 + r) * d + t] = 0.0;
      }
      for (int64_t k0 = 0; k0 < N; k0 += Bc) {
        if (causal && k0 > q0 + nr - 1) break; /* whole block in the future */
        const int64_t nc = (N - k0 < Bc) ? (N - k0) : Bc;
        /* S_ij = Q_i K_j^T * scale, masked */
        for (int64_t r = 0; r < nr; ++r)
          for (int64_t c = 0; c < nc; ++c) {
            double acc = 0.0;
            for (int64_t t = 0; t < d; ++t)
              acc += Qh[(q0 + r) * d + t] * Kh[(k0 + c) * d + t];
            Sij[r * Bc + c] =
                (causal && k0 + c > q0 + r) ? -INFINITY : scale * acc;
          }
        for (int64_t r = 0; r < nr; ++r) {
          /* m_ij = rowmax(S_ij) */
          double mij = -INFINITY;
          for (int64_t c = 0; c < nc; ++c)
            if (Sij[r * Bc + c] > mij) mij = Sij[r * Bc + c];
          if (mij == -INFINITY) continue; /* row fully masked in this block */
          /* P_ij = exp(S_ij - m_ij), l_ij = rowsum(P_ij), (P_ij V_j) */
          double lij = 0.0;
          for (int64_t t = 0; t < d; ++t) PV[r * d + t] = 0.0;
          for (int64_t c = 0; c < nc; ++c) {
            double pc = exp(Sij[r * Bc + c] - mij);
            lij += pc;
            for (int64_t t = 0; t < d; ++t) PV[r * d + t] += pc * Vh[(k0 + c) * d + t];
          }
          /* merge into the running statistics */
          const double mnew = (mi[r] > mij) ? mi[r] : mij;
          const double wold = li[r] * exp(mi[r] - mnew); /* 0 when li = 0 */
          const double wnew = exp(mij - mnew);
          const double lnew = wold + lij * wnew;
          double *orow = Oh + (q0 + r) * d;
          for (int64_t t = 0; t < d; ++t)
            orow[t] = orow[t] * (wold / lnew) + PV[r * d + t] * (wnew / lnew);
          mi[r] = mnew;
          li[r] = lnew;
        }
      }
      for (int64_t r = 0; r < nr; ++r) lh[q0 + r] = mi[r] + log(li[r]);
    }
  }
  free(Sij); free(PV); free(mi); free(li);
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Backward pass.                                                           */
/* ------------------------------------------------------------------------ */

/* Gradients of the attention forward for one (b, h) head: Q, K, V, dO are
 * [N, d]; dQ, dK, dV are [N, d] outputs.  P is materialised row by row with
 * the two-pass softmax; dK and dV accumulate over the rows of the head in
 * ascending row order. */
static int backward_head(const double *Q, const double *K, const double *V,
                         const double *dO, double *dQ, double *dK, double *dV,
                         int64_t N, int64_t d, int causal, double scale) {
  double *s = (double *)malloc(sizeof(double) * (size_t)N);
  double *pr = (double *)malloc(sizeof(double) * (size_t)N);
  double *dp = (double *)malloc(sizeof(double) * (size_t)N);
  if (!s || !pr || !dp) { free(s); free(pr); free(dp); return ORACLE_ENOMEM; }
  for (int64_t x = 0; x < N * d; ++x) { dQ[x] = 0.0; dK[x] = 0.0; dV[x] = 0.0; }
  for (int64_t i = 0; i < N; ++i) {
    const int64_t n = visible_keys(i, N, causal);
    const double *qi = Q + i * d, *doi = dO + i * d;
    /* scores and probabilities of row i */
    for (int64_t j = 0; j < n; ++j) {
      double acc = 0.0;
      for (int64_t t = 0; t < d; ++t) acc += qi[t] * K[j * d + t];
      s[j] = scale * acc;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) if (s[j] > m) m = s[j];
    double l = 0.0;
    for (int64_t j = 0; j < n; ++j) { pr[j] = exp(s[j] - m); l += pr[j]; }
    for (int64_t j = 0; j < n; ++j) pr[j] /= l;
    /* dP_ij = dO_i . V_j ; D_i = sum_j P_ij dP_ij */
    double Di = 0.0;
    for (int64_t j = 0; j < n; ++j) {
      double acc = 0.0;
      for (int64_t t = 0; t < d; ++t) acc += doi[t] * V[j * d + t];
      dp[j] = acc;
      Di += pr[j] * acc;
    }
    for (int64_t j = 0; j < n; ++j) {
      const double dsij = pr[j] * (dp[j] - Di);
      for (int64_t t = 0; t < d; ++t) {
        dV[j * d + t] += pr[j] * doi[t];
        dQ[i * d + t] += scale * dsij * K[j * d + t];
        dK[j * d + t] += scale * dsij * qi[t];
      }
    }
  }
  free(s); free(pr); free(dp);
  return ORACLE_OK;
}

/* Backward of the attention forward over fp64 [B, H, N, d] inputs.  OpenMP
 * parallel over heads (each head's dK, dV sum over all of its rows). */
int oracle_attention_backward_f64(const double *Q, const double *K,
                                  const double *V, const double *dO,
                                  double *dQ, double *dK, double *dV,
                                  int64_t B, int64_t H, int64_t N, int64_t d,
                                  int causal, double scale, int nthreads) {
  if (!Q || !K || !V || !dO || !dQ || !dK || !dV || B < 0 || H < 0 ||
      N < 0 || d < 1)
    return ORACLE_EBADARG;
  const int64_t heads = B * H;
  int err = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
  for (int64_t h = 0; h < heads; ++h) {
    const int64_t off = h * N * d;
    int rc = backward_head(Q + off, K + off, V + off, dO + off, dQ + off,
                           dK + off, dV + off, N, d, causal, scale);
    if (rc != ORACLE_OK) {
#pragma omp atomic write
      err = rc;
    }
  }
  return err;
}

/* Threads OpenMP would use by default (for reporting). */
/* Backward on sampled rows of ONE head of bf16 inputs (raw bit patterns,
 * Q, K, V, dO each [N, d]): dQ for query rows qrows[0..nq) and dK, dV for
 * key rows krows[0..nk), the same formulas as oracle_attention_backward_f64.
 * Every row's lse and D_i = sum_t dO_it O_it come first (the whole forward of
 * the head, O(N^2 d)); then each sampled query row needs its score row, and
 * each sampled key row one column of P and dS over all queries.  For the
 * full-size checks, where the full backward would take too long. */
int oracle_attention_backward_rows_bf16(
    const uint16_t *Qb, const uint16_t *Kb, const uint16_t *Vb,
    const uint16_t *dOb, int64_t N, int64_t d, int causal, double scale,
    const int64_t *qrows, int64_t nq, double *dQ, const int64_t *krows,
    int64_t nk, double *dK, double *dV, int nthreads) {
  if (!Qb || !Kb || !Vb || !dOb || N < 1 || d < 1 || (nq && (!qrows || !dQ)) ||
      (nk && (!krows || !dK || !dV)))
    return ORACLE_EBADARG;
  for (int64_t a = 0; a < nq; ++a)
    if (qrows[a] < 0 || qrows[a] >= N) return ORACLE_EBADARG;
  for (int64_t a = 0; a < nk; ++a)
    if (krows[a] < 0 || krows[a] >= N) return ORACLE_EBADARG;
  double *Q = (double *)malloc(sizeof(double) * (size_t)(N * d));
  double *K = (double *)malloc(sizeof(double) * (size_t)(N * d));
  double *V = (double *)malloc(sizeof(double) * (size_t)(N * d));
  double *dO = (double *)malloc(sizeof(double) * (size_t)(N * d));
  double *lse = (double *)malloc(sizeof(double) * (size_t)N);
  double *Dv = (double *)malloc(sizeof(double) * (size_t)N);
  if (!Q || !K || !V || !dO || !lse || !Dv) {
    free(Q); free(K); free(V); free(dO); free(lse); free(Dv);
    return ORACLE_ENOMEM;
  }
  for (int64_t e = 0; e < N * d; ++e) {
    Q[e] = bf16_bits_to_double(Qb[e]);
    K[e] = bf16_bits_to_double(Kb[e]);
    V[e] = bf16_bits_to_double(Vb[e]);
    dO[e] = bf16_bits_to_double(dOb[e]);
  }
  int err = ORACLE_OK;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    if (!s || !o) {
#pragma omp atomic write
      err = ORACLE_ENOMEM;
    }
    /* every row: lse_i and D_i (the forward of the head) */
#pragma omp for schedule(dynamic, 8)
    for (int64_t i = 0; i < N; ++i) {
      if (!s || !o) continue;
      const int64_t n = visible_keys(i, N, causal);
      for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t t = 0; t < d; ++t) acc += Q[i * d + t] * K[j * d + t];
        s[j] = scale * acc;
      }
      attend_row(s, n, V, d, o, lse + i, NULL);
      double Di = 0.0;
      for (int64_t t = 0; t < d; ++t) Di += dO[i * d + t] * o[t];
      Dv[i] = Di;
    }
    /* dQ for the sampled query rows */
#pragma omp for schedule(dynamic, 1)
    for (int64_t a = 0; a < nq; ++a) {
      if (!s || !o) continue;
      const int64_t i = qrows[a];
      const int64_t n = visible_keys(i, N, causal);
      for (int64_t t = 0; t < d; ++t) dQ[a * d + t] = 0.0;
      for (int64_t j = 0; j < n; ++j) {
        double acc = 0.0, dp = 0.0;
        for (int64_t t = 0; t < d; ++t) {
          acc += Q[i * d + t] * K[j * d + t];
          dp += dO[i * d + t] * V[j * d + t];
        }
        const double pij = exp(scale * acc - lse[i]);
        const double dsij = pij * (dp - Dv[i]);
        for (int64_t t = 0; t < d; ++t) dQ[a * d + t] += scale * dsij * K[j * d + t];
      }
    }
    /* dK, dV for the sampled key rows: over every query that sees the key */
#pragma omp for schedule(dynamic, 1)
    for (int64_t b = 0; b < nk; ++b) {
      if (!s || !o) continue;
      const int64_t j = krows[b];
      for (int64_t t = 0; t < d; ++t) dK[b * d + t] = dV[b * d + t] = 0.0;
      for (int64_t i = causal ? j : 0; i < N; ++i) {
        double acc = 0.0, dp = 0.0;
        for (int64_t t = 0; t < d; ++t) {
          acc += Q[i * d + t] * K[j * d + t];
          dp += dO[i * d + t] * V[j * d + t];
        }
        const double pij = exp(scale * acc - lse[i]);
        const double dsij = pij * (dp - Dv[i]);
        for (int64_t t = 0; t < d; ++t) {
          dV[b * d + t] += pij * dO[i * d + t];
          dK[b * d + t] += scale * dsij * Q[i * d + t];
        }
      }
    }
    free(s); free(o);
  }
  free(Q); free(K); free(V); free(dO); free(lse); free(Dv);
  return err;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
