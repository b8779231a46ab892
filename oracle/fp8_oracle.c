/*
 * fp8_oracle.c -- CPU oracle for FP8 attention with incoherent processing.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * with the CUDA library and includes none of the library's files.
 *
 * Source, cited as [MM]: the marketmaker.cc blog post (Indonesian edition)
 * "Apakah Konteks Sehari Penuh Mengalahkan Konteks Sepuluh Menit? Perhatian
 * Kilat dan Pertanyaan Panjang Urutan", section "FA3: Mekanika hopper",
 * item 3: FP8 attention is spoiled by outliers when done naively; the vectors
 * are rotated at random before block quantization so that an outlier's
 * magnitude is spread over all coordinates.  The section gives no formulas;
 * the readings taken here (one sentence each):
 *
 *   * the rotation is applied to Q and K (the pair whose product it leaves
 *     unchanged); it is the randomized Hadamard map x -> x diag(s) H with
 *     s_t = +-1 drawn at random (passed in) and H the d x d Sylvester
 *     Hadamard matrix, H[a][t] = (-1)^popcount(a & t).  H is kept unscaled
 *     (H H^T = d I), so (Q D H)(K D H)^T = d Q K^T and the softmax scale of
 *     the rotated problem is scale / d;
 *   * FP8 is OCP E4M3 ("fn": max finite 448, no infinities), rounding to
 *     nearest, ties to even;
 *   * block quantization: one power-of-two scale per block of rows, the
 *     largest 2^e with amax * 2^e <= 448 (amax over the block after the
 *     rotation, values first rounded to fp32); code = e4m3(x * 2^e); the
 *     stored dequantization scale is 2^-e.  Blocks are the 128-row tiles
 *     for Q and K and the whole head for V (so V's scale factors out of
 *     the P.V sum);
 *   * the attention itself is the blocked online softmax of [MM] "Algoritma
 *     Flash Attention" over the dequantized operands, key blocks of Bc = 128,
 *     with a running base m (natural-log units) per row: the first block's
 *     maximum, then a later block's maximum mb whenever (mb - m) / ln 2
 *     exceeds tau (tau = 0: the exact running maximum).  The block's
 *     probabilities are carried as p = 2^(8 - tau) exp(s - m) (<= 256 <
 *     448), rounded to fp32 and then to E4M3 before they multiply V (the
 *     FP8 P.V product); the row sum l adds the unrounded p; O = acc / l and
 *     lse = m + ln(l) - (8 - tau) ln 2.  Bc, tau and the 2^(8 - tau) are the
 *     kernel's choices, not the pages'.
 *
 * Arithmetic is IEEE double except where a rounding step is part of the
 * method (fp32 before E4M3).  Layouts: codes are row-major [BH, N, d] bytes;
 * Q and K scales [BH, ceil(N / 128)]; V scale [BH].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define FP8_OK 0
#define FP8_EBADARG 1
#define FP8_ENOMEM 2

#define E4M3_MAX 448.0

/* Value of an E4M3 code: sign bit 7, exponent bits 6..3 (bias 7), mantissa
 * bits 2..0; exponent field 0 is subnormal (m / 8 * 2^-6); code 0x7F / 0xFF
 * is NaN (never produced here). */
double oracle_e4m3_decode(uint8_t c) {
  const int sign = (c >> 7) & 1;
  const int ex = (c >> 3) & 15;
  const int man = c & 7;
  double v;
  if (ex == 15 && man == 7) return NAN;
  if (ex == 0)
    v = ldexp((double)man, -9); /* (man / 8) * 2^-6 */
  else
    v = ldexp(1.0 + man / 8.0, ex - 7);
  return sign ? -v : v;
}

/* Nearest E4M3 code to a float, ties to the even code (even mantissa), with
 * saturation to +-448 for values beyond the largest finite code.  Done by
 * definition: among the non-negative finite codes (0x00 .. 0x7E, increasing
 * in value) find the neighbours of |x| and take the nearer one. */
uint8_t oracle_e4m3_encode(float xf) {
  const double x = (double)xf;
  if (isnan(x)) return 0x7F;
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  const double a = fabs(x);
  if (a >= E4M3_MAX) return sign | 0x7E;
  /* largest code with value <= a (values increase with the code): bisection
   * with the invariant decode(lo) <= a < decode(hi_ex) */
  int lo = 0, hi_ex = 0x7F;
  while (hi_ex - lo > 1) {
    const int mid = (lo + hi_ex) / 2;
    if (oracle_e4m3_decode((uint8_t)mid) <= a) lo = mid;
    else hi_ex = mid;
  }
  if (oracle_e4m3_decode((uint8_t)lo) == a || lo == 0x7E) return sign | (uint8_t)lo;
  const int hi = lo + 1;
  const double dlo = a - oracle_e4m3_decode((uint8_t)lo);
  const double dhi = oracle_e4m3_decode((uint8_t)hi) - a;
  int pick;
  if (dlo < dhi) pick = lo;
  else if (dhi < dlo) pick = hi;
  else pick = (lo & 1) ? hi : lo; /* tie: even mantissa (code parity) */
  return sign | (uint8_t)pick;
}

int oracle_e4m3_encode_array(const float *x, int64_t n, uint8_t *out) {
  if ((!x || !out) && n > 0) return FP8_EBADARG;
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(x[i]);
  return FP8_OK;
}

static double bf16_to_double(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static int popcount_u32(uint32_t v) {
  int c = 0;
  while (v) { c += (int)(v & 1u); v >>= 1; }
  return c;
}

/* Entry (a, t) of the d x d Sylvester Hadamard matrix. */
static double hadamard_entry(int64_t a, int64_t t) {
  return (popcount_u32((uint32_t)(a & t)) & 1) ? -1.0 : 1.0;
}

/* y = x diag(s) H for one row, as the plain matrix-vector product in fp64
 * (every partial sum is exact for bf16 inputs whose magnitudes within a row
 * span fewer than ~2^38). */
static void rotate_row(const double *x, const int8_t *s, int64_t d, double *y) {
  for (int64_t t = 0; t < d; ++t) {
    double acc = 0.0;
    for (int64_t a = 0; a < d; ++a) acc += x[a] * (double)s[a] * hadamard_entry(a, t);
    y[t] = acc;
  }
}

int oracle_hadamard_rotate(const double *x, int64_t rows, int64_t d,
                           const int8_t *signs, double *y) {
  if (!x || !signs || !y || rows < 0 || d < 1 || (d & (d - 1))) return FP8_EBADARG;
  for (int64_t r = 0; r < rows; ++r) rotate_row(x + r * d, signs, d, y + r * d);
  return FP8_OK;
}

/* Largest integer e (capped at 126) with amax * 2^e <= 448; 0 for amax = 0. */
static int block_exponent(double amax) {
  if (amax == 0.0) return 0;
  int E;
  frexp(amax, &E); /* amax = f 2^E, f in [0.5, 1) */
  int e = 9 - E;   /* amax * 2^e < 2^9: start above the answer */
  while (ldexp(amax, e) > E4M3_MAX) --e;
  return e > 126 ? 126 : e;
}

/* Block quantization of a bf16 tensor [BH, N, d] (raw bits), optionally
 * rotated first.  block_rows rows share one scale (block_rows >= N: one per
 * head).  codes: [BH, N, d]; scales: [BH, ceil(N / block_rows)], each the
 * dequantization multiplier 2^-e. */
int oracle_fp8_quantize(const uint16_t *x, int64_t BH, int64_t N, int64_t d,
                        int rotate, const int8_t *signs, int64_t block_rows,
                        uint8_t *codes, double *scales) {
  if (!x || !codes || !scales || BH < 0 || N < 1 || d < 1 || block_rows < 1 ||
      (rotate && (!signs || (d & (d - 1)))))
    return FP8_EBADARG;
  const int64_t nblk = (N + block_rows - 1) / block_rows;
  double *row = (double *)malloc(sizeof(double) * (size_t)d);
  double *rot = (double *)malloc(sizeof(double) * (size_t)d);
  float *yf = (float *)malloc(sizeof(float) * (size_t)(block_rows < N ? block_rows : N) * (size_t)d);
  if (!row || !rot || !yf) {
    free(row); free(rot); free(yf);
    return FP8_ENOMEM;
  }
  for (int64_t bh = 0; bh < BH; ++bh)
    for (int64_t b = 0; b < nblk; ++b) {
      const int64_t r0 = b * block_rows;
      const int64_t nr = (N - r0 < block_rows) ? (N - r0) : block_rows;
      /* rotated (or plain) values, rounded to fp32 */
      double amax = 0.0;
      for (int64_t r = 0; r < nr; ++r) {
        const uint16_t *xr = x + ((bh * N) + r0 + r) * d;
        for (int64_t t = 0; t < d; ++t) row[t] = bf16_to_double(xr[t]);
        if (rotate) rotate_row(row, signs, d, rot);
        else memcpy(rot, row, sizeof(double) * (size_t)d);
        for (int64_t t = 0; t < d; ++t) {
          yf[r * d + t] = (float)rot[t];
          const double a = fabs((double)yf[r * d + t]);
          if (a > amax) amax = a;
        }
      }
      const int e = block_exponent(amax);
      scales[bh * nblk + b] = ldexp(1.0, -e);
      for (int64_t r = 0; r < nr; ++r)
        for (int64_t t = 0; t < d; ++t)
          codes[((bh * N) + r0 + r) * d + t] =
              oracle_e4m3_encode((float)ldexp((double)yf[r * d + t], e));
    }
  free(row); free(rot); free(yf);
  return FP8_OK;
}

/* Distance (relative to p) from p > 0 to the nearest E4M3 rounding boundary
 * around the code p rounds to, and the larger code spacing next to it. */
static void boundary_distance(double p, double *rel_dist, double *step) {
  const uint8_t c = oracle_e4m3_encode((float)p);
  const double v = oracle_e4m3_decode(c);
  const double below = (c > 0) ? oracle_e4m3_decode((uint8_t)(c - 1)) : 0.0;
  const double above = (c < 0x7E) ? oracle_e4m3_decode((uint8_t)(c + 1)) : v;
  const double lo_mid = 0.5 * (v + below), hi_mid = 0.5 * (v + above);
  double dist = fabs(p - lo_mid);
  if (fabs(hi_mid - p) < dist) dist = fabs(hi_mid - p);
  *rel_dist = dist / p;
  *step = (above - v > v - below) ? (above - v) : (v - below);
}

/* One output row of the FP8 attention ([MM] "Algoritma Flash Attention",
 * one query row at a time; blocks of Bc keys).  Khat / Vhat: the head's
 * dequantized K (already rotated if Q is) and V codes times their scales,
 * [N, d]; qhat: the row's dequantized query.  If flip_delta > 0, *flip_bound
 * receives sum over keys whose p lies within relative flip_delta of an E4M3
 * rounding boundary of (code spacing) * max_t |Vhat[key, t]|, divided by l:
 * the most a one-step change of those codes can move any output of the row.
 * A relative error flip_delta in p is an error of flip_delta / ln 2 in the
 * exponent (log2 units), so when a base decision (block gap against tau)
 * lies within twice that of tau, a kernel computing the scores in fp32 may
 * decide it the other way and carry every later p of the row on another
 * base: *flip_bound is then +infinity (the row's codes are not predicted). */
static void fp8_row(const double *qhat, const double *Khat, const double *Vhat,
                    int64_t N, int64_t d, int64_t i, int causal, double scale,
                    int64_t Bc, double tau, double *s, double *acc, double *orow,
                    double *lse, double flip_delta, double *flip_bound) {
  const double ln2 = log(2.0);
  const double offset = exp2(8.0 - tau);
  double m = -INFINITY, l = 0.0, flip = 0.0;
  int ambiguous = 0;
  for (int64_t t = 0; t < d; ++t) acc[t] = 0.0;
  const int64_t kend = causal ? i + 1 : N;
  for (int64_t k0 = 0; k0 < kend; k0 += Bc) {
    const int64_t k1 = (k0 + Bc < kend) ? k0 + Bc : kend;
    /* S_ij over the block (keys beyond kend are masked: not visited) */
    double mb = -INFINITY;
    for (int64_t c = k0; c < k1; ++c) {
      double dot = 0.0;
      for (int64_t t = 0; t < d; ++t) dot += qhat[t] * Khat[c * d + t];
      s[c - k0] = scale * dot;
      if (s[c - k0] > mb) mb = s[c - k0];
    }
    /* the base: the first block's maximum, later a block maximum that
       exceeds it by more than tau (log2 units); rescale what was
       accumulated */
    if (m == -INFINITY) {
      m = mb;
    } else {
      const double gap = (mb - m) / ln2;
      /* (at tau = 0 the two choices of a near tie are nearly the same base,
         which the flip bound covers) */
      if (flip_delta > 0.0 && tau > 0.0 && fabs(gap - tau) <= 2.0 * flip_delta / ln2)
        ambiguous = 1;
      if (gap > tau) {
        const double alpha = exp(m - mb);
        l *= alpha;
        flip *= alpha;
        for (int64_t t = 0; t < d; ++t) acc[t] *= alpha;
        m = mb;
      }
    }
    /* p = 2^(8 - tau) exp(s - m); l adds p; the P.V product uses
       E4M3(fp32(p)) */
    for (int64_t c = k0; c < k1; ++c) {
      const double p = offset * exp(s[c - k0] - m);
      l += p;
      const double pq = oracle_e4m3_decode(oracle_e4m3_encode((float)p));
      for (int64_t t = 0; t < d; ++t) acc[t] += pq * Vhat[c * d + t];
      if (flip_delta > 0.0 && p > 0.0) {
        double rel, step;
        boundary_distance(p, &rel, &step);
        if (rel <= flip_delta) {
          double vmax = 0.0;
          for (int64_t t = 0; t < d; ++t)
            if (fabs(Vhat[c * d + t]) > vmax) vmax = fabs(Vhat[c * d + t]);
          flip += step * vmax;
        }
      }
    }
  }
  for (int64_t t = 0; t < d; ++t) orow[t] = acc[t] / l;
  *lse = m + log(l) - (8.0 - tau) * ln2;
  if (flip_bound) *flip_bound = ambiguous ? INFINITY : flip / l;
}

static void dequant_head(const uint8_t *codes, const double *scales, int64_t N,
                         int64_t d, int64_t block_rows, double *out) {
  for (int64_t r = 0; r < N; ++r) {
    const double sc = scales[r / block_rows];
    for (int64_t t = 0; t < d; ++t)
      out[r * d + t] = oracle_e4m3_decode(codes[r * d + t]) * sc;
  }
}

/* FP8 attention on quantized operands for a list of rows (flat indices
 * bh * N + i).  q_block / k_block: rows per Q / K scale block; V has one
 * scale per head.  scale: the softmax scale of the (rotated) problem.
 * O [nrows, d], lse [nrows]; flip_bound [nrows] optional (see fp8_row). */
int oracle_attention_fp8_rows(const uint8_t *q8, const double *q_scale,
                              const uint8_t *k8, const double *k_scale,
                              const uint8_t *v8, const double *v_scale,
                              int64_t BH, int64_t N, int64_t d, int causal,
                              double scale, int64_t q_block, int64_t k_block,
                              int64_t Bc, double tau, const int64_t *rows, int64_t nrows,
                              double *O, double *lse, double flip_delta,
                              double *flip_bound, int threads) {
  if (!q8 || !q_scale || !k8 || !k_scale || !v8 || !v_scale || !rows || !O ||
      !lse || BH < 1 || N < 1 || d < 1 || q_block < 1 || k_block < 1 || Bc < 1 ||
      !(tau >= 0.0 && tau <= 8.0))
    return FP8_EBADARG;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= BH * N) return FP8_EBADARG;
  const int64_t qblocks = (N + q_block - 1) / q_block;
  const int64_t kblocks = (N + k_block - 1) / k_block;
  int rc = FP8_OK;
  /* rows are grouped by head so that each head's K, V are dequantized once */
  for (int64_t bh = 0; bh < BH && rc == FP8_OK; ++bh) {
    int64_t cnt = 0;
    for (int64_t r = 0; r < nrows; ++r) cnt += (rows[r] / N == bh);
    if (cnt == 0) continue;
    double *Khat = (double *)malloc(sizeof(double) * (size_t)(N * d));
    double *Vhat = (double *)malloc(sizeof(double) * (size_t)(N * d));
    if (!Khat || !Vhat) {
      free(Khat); free(Vhat);
      return FP8_ENOMEM;
    }
    dequant_head(k8 + bh * N * d, k_scale + bh * kblocks, N, d, k_block, Khat);
    dequant_head(v8 + bh * N * d, v_scale + bh, N, d, N, Vhat);
#ifdef _OPENMP
#pragma omp parallel num_threads(threads > 0 ? threads : 1)
#endif
    {
      double *s = (double *)malloc(sizeof(double) * (size_t)Bc);
      double *acc = (double *)malloc(sizeof(double) * (size_t)d);
      double *qhat = (double *)malloc(sizeof(double) * (size_t)d);
      if (!s || !acc || !qhat) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
        rc = FP8_ENOMEM;
      } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
        for (int64_t r = 0; r < nrows; ++r) {
          if (rows[r] / N != bh) continue;
          const int64_t i = rows[r] % N;
          const double qs = q_scale[bh * qblocks + i / q_block];
          for (int64_t t = 0; t < d; ++t)
            qhat[t] = oracle_e4m3_decode(q8[rows[r] * d + t]) * qs;
          fp8_row(qhat, Khat, Vhat, N, d, i, causal, scale, Bc, tau, s, acc,
                  O + r * d, lse + r, flip_delta, flip_bound ? flip_bound + r : NULL);
        }
      }
      free(s); free(acc); free(qhat);
    }
    free(Khat); free(Vhat);
  }
  (void)threads;
  return rc;
}
