/*
 * Flash PD-SSM forward pass -- dense CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. It shares no code, header, table or
 * helper with the CUDA path, and it is never a fallback for it.
 *
 * What it computes (plain, slow and literal, in fp64 / complex128):
 *
 *   1. Selection: s_t = argmax_k logits_t[k], lowest k on ties
 *      [Flash PD-SSM page, Technical Summary, Methodology 1 "Novel Selection
 *      Mechanism": the K scores come from a linear map of u_t and the single
 *      highest-scoring dictionary matrix is used; Methodology 2: the forward
 *      pass uses hard argmax]. The pages name no tie rule; the lowest index
 *      wins, +0 and -0 compare equal, and the first NaN wins.
 *
 *   2. Dictionary: P_k is the dense N x N matrix with P_k[idx[k][j]][j] = 1 and
 *      zeros elsewhere -- one nonzero per column, the "one-hot column selector"
 *      of Methodology 1 (column-wise hardmax of the original PD-SSM, same
 *      section).
 *
 *   3. Recurrence, read from the PD (one-hot-column times diagonal) structure
 *      the Problem Statement and Methodology 1 describe in words (the page
 *      prints no formula): with A_t = P_{s_t} diag(d_t),
 *          H_t = A_t H_{t-1} + B_t x_t^T        (N x P state, H_{-1} = h0 or 0)
 *          y_t = H_t^T C_t                      (plain transpose, no conjugate)
 *          M_t = A_t M_{t-1}, M_{-1} = I        (running product)
 *      Every product here is a dense N x N times N x P (or N x N) product;
 *      nothing exploits the sparsity, which is the point of an oracle.
 *
 *   4. Outputs: y, h_final = H_{L-1}, and the whole-sequence product M written
 *      as (prod_idx[j], prod_val[j]) = (row of the nonzero in column j of M,
 *      its value). The row is taken from the 0/1 pattern product of the P_k
 *      (kept exactly in integers), the value from the fp64 product, so a value
 *      that underflows to 0 over a long sequence keeps its row.
 *
 * Arrays are slice-major: S independent (batch, head) slices, each holding
 * all L steps contiguously, e.g. d[S][L][N], x[S][L][P], y[S][L][P],
 * h0/h_final[S][N][P], prod_*[S][N]. Complex arrays are interleaved (re, im)
 * doubles. The slices are independent and are spread over OpenMP threads.
 */
#include <complex.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ALLOC 1
#define ORACLE_ERR_PATTERN 2

int pdssm_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Methodology 1/2: hard argmax; lowest k on ties, first NaN wins. */
static int32_t argmax_row(const double *v, int64_t K) {
  if (isnan(v[0])) return 0;
  int32_t best = 0;
  double bv = v[0];
  for (int64_t k = 1; k < K; ++k) {
    if (isnan(v[k])) return (int32_t)k;
    if (v[k] > bv) {
      bv = v[k];
      best = (int32_t)k;
    }
  }
  return best;
}

void pdssm_oracle_select(const double *logits, int64_t rows, int64_t K, int32_t *s) {
  for (int64_t r = 0; r < rows; ++r) s[r] = argmax_row(logits + r * K, K);
}

/* Row of the single nonzero of column j of the 0/1 pattern matrix, or -1. */
static int pattern_row(const uint8_t *Mp, int64_t N, int64_t j, int64_t *row) {
  int64_t found = -1;
  for (int64_t i = 0; i < N; ++i) {
    if (Mp[i * N + j]) {
      if (found >= 0) return ORACLE_ERR_PATTERN;
      found = i;
    }
  }
  if (found < 0) return ORACLE_ERR_PATTERN;
  *row = found;
  return ORACLE_OK;
}

/* Dense 0/1 pattern product Mp <- P_s Mp, in integers. */
static void pattern_step(const int32_t *idx_s, int64_t N, const uint8_t *Mp, uint8_t *Mn) {
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < N; ++j) {
      int acc = 0;
      for (int64_t r = 0; r < N; ++r) acc |= (idx_s[r] == i) & (Mp[r * N + j] != 0);
      Mn[i * N + j] = (uint8_t)acc;
    }
}

/* ------------------------------------------------------------------ real */

static int scan_real_slice(int64_t L, int64_t N, int64_t P, int64_t K, const double *logits,
                           const int32_t *idx, const double *d, const double *B, const double *C,
                           const double *x, const double *h0, double *y, double *h_final,
                           int32_t *prod_idx, double *prod_val, int32_t *s_out) {
  const int want_prod = (prod_idx != NULL) || (prod_val != NULL);
  double *A = calloc((size_t)(N * N), sizeof(double));
  double *H = calloc((size_t)(N * P), sizeof(double));
  double *Hn = calloc((size_t)(N * P), sizeof(double));
  double *Mv = want_prod ? calloc((size_t)(N * N), sizeof(double)) : NULL;
  double *Mvn = want_prod ? calloc((size_t)(N * N), sizeof(double)) : NULL;
  uint8_t *Mp = want_prod ? calloc((size_t)(N * N), 1) : NULL;
  uint8_t *Mpn = want_prod ? calloc((size_t)(N * N), 1) : NULL;
  int rc = ORACLE_OK;
  if (!A || !H || !Hn || (want_prod && (!Mv || !Mvn || !Mp || !Mpn))) {
    rc = ORACLE_ERR_ALLOC;
    goto done;
  }
  if (h0) memcpy(H, h0, sizeof(double) * (size_t)(N * P));
  if (want_prod)
    for (int64_t i = 0; i < N; ++i) {
      Mv[i * N + i] = 1.0;
      Mp[i * N + i] = 1;
    }

  for (int64_t t = 0; t < L; ++t) {
    const int32_t s = argmax_row(logits + t * K, K);
    if (s_out) s_out[t] = s;
    const int32_t *idx_s = idx + (int64_t)s * N;
    const double *dt = d + t * N, *Bt = B + t * N, *Ct = C + t * N, *xt = x + t * P;

    /* A_t = P_s diag(d_t), dense */
    memset(A, 0, sizeof(double) * (size_t)(N * N));
    for (int64_t j = 0; j < N; ++j) A[(int64_t)idx_s[j] * N + j] = dt[j];

    /* H_t = A_t H_{t-1} + B_t x_t^T */
    for (int64_t i = 0; i < N; ++i) {
      double *hn = Hn + i * P;
      for (int64_t p = 0; p < P; ++p) hn[p] = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        const double a = A[i * N + j];
        const double *hj = H + j * P;
        for (int64_t p = 0; p < P; ++p) hn[p] += a * hj[p];
      }
      for (int64_t p = 0; p < P; ++p) hn[p] += Bt[i] * xt[p];
    }
    double *tmp = H;
    H = Hn;
    Hn = tmp;

    /* y_t = H_t^T C_t */
    double *yt = y + t * P;
    for (int64_t p = 0; p < P; ++p) {
      double acc = 0.0;
      for (int64_t i = 0; i < N; ++i) acc += H[i * P + p] * Ct[i];
      yt[p] = acc;
    }

    /* M_t = A_t M_{t-1} (values) and the 0/1 pattern alongside */
    if (want_prod) {
      for (int64_t i = 0; i < N; ++i)
        for (int64_t j = 0; j < N; ++j) {
          double acc = 0.0;
          for (int64_t r = 0; r < N; ++r) acc += A[i * N + r] * Mv[r * N + j];
          Mvn[i * N + j] = acc;
        }
      double *tv = Mv;
      Mv = Mvn;
      Mvn = tv;
      pattern_step(idx_s, N, Mp, Mpn);
      uint8_t *tp = Mp;
      Mp = Mpn;
      Mpn = tp;
    }
  }

  if (h_final) memcpy(h_final, H, sizeof(double) * (size_t)(N * P));
  if (want_prod)
    for (int64_t j = 0; j < N; ++j) {
      int64_t row = 0;
      rc = pattern_row(Mp, N, j, &row);
      if (rc != ORACLE_OK) goto done;
      if (prod_idx) prod_idx[j] = (int32_t)row;
      if (prod_val) prod_val[j] = Mv[row * N + j];
    }

done:
  free(A);
  free(H);
  free(Hn);
  free(Mv);
  free(Mvn);
  free(Mp);
  free(Mpn);
  return rc;
}

int pdssm_oracle_scan_real(int64_t S, int64_t L, int64_t N, int64_t P, int64_t K,
                           const double *logits, const int32_t *idx, const double *d,
                           const double *B, const double *C, const double *x, const double *h0,
                           double *y, double *h_final, int32_t *prod_idx, double *prod_val,
                           int32_t *s_out) {
  int rc = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t sl = 0; sl < S; ++sl) {
    int r = scan_real_slice(
        L, N, P, K, logits + sl * L * K, idx, d + sl * L * N, B + sl * L * N, C + sl * L * N,
        x + sl * L * P, h0 ? h0 + sl * N * P : NULL, y + sl * L * P,
        h_final ? h_final + sl * N * P : NULL, prod_idx ? prod_idx + sl * N : NULL,
        prod_val ? prod_val + sl * N : NULL, s_out ? s_out + sl * L : NULL);
    if (r != ORACLE_OK) {
#pragma omp atomic write
      rc = r;
    }
  }
  return rc;
}

/* --------------------------------------------------------------- complex */
/* Same steps with complex d, complex state and complex y; B, C, x real. */

static int scan_complex_slice(int64_t L, int64_t N, int64_t P, int64_t K, const double *logits,
                              const int32_t *idx, const double complex *d, const double *B,
                              const double *C, const double *x, const double complex *h0,
                              double complex *y, double complex *h_final, int32_t *prod_idx,
                              double complex *prod_val, int32_t *s_out) {
  const int want_prod = (prod_idx != NULL) || (prod_val != NULL);
  double complex *A = calloc((size_t)(N * N), sizeof(double complex));
  double complex *H = calloc((size_t)(N * P), sizeof(double complex));
  double complex *Hn = calloc((size_t)(N * P), sizeof(double complex));
  double complex *Mv = want_prod ? calloc((size_t)(N * N), sizeof(double complex)) : NULL;
  double complex *Mvn = want_prod ? calloc((size_t)(N * N), sizeof(double complex)) : NULL;
  uint8_t *Mp = want_prod ? calloc((size_t)(N * N), 1) : NULL;
  uint8_t *Mpn = want_prod ? calloc((size_t)(N * N), 1) : NULL;
  int rc = ORACLE_OK;
  if (!A || !H || !Hn || (want_prod && (!Mv || !Mvn || !Mp || !Mpn))) {
    rc = ORACLE_ERR_ALLOC;
    goto done;
  }
  if (h0) memcpy(H, h0, sizeof(double complex) * (size_t)(N * P));
  if (want_prod)
    for (int64_t i = 0; i < N; ++i) {
      Mv[i * N + i] = 1.0;
      Mp[i * N + i] = 1;
    }

  for (int64_t t = 0; t < L; ++t) {
    const int32_t s = argmax_row(logits + t * K, K);
    if (s_out) s_out[t] = s;
    const int32_t *idx_s = idx + (int64_t)s * N;
    const double complex *dt = d + t * N;
    const double *Bt = B + t * N, *Ct = C + t * N, *xt = x + t * P;

    for (int64_t q = 0; q < N * N; ++q) A[q] = 0.0;
    for (int64_t j = 0; j < N; ++j) A[(int64_t)idx_s[j] * N + j] = dt[j];

    for (int64_t i = 0; i < N; ++i) {
      double complex *hn = Hn + i * P;
      for (int64_t p = 0; p < P; ++p) hn[p] = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        const double complex a = A[i * N + j];
        const double complex *hj = H + j * P;
        for (int64_t p = 0; p < P; ++p) hn[p] += a * hj[p];
      }
      for (int64_t p = 0; p < P; ++p) hn[p] += Bt[i] * xt[p];
    }
    double complex *tmp = H;
    H = Hn;
    Hn = tmp;

    double complex *yt = y + t * P;
    for (int64_t p = 0; p < P; ++p) {
      double complex acc = 0.0;
      for (int64_t i = 0; i < N; ++i) acc += H[i * P + p] * Ct[i];
      yt[p] = acc;
    }

    if (want_prod) {
      for (int64_t i = 0; i < N; ++i)
        for (int64_t j = 0; j < N; ++j) {
          double complex acc = 0.0;
          for (int64_t r = 0; r < N; ++r) acc += A[i * N + r] * Mv[r * N + j];
          Mvn[i * N + j] = acc;
        }
      double complex *tv = Mv;
      Mv = Mvn;
      Mvn = tv;
      pattern_step(idx_s, N, Mp, Mpn);
      uint8_t *tp = Mp;
      Mp = Mpn;
      Mpn = tp;
    }
  }

  if (h_final) memcpy(h_final, H, sizeof(double complex) * (size_t)(N * P));
  if (want_prod)
    for (int64_t j = 0; j < N; ++j) {
      int64_t row = 0;
      rc = pattern_row(Mp, N, j, &row);
      if (rc != ORACLE_OK) goto done;
      if (prod_idx) prod_idx[j] = (int32_t)row;
      if (prod_val) prod_val[j] = Mv[row * N + j];
    }

done:
  free(A);
  free(H);
  free(Hn);
  free(Mv);
  free(Mvn);
  free(Mp);
  free(Mpn);
  return rc;
}

int pdssm_oracle_scan_complex(int64_t S, int64_t L, int64_t N, int64_t P, int64_t K,
                              const double *logits, const int32_t *idx, const double *d,
                              const double *B, const double *C, const double *x,
                              const double *h0, double *y, double *h_final, int32_t *prod_idx,
                              double *prod_val, int32_t *s_out) {
  const double complex *dc = (const double complex *)d;
  const double complex *h0c = (const double complex *)h0;
  double complex *yc = (double complex *)y;
  double complex *hfc = (double complex *)h_final;
  double complex *pvc = (double complex *)prod_val;
  int rc = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t sl = 0; sl < S; ++sl) {
    int r = scan_complex_slice(
        L, N, P, K, logits + sl * L * K, idx, dc + sl * L * N, B + sl * L * N, C + sl * L * N,
        x + sl * L * P, h0c ? h0c + sl * N * P : NULL, yc + sl * L * P,
        hfc ? hfc + sl * N * P : NULL, prod_idx ? prod_idx + sl * N : NULL,
        pvc ? pvc + sl * N : NULL, s_out ? s_out + sl * L : NULL);
    if (r != ORACLE_OK) {
#pragma omp atomic write
      rc = r;
    }
  }
  return rc;
}
