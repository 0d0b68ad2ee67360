/*
 * himuon_oracle.c -- plain fp64 CPU oracle for the tiled Newton-Schulz map.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library path links, loads or
 * calls this file; only the tests, the package's smoke check and the bench's
 * CPU baseline do.  It shares no code, header or constant with the CUDA path.
 *
 * Every routine is the plain definition, in fp64, with naive loops and no
 * blocking, fusion or reordering beyond what the pages state.  OpenMP (when
 * compiled with -fopenmp) only spreads independent rows or tiles across
 * threads; it does not change the arithmetic.
 *
 * Sources (page titles and sections):
 *  - "Gram Newton-Schulz" summary, sec. 3, Muon recap: the update
 *      M_k = mu M_{k-1} + G_k ;  W_{k+1} = W_k - eta polar(M_k).
 *  - same page, sec. 3, Algorithm 1 (standard Newton-Schulz): normalise by
 *      (||X||_F + eps), transpose when the input is taller than wide, then per
 *      step A = X X^T, B = b_t A + c_t A^2, X = a_t X + B X, undo the transpose.
 *  - same page, sec. 6, Algorithm 3 (stabilised Gram Newton-Schulz):
 *      R = X X^T, Q = I; per step (with a restart X <- Q X, R <- X X^T, Q <- I
 *      before the listed steps) Z = b R + c R^2, Q <- Q Z + a Q,
 *      RZ <- R Z + a R, R <- Z RZ + a RZ; output Q X.
 *  - "Hierarchical Muon: Tiled Newton-Schulz Updates", abstract: cut the
 *      matrix into T x T tiles, apply the same NS map to each tile on its own,
 *      put the results back in place.
 *  - CMuon article: split a fused tensor into its functional blocks and
 *      orthogonalise each block separately.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - Ragged edge tiles are smaller matrices under the same map (transposed
 *    when taller than wide); tiles start at the top-left corner.
 *  - The bf16 cast that Algorithm 1 applies "for speed" is not part of the
 *    map; the oracle stays in fp64 throughout.
 *  - A zero tile gives 0 / (0 + eps) = 0, so its output is 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* C = A * B^T, A: n x k (row-major), B: m x k (row-major), C: n x m. */
static void mm_abt(const double *A, const double *B, double *C, int64_t n, int64_t m, int64_t k) {
#pragma omp parallel for schedule(static) if (n * m * k > (1 << 22))
  for (int64_t i = 0; i < n; ++i) {
    for (int64_t j = 0; j < m; ++j) {
      double s = 0.0;
      for (int64_t p = 0; p < k; ++p) s += A[i * k + p] * B[j * k + p];
      C[i * m + j] = s;
    }
  }
}

/* C = A * B, A: n x k, B: k x m, C: n x m (all row-major). */
static void mm_ab(const double *A, const double *B, double *C, int64_t n, int64_t m, int64_t k) {
#pragma omp parallel for schedule(static) if (n * m * k > (1 << 22))
  for (int64_t i = 0; i < n; ++i) {
    double *c = C + i * m;
    for (int64_t j = 0; j < m; ++j) c[j] = 0.0;
    for (int64_t p = 0; p < k; ++p) {
      const double a = A[i * k + p];
      const double *b = B + p * m;
      for (int64_t j = 0; j < m; ++j) c[j] += a * b[j];
    }
  }
}

static void transpose(const double *X, double *Y, int64_t rows, int64_t cols) {
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t j = 0; j < cols; ++j) Y[j * rows + i] = X[i * cols + j];
}

static double frobenius(const double *X, int64_t count) {
  double s = 0.0;
  for (int64_t i = 0; i < count; ++i) s += X[i] * X[i];
  return sqrt(s);
}

/*
 * Algorithm 1 (standard NS) on one h x w matrix x (row-major, leading dim ldx).
 * coeffs holds K triples (a_t, b_t, c_t).  Result to out (leading dim ldo).
 * Returns 0, or -1 on allocation failure.
 */
int oracle_ns_map(const double *x, int64_t ldx, int64_t h, int64_t w, int K,
                  const double *coeffs, double eps, double *out, int64_t ldo) {
  if (h <= 0 || w <= 0) return 0;
  const int tr = h > w;              /* "If m < n: X <- X^T" for an n x m input */
  const int64_t n = tr ? w : h;      /* rows of the iterate, n <= m */
  const int64_t m = tr ? h : w;
  double *X = malloc(sizeof(double) * n * m);
  double *Y = malloc(sizeof(double) * n * m);
  double *A = malloc(sizeof(double) * n * n);
  double *A2 = malloc(sizeof(double) * n * n);
  double *B = malloc(sizeof(double) * n * n);
  double *BX = malloc(sizeof(double) * n * m);
  if (!X || !Y || !A || !A2 || !B || !BX) {
    free(X); free(Y); free(A); free(A2); free(B); free(BX);
    return -1;
  }
  /* copy the input as an h x w dense block */
  for (int64_t i = 0; i < h; ++i)
    for (int64_t j = 0; j < w; ++j) Y[i * w + j] = x[i * ldx + j];
  /* X <- X / (||X||_F + eps) */
  const double nrm = frobenius(Y, h * w);
  for (int64_t i = 0; i < h * w; ++i) Y[i] = Y[i] / (nrm + eps);
  if (tr) transpose(Y, X, h, w); else memcpy(X, Y, sizeof(double) * n * m);
  for (int t = 0; t < K; ++t) {
    const double a = coeffs[3 * t + 0], b = coeffs[3 * t + 1], c = coeffs[3 * t + 2];
    mm_abt(X, X, A, n, n, m);                         /* A = X X^T        */
    mm_ab(A, A, A2, n, n, n);                         /* A^2              */
    for (int64_t i = 0; i < n * n; ++i) B[i] = b * A[i] + c * A2[i];   /* B = bA + cA^2 */
    mm_ab(B, X, BX, n, m, n);                         /* B X              */
    for (int64_t i = 0; i < n * m; ++i) X[i] = a * X[i] + BX[i];       /* X = aX + BX   */
  }
  if (tr) transpose(X, Y, n, m); else memcpy(Y, X, sizeof(double) * n * m);
  for (int64_t i = 0; i < h; ++i)
    for (int64_t j = 0; j < w; ++j) out[i * ldo + j] = Y[i * w + j];
  free(X); free(Y); free(A); free(A2); free(B); free(BX);
  return 0;
}

/*
 * HiMuon tiling of one H x W matrix with tile size T: tile (p, q) covers rows
 * [pT, min(pT+T, H)) and columns [qT, min(qT+T, W)); each tile gets the NS map
 * on its own and is written back in place.  T >= max(H, W) is full-matrix NS.
 */
int oracle_ns_tiled(const double *in, int64_t ldi, int64_t H, int64_t W, int64_t T, int K,
                    const double *coeffs, double eps, double *out, int64_t ldo) {
  if (T <= 0) return -2;
  const int64_t tr = (H + T - 1) / T, tc = (W + T - 1) / T;
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
  for (int64_t t = 0; t < tr * tc; ++t) {
    const int64_t p = t / tc, q = t % tc;
    const int64_t r0 = p * T, c0 = q * T;
    const int64_t h = (H - r0 < T) ? H - r0 : T;
    const int64_t w = (W - c0 < T) ? W - c0 : T;
    err |= oracle_ns_map(in + r0 * ldi + c0, ldi, h, w, K, coeffs, eps, out + r0 * ldo + c0, ldo);
  }
  return err ? -1 : 0;
}

/*
 * Algorithm 3 (stabilised Gram NS) on one h x w matrix.  restart[] lists the
 * 1-based step indices t before which X <- Q X, R <- X X^T, Q <- I happens
 * (the page restarts at t = 3).  With n_restart = 0 this is Algorithm 2 with
 * the identity term added explicitly, which is the same map.
 */
int oracle_gram_ns(const double *x, int64_t ldx, int64_t h, int64_t w, int K, const double *coeffs,
                   double eps, const int *restart, int n_restart, double *out, int64_t ldo) {
  if (h <= 0 || w <= 0) return 0;
  const int tr = h > w;
  const int64_t n = tr ? w : h, m = tr ? h : w;
  double *X = malloc(sizeof(double) * n * m), *Y = malloc(sizeof(double) * n * m);
  double *R = malloc(sizeof(double) * n * n), *Q = malloc(sizeof(double) * n * n);
  double *Z = malloc(sizeof(double) * n * n), *R2 = malloc(sizeof(double) * n * n);
  double *RZ = malloc(sizeof(double) * n * n), *T1 = malloc(sizeof(double) * n * n);
  if (!X || !Y || !R || !Q || !Z || !R2 || !RZ || !T1) {
    free(X); free(Y); free(R); free(Q); free(Z); free(R2); free(RZ); free(T1);
    return -1;
  }
  for (int64_t i = 0; i < h; ++i)
    for (int64_t j = 0; j < w; ++j) Y[i * w + j] = x[i * ldx + j];
  const double nrm = frobenius(Y, h * w);
  for (int64_t i = 0; i < h * w; ++i) Y[i] = Y[i] / (nrm + eps);
  if (tr) transpose(Y, X, h, w); else memcpy(X, Y, sizeof(double) * n * m);
  mm_abt(X, X, R, n, n, m);                                   /* R_0 = X X^T */
  for (int64_t i = 0; i < n * n; ++i) Q[i] = (i / n == i % n) ? 1.0 : 0.0;   /* Q_0 = I */
  for (int t = 1; t <= K; ++t) {
    const double a = coeffs[3 * (t - 1) + 0], b = coeffs[3 * (t - 1) + 1], c = coeffs[3 * (t - 1) + 2];
    int is_restart = 0;
    for (int r = 0; r < n_restart; ++r) is_restart |= (restart[r] == t);
    if (is_restart) {
      mm_ab(Q, X, Y, n, m, n);                                /* X <- Q X    */
      memcpy(X, Y, sizeof(double) * n * m);
      mm_abt(X, X, R, n, n, m);                               /* R <- X X^T  */
      for (int64_t i = 0; i < n * n; ++i) Q[i] = (i / n == i % n) ? 1.0 : 0.0;
    }
    mm_ab(R, R, R2, n, n, n);
    for (int64_t i = 0; i < n * n; ++i) Z[i] = b * R[i] + c * R2[i];           /* Z = bR + cR^2   */
    mm_ab(Q, Z, T1, n, n, n);
    for (int64_t i = 0; i < n * n; ++i) Q[i] = T1[i] + a * Q[i];               /* Q = QZ + aQ     */
    mm_ab(R, Z, T1, n, n, n);
    for (int64_t i = 0; i < n * n; ++i) RZ[i] = T1[i] + a * R[i];              /* RZ = RZ + aR    */
    mm_ab(Z, RZ, T1, n, n, n);
    for (int64_t i = 0; i < n * n; ++i) R[i] = T1[i] + a * RZ[i];              /* R = Z RZ + a RZ */
  }
  mm_ab(Q, X, Y, n, m, n);                                    /* output Q X  */
  if (tr) { transpose(Y, X, n, m); memcpy(Y, X, sizeof(double) * n * m); }
  for (int64_t i = 0; i < h; ++i)
    for (int64_t j = 0; j < w; ++j) out[i * ldo + j] = Y[i * w + j];
  free(X); free(Y); free(R); free(Q); free(Z); free(R2); free(RZ); free(T1);
  return 0;
}

/* Muon recap: M' = mu M + G, elementwise over `count` values. */
void oracle_momentum(const double *M, const double *G, double mu, double *Mout, int64_t count) {
  for (int64_t i = 0; i < count; ++i) Mout[i] = mu * M[i] + G[i];
}

/* Muon recap: W' = W - eta O, elementwise. */
void oracle_apply_update(const double *W, const double *O, double eta, double *Wout, int64_t count) {
  for (int64_t i = 0; i < count; ++i) Wout[i] = W[i] - eta * O[i];
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
