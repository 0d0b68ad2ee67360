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
 *  - same page, sec. 2 and 5-6 (Gram Newton-Schulz): one NS step is
 *      X_t = p_t(R_{t-1}) X_{t-1} with R = X X^T and the step polynomial
 *      p_t(R) = a_t I + b_t R + c_t R^2, so after t steps X_t = Q_t X_0 with
 *      Q_t = p_t(R_{t-1}) Q_{t-1}, and the Gram matrix evolves as
 *      R_t = p_t(R_{t-1}) R_{t-1} p_t(R_{t-1}); the method tracks R and Q and
 *      forms X only at the end (or at a restart, which materialises X = Q X,
 *      recomputes R from it and starts Q again from I).
 *  - same page, sec. 6, implementation notes: the optional safety factor
 *      divides the normalised input (the example given is 1.05).
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
 * coeffs holds K triples (a_t, b_t, c_t).  The normalised input is divided by
 * `safety` (1 = off).  Result to out (leading dim ldo).
 * Returns 0, or -1 on allocation failure.
 */
int oracle_ns_map(const double *x, int64_t ldx, int64_t h, int64_t w, int K,
                  const double *coeffs, double eps, double safety, double *out, int64_t ldo) {
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
  /* X <- X / (||X||_F + eps), then X <- X / safety */
  const double nrm = frobenius(Y, h * w);
  for (int64_t i = 0; i < h * w; ++i) Y[i] = Y[i] / (nrm + eps) / safety;
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
                    const double *coeffs, double eps, double safety, double *out, int64_t ldo) {
  if (T <= 0) return -2;
  const int64_t tr = (H + T - 1) / T, tc = (W + T - 1) / T;
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
  for (int64_t t = 0; t < tr * tc; ++t) {
    const int64_t p = t / tc, q = t % tc;
    const int64_t r0 = p * T, c0 = q * T;
    const int64_t h = (H - r0 < T) ? H - r0 : T;
    const int64_t w = (W - c0 < T) ? W - c0 : T;
    err |= oracle_ns_map(in + r0 * ldi + c0, ldi, h, w, K, coeffs, eps, safety, out + r0 * ldo + c0, ldo);
  }
  return err ? -1 : 0;
}

/* P = a I + b R + c R^2 (n x n), the step polynomial of the Gram matrix R. */
static void step_polynomial(const double *R, double a, double b, double c, double *P, double *tmp, int64_t n) {
  mm_ab(R, R, tmp, n, n, n);
  for (int64_t i = 0; i < n * n; ++i) P[i] = b * R[i] + c * tmp[i] + ((i / n == i % n) ? a : 0.0);
}

static void set_identity(double *Q, int64_t n) {
  for (int64_t i = 0; i < n * n; ++i) Q[i] = (i / n == i % n) ? 1.0 : 0.0;
}

/*
 * Gram NS on one h x w matrix: the NS map computed through the Gram matrix.
 * Normalise (and divide by `safety`) and transpose exactly as in Algorithm 1;
 * then R = X X^T and Q = I, and per step t, with P = p_t(R):
 *     Q <- P Q          (the accumulated left factor: X_t = Q X_0)
 *     R <- P R P        (the Gram matrix of X_t)
 * and the output is Q X.  restart[] lists the 1-based steps t before which
 * the current iterate is materialised (X <- Q X), its Gram matrix recomputed
 * (R <- X X^T) and Q started again from I; the page restarts before t = 3.
 * In exact arithmetic every restart leaves the result unchanged.
 */
int oracle_gram_ns(const double *x, int64_t ldx, int64_t h, int64_t w, int K, const double *coeffs,
                   double eps, double safety, const int *restart, int n_restart, double *out, int64_t ldo) {
  if (h <= 0 || w <= 0) return 0;
  const int tr = h > w;
  const int64_t n = tr ? w : h, m = tr ? h : w;
  double *X = malloc(sizeof(double) * n * m), *Y = malloc(sizeof(double) * n * m);
  double *R = malloc(sizeof(double) * n * n), *Q = malloc(sizeof(double) * n * n);
  double *P = malloc(sizeof(double) * n * n), *T1 = malloc(sizeof(double) * n * n);
  double *T2 = malloc(sizeof(double) * n * n);
  if (!X || !Y || !R || !Q || !P || !T1 || !T2) {
    free(X); free(Y); free(R); free(Q); free(P); free(T1); free(T2);
    return -1;
  }
  for (int64_t i = 0; i < h; ++i)
    for (int64_t j = 0; j < w; ++j) Y[i * w + j] = x[i * ldx + j];
  const double nrm = frobenius(Y, h * w);
  for (int64_t i = 0; i < h * w; ++i) Y[i] = Y[i] / (nrm + eps) / safety;
  if (tr) transpose(Y, X, h, w); else memcpy(X, Y, sizeof(double) * n * m);
  mm_abt(X, X, R, n, n, m);
  set_identity(Q, n);
  for (int t = 1; t <= K; ++t) {
    int is_restart = 0;
    for (int r = 0; r < n_restart; ++r) is_restart |= (restart[r] == t);
    if (is_restart) {
      mm_ab(Q, X, Y, n, m, n);
      memcpy(X, Y, sizeof(double) * n * m);
      mm_abt(X, X, R, n, n, m);
      set_identity(Q, n);
    }
    const double *ct = coeffs + 3 * (t - 1);
    step_polynomial(R, ct[0], ct[1], ct[2], P, T1, n);
    mm_ab(P, Q, T1, n, n, n);                 /* Q <- P Q   */
    memcpy(Q, T1, sizeof(double) * n * n);
    mm_ab(P, R, T1, n, n, n);                 /* R <- P R P */
    mm_ab(T1, P, T2, n, n, n);
    memcpy(R, T2, sizeof(double) * n * n);
  }
  mm_ab(Q, X, Y, n, m, n);
  if (tr) { transpose(Y, X, n, m); memcpy(Y, X, sizeof(double) * n * m); }
  for (int64_t i = 0; i < h; ++i)
    for (int64_t j = 0; j < w; ++j) out[i * ldo + j] = Y[i * w + j];
  free(X); free(Y); free(R); free(Q); free(P); free(T1); free(T2);
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
