// Oracle of the hybrid Muon + AdamW optimizer update -- TEST INFRASTRUCTURE ONLY.
//
// Plain single-threaded loops in double, every sum in index order; shares nothing with the
// CUDA library. What each part follows (nanochat architecture page, section
// "Optimierungsstrategien Muon und AdamW"):
//  * the split: Muon for the 2-D matrices of the blocks (attention and MLP weights), AdamW
//    for the embeddings, the (tied) lm_head and the 0-D/1-D parameters;
//  * "Polar Express Details": X = the update in bf16, X /= (||X||_F * 1.01 + 1e-6), then for
//    each (a, b, c) of the first ns coefficient triples: a tall matrix takes A = X^T X,
//    B = b A + c A^2, X = a X + X B; a wide one A = X X^T, X = a X + B X;
//  * "Zustandsverwaltung": two buffers per matrix, the momentum and a factored second moment
//    that is reduced per row for tall matrices and per column for wide ones;
//  * "Cautious Update Mechanismus": mask = (update * param >= 0);
//    param -= lr * update + lr * wd * param * mask.
// Readings where the page is silent or its figure did not survive (the four-stage pipeline
// diagram is missing):
//  * tall means rows > cols (a square matrix takes the wide branch);
//  * stage 1, momentum, Nesterov form in the lerp notation of the AdamW listing:
//    buf = lerp(buf, g, 1 - mu); u = lerp(g, buf, mu);
//  * the iteration runs in exact (double) arithmetic, or, with `bf16`, at the page's precision:
//    the update is cast to bf16 (X = g.bfloat16()), and every matrix the iteration stores
//    (X after the normalisation, A, B, each new X) is rounded to bf16 once it is formed, its
//    products and sums taken exactly before that rounding;
//  * stage 3, the factored second moment: v = mean of X^2 over the reduced dimension,
//    s = lerp(s, v, 1 - beta2), X' = X / sqrt(max(s, eps)) broadcast along that dimension,
//    then X' is rescaled to the Frobenius norm of X (the step size stays Muon's);
//  * the global clip coefficient of the step (min(1, clip / (||g|| + 1e-6))) scales the raw
//    gradient of both optimizers.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "gpt_oracle.h"

namespace {

// Round to bf16 (nearest even), through float: the value a float accumulator would hold.
double bf16r(double x) {
  float f = (float)x;
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u) return x;  // inf / nan unchanged
  u = (u + 0x7fffu + ((u >> 16) & 1u)) & 0xffff0000u;
  std::memcpy(&f, &u, 4);
  return (double)f;
}
void round_all(std::vector<double> &v, bool on) {
  if (on)
    for (double &x : v) x = bf16r(x);
}

// C[m][n] = sum_k A[m][k] * B[k][n]   (A: m x k, B: k x n, row-major)
void matmul(const double *A, const double *B, int m, int k, int n, double *C) {
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < n; ++j) {
      double s = 0;
      for (int t = 0; t < k; ++t) s += A[(size_t)i * k + t] * B[(size_t)t * n + j];
      C[(size_t)i * n + j] = s;
    }
}

void transpose(const double *X, int r, int c, double *Y) {
  for (int i = 0; i < r; ++i)
    for (int j = 0; j < c; ++j) Y[(size_t)j * r + i] = X[(size_t)i * c + j];
}

// The Polar Express iteration in place on X (r x c), after the Frobenius normalisation.
void polar_express(double *X, int r, int c, const double *coeffs, int ns, bool bf16) {
  const size_t n = (size_t)r * c;
  double ss = 0;
  for (size_t i = 0; i < n; ++i) ss += X[i] * X[i];
  double scale = 1.0 / (std::sqrt(ss) * 1.01 + 1e-6);
  if (bf16) scale = (double)(float)scale;
  for (size_t i = 0; i < n; ++i) X[i] = bf16 ? bf16r(X[i] * scale) : X[i] * scale;
  const bool tall = r > c;
  const int d = tall ? c : r;  // A and B are d x d
  std::vector<double> Xt(n), A((size_t)d * d), A2((size_t)d * d), Bm((size_t)d * d), XB(n);
  for (int it = 0; it < ns; ++it) {
    const double a = coeffs[3 * it], b = coeffs[3 * it + 1], cc = coeffs[3 * it + 2];
    transpose(X, r, c, Xt.data());
    if (tall) matmul(Xt.data(), X, c, r, c, A.data());   // A = X^T X
    else matmul(X, Xt.data(), r, c, r, A.data());        // A = X X^T
    round_all(A, bf16);
    matmul(A.data(), A.data(), d, d, d, A2.data());
    for (size_t i = 0; i < (size_t)d * d; ++i) Bm[i] = b * A[i] + cc * A2[i];
    round_all(Bm, bf16);
    if (tall) matmul(X, Bm.data(), r, c, c, XB.data());  // X B
    else matmul(Bm.data(), X, r, r, c, XB.data());       // B X
    for (size_t i = 0; i < n; ++i) X[i] = bf16 ? bf16r(a * X[i] + XB[i]) : a * X[i] + XB[i];
  }
}

}  // namespace

extern "C" {

void oracle_polar_express_f64(double *X, int rows, int cols, const double *coeffs, int ns,
                              int bf16) {
  polar_express(X, rows, cols, coeffs, ns, bf16 != 0);
}

double oracle_muon_adamw_f64(size_t n, double *p, const double *g, double *m, double *v,
                             int n_mat, const int64_t *mat_off, const int *mat_rows,
                             const int *mat_cols, double lr, double wd, double beta1,
                             double beta2, double eps, double matrix_lr, double muon_wd,
                             double mu, double beta2_muon, double s_eps, const double *coeffs,
                             int ns, double clip, long step, int bf16) {
  // global clip coefficient
  double ss = 0;
  for (size_t i = 0; i < n; ++i) ss += g[i] * g[i];
  const double norm = std::sqrt(ss);
  double coef = clip / (norm + 1e-6);
  if (coef > 1.0) coef = 1.0;
  // AdamW on every element outside the matrices (the order of the AdamW listing)
  std::vector<char> in_mat(n, 0);
  for (int k = 0; k < n_mat; ++k)
    for (int64_t i = 0; i < (int64_t)mat_rows[k] * mat_cols[k]; ++i) in_mat[mat_off[k] + i] = 1;
  const double bias1 = 1.0 - std::pow(beta1, (double)step);
  const double bias2 = 1.0 - std::pow(beta2, (double)step);
  for (size_t i = 0; i < n; ++i) {
    if (in_mat[i]) continue;
    const double gi = coef * g[i];
    p[i] = p[i] * (1.0 - lr * wd);
    m[i] = m[i] + (1.0 - beta1) * (gi - m[i]);
    v[i] = beta2 * v[i] + (1.0 - beta2) * gi * gi;
    const double denom = std::sqrt(v[i] / bias2) + eps;
    p[i] = p[i] - (lr / bias1) * m[i] / denom;
  }
  // Muon on each matrix: m holds the momentum, v (at the matrix's offset) the second moment
  for (int k = 0; k < n_mat; ++k) {
    const int r = mat_rows[k], c = mat_cols[k];
    const size_t cnt = (size_t)r * c, off = (size_t)mat_off[k];
    std::vector<double> X(cnt);
    for (size_t i = 0; i < cnt; ++i) {  // stage 1: momentum (Nesterov)
      const double gi = coef * g[off + i];
      m[off + i] = m[off + i] + (1.0 - mu) * (gi - m[off + i]);
      X[i] = gi + mu * (m[off + i] - gi);
      if (bf16) X[i] = bf16r(X[i]);  // X = g.bfloat16()
    }
    polar_express(X.data(), r, c, coeffs, ns, bf16 != 0);  // stage 2
    // stage 3: factored second moment, per row (tall) or per column (wide)
    const bool tall = r > c;
    const int nl = tall ? r : c;
    double *s = v + off;
    std::vector<double> line(nl, 0.0);
    for (int i = 0; i < r; ++i)
      for (int j = 0; j < c; ++j) line[tall ? i : j] += X[(size_t)i * c + j] * X[(size_t)i * c + j];
    for (int l = 0; l < nl; ++l) {
      const double vm = line[l] / (tall ? c : r);
      s[l] = s[l] + (1.0 - beta2_muon) * (vm - s[l]);
    }
    double n0 = 0, n1 = 0;
    std::vector<double> Y(cnt);
    for (int i = 0; i < r; ++i)
      for (int j = 0; j < c; ++j) {
        const double x = X[(size_t)i * c + j];
        const double y = x / std::sqrt(std::fmax(s[tall ? i : j], s_eps));
        Y[(size_t)i * c + j] = y;
        n0 += x * x;
        n1 += y * y;
      }
    const double gam = n1 > 0 ? std::sqrt(n0 / n1) : 0.0;
    // stage 4: cautious update
    for (size_t i = 0; i < cnt; ++i) {
      const double u = gam * Y[i];
      const double mask = (u * p[off + i] >= 0) ? 1.0 : 0.0;
      p[off + i] = p[off + i] - (matrix_lr * u + matrix_lr * muon_wd * p[off + i] * mask);
    }
  }
  return norm;
}

}  // extern "C"
