// Truncated SVD for the offline pack (SVDQuant review section 5, eq. 10):
// the leading singular triplets of the smoothed weight W~ (K x N, fp64).
//
// Method: the Gram matrix of the shorter side, G = A A^T (d x d, d =
// min(K, N)), then block subspace iteration with a Rayleigh-Ritz step per
// iteration (Jacobi on the small projected matrix), iterated until the
// residual of every wanted Ritz pair is below 1e-13 of the largest
// eigenvalue or stops improving.  Singular values are the square roots of
// the Ritz values; the other side's vectors come from one product with A.
// OpenMP parallelises the O(d^2 D) Gram and the O(d^2 p) products.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "svdq_internal.h"

namespace svdq {
namespace {

// G = A A^T for A d x D row-major; G d x d full (both triangles).
void gram_rows(const double* A, int d, long D, double* G) {
  const int T = 32;       // row tile
  const long KC = 512;    // column chunk kept in cache
  const int nb = (d + T - 1) / T;
  const long ntiles = (long)nb * (nb + 1) / 2;
#pragma omp parallel for schedule(dynamic, 1)
  for (long t = 0; t < ntiles; ++t) {
    int bi = (int)((std::sqrt(8.0 * (double)t + 1.0) - 1.0) / 2.0);
    while ((long)(bi + 1) * (bi + 2) / 2 <= t) ++bi;
    while ((long)bi * (bi + 1) / 2 > t) --bi;
    const int bj = (int)(t - (long)bi * (bi + 1) / 2);
    const int i0 = bi * T, j0 = bj * T;
    const int ni = std::min(T, d - i0), nj = std::min(T, d - j0);
    double acc[T][T];
    for (int a = 0; a < T; ++a)
      for (int b = 0; b < T; ++b) acc[a][b] = 0.0;
    for (long k0 = 0; k0 < D; k0 += KC) {
      const long kn = std::min(KC, D - k0);
      for (int a = 0; a < ni; a += 2) {
        const double* ra0 = A + (long)(i0 + a) * D + k0;
        const double* ra1 = (a + 1 < ni) ? ra0 + D : ra0;
        for (int b = 0; b < nj; b += 2) {
          const double* rb0 = A + (long)(j0 + b) * D + k0;
          const double* rb1 = (b + 1 < nj) ? rb0 + D : rb0;
          double s00 = 0, s01 = 0, s10 = 0, s11 = 0;
#pragma omp simd reduction(+ : s00, s01, s10, s11)
          for (long k = 0; k < kn; ++k) {
            s00 += ra0[k] * rb0[k];
            s01 += ra0[k] * rb1[k];
            s10 += ra1[k] * rb0[k];
            s11 += ra1[k] * rb1[k];
          }
          acc[a][b] += s00;
          if (b + 1 < nj) acc[a][b + 1] += s01;
          if (a + 1 < ni) {
            acc[a + 1][b] += s10;
            if (b + 1 < nj) acc[a + 1][b + 1] += s11;
          }
        }
      }
    }
    for (int a = 0; a < ni; ++a)
      for (int b = 0; b < nj; ++b) {
        G[(long)(i0 + a) * d + (j0 + b)] = acc[a][b];
        G[(long)(j0 + b) * d + (i0 + a)] = acc[a][b];
      }
  }
}

// Cyclic Jacobi eigen-decomposition of a symmetric n x n matrix H (row-major,
// destroyed).  On return evals[i] and column i of S (row-major n x n) hold
// the eigenpairs, sorted by decreasing eigenvalue.
void jacobi_eig(std::vector<double>& H, int n, std::vector<double>& evals,
                std::vector<double>& S) {
  S.assign((size_t)n * n, 0.0);
  for (int i = 0; i < n; ++i) S[(size_t)i * n + i] = 1.0;
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0, tot = 0.0;
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j) {
        double v = H[(size_t)i * n + j] * H[(size_t)i * n + j];
        tot += v;
        if (i != j) off += v;
      }
    if (off <= 1e-30 * tot || off == 0.0) break;
    for (int p = 0; p < n - 1; ++p)
      for (int q = p + 1; q < n; ++q) {
        const double apq = H[(size_t)p * n + q];
        if (apq == 0.0) continue;
        const double app = H[(size_t)p * n + p], aqq = H[(size_t)q * n + q];
        // rotation angle that annihilates H[p][q]
        const double theta = (aqq - app) / (2.0 * apq);
        const double tt = (theta >= 0 ? 1.0 : -1.0) /
                          (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(tt * tt + 1.0), s = tt * c;
        for (int k = 0; k < n; ++k) {  // rows p, q  (H <- J^T H)
          const double hp = H[(size_t)p * n + k], hq = H[(size_t)q * n + k];
          H[(size_t)p * n + k] = c * hp - s * hq;
          H[(size_t)q * n + k] = s * hp + c * hq;
        }
        for (int k = 0; k < n; ++k) {  // columns p, q  (H <- H J)
          const double hp = H[(size_t)k * n + p], hq = H[(size_t)k * n + q];
          H[(size_t)k * n + p] = c * hp - s * hq;
          H[(size_t)k * n + q] = s * hp + c * hq;
        }
        H[(size_t)p * n + q] = H[(size_t)q * n + p] = 0.0;
        for (int k = 0; k < n; ++k) {  // accumulate S <- S J
          const double sp = S[(size_t)k * n + p], sq = S[(size_t)k * n + q];
          S[(size_t)k * n + p] = c * sp - s * sq;
          S[(size_t)k * n + q] = s * sp + c * sq;
        }
      }
  }
  std::vector<int> idx(n);
  for (int i = 0; i < n; ++i) idx[i] = i;
  std::vector<double> diag(n);
  for (int i = 0; i < n; ++i) diag[i] = H[(size_t)i * n + i];
  std::stable_sort(idx.begin(), idx.end(),
                   [&](int a, int b) { return diag[a] > diag[b]; });
  std::vector<double> S2((size_t)n * n);
  evals.resize(n);
  for (int c = 0; c < n; ++c) {
    evals[c] = diag[idx[c]];
    for (int k = 0; k < n; ++k) S2[(size_t)k * n + c] = S[(size_t)k * n + idx[c]];
  }
  S.swap(S2);
}

// Deterministic pseudo-random fill (splitmix64) for the start block.
void random_fill(double* v, long n, uint64_t seed) {
  uint64_t x = seed;
  for (long i = 0; i < n; ++i) {
    x += 0x9E3779B97F4A7C15ull;
    uint64_t z = x;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    v[i] = (double)(z >> 11) * 0x1p-53 - 0.5;
  }
}

// Orthonormalise the p columns (column-major, length d) in place with
// modified Gram-Schmidt applied twice; a column that vanishes is replaced by
// a fresh random vector.  Serial; used when Cholesky QR breaks down.
void mgs(double* V, int d, int p, uint64_t seed) {
  for (int c = 0; c < p; ++c) {
    double* vc = V + (long)c * d;
    for (int attempt = 0; attempt < 4; ++attempt) {
      double before = 0.0;
      for (long i = 0; i < d; ++i) before += vc[i] * vc[i];
      for (int pass = 0; pass < 2; ++pass)
        for (int c2 = 0; c2 < c; ++c2) {
          const double* u = V + (long)c2 * d;
          double dot = 0.0;
          for (long i = 0; i < d; ++i) dot += u[i] * vc[i];
          for (long i = 0; i < d; ++i) vc[i] -= dot * u[i];
        }
      double nrm = 0.0;
      for (long i = 0; i < d; ++i) nrm += vc[i] * vc[i];
      if (nrm > 1e-24 * before && nrm > 0.0) {
        const double inv = 1.0 / std::sqrt(nrm);
        for (long i = 0; i < d; ++i) vc[i] *= inv;
        break;
      }
      random_fill(vc, d, seed + 7919u * (uint64_t)(c + 1) + (uint64_t)attempt);
    }
  }
}

// One Cholesky-QR pass: C = V^T V = L L^T, V <- V L^-T.  Returns false (V
// untouched) if C is numerically singular.
bool cholqr(double* V, int d, int p) {
  std::vector<double> C((size_t)p * p), L((size_t)p * p, 0.0);
#pragma omp parallel for schedule(dynamic, 1)
  for (int a = 0; a < p; ++a)
    for (int b = 0; b <= a; ++b) {
      const double* va = V + (long)a * d;
      const double* vb = V + (long)b * d;
      double s = 0.0;
#pragma omp simd reduction(+ : s)
      for (long i = 0; i < d; ++i) s += va[i] * vb[i];
      C[(size_t)a * p + b] = C[(size_t)b * p + a] = s;
    }
  for (int j = 0; j < p; ++j) {
    double s = C[(size_t)j * p + j];
    for (int k = 0; k < j; ++k) s -= L[(size_t)j * p + k] * L[(size_t)j * p + k];
    if (!(s > 1e-20 * C[(size_t)j * p + j]) || !(s > 0.0)) return false;
    const double ljj = std::sqrt(s);
    L[(size_t)j * p + j] = ljj;
    for (int i = j + 1; i < p; ++i) {
      double t = C[(size_t)i * p + j];
      for (int k = 0; k < j; ++k) t -= L[(size_t)i * p + k] * L[(size_t)j * p + k];
      L[(size_t)i * p + j] = t / ljj;
    }
  }
#pragma omp parallel
  {
    std::vector<double> x(p);
#pragma omp for schedule(static)
    for (long i = 0; i < d; ++i) {
      for (int c = 0; c < p; ++c) {
        double v = V[(long)c * d + i];
        for (int k = 0; k < c; ++k) v -= x[k] * L[(size_t)c * p + k];
        x[c] = v / L[(size_t)c * p + c];
      }
      for (int c = 0; c < p; ++c) V[(long)c * d + i] = x[c];
    }
  }
  return true;
}

void orthonormalize(double* V, int d, int p, uint64_t seed) {
  if (cholqr(V, d, p) && cholqr(V, d, p)) return;
  mgs(V, d, p, seed);
}

// Y = G V for G d x d row-major, V and Y column-major d x p.
void gemm_gv(const double* G, const double* V, int d, int p, double* Y) {
#pragma omp parallel for schedule(static)
  for (int i = 0; i < d; ++i) {
    const double* g = G + (long)i * d;
    for (int c = 0; c < p; ++c) {
      const double* v = V + (long)c * d;
      double s = 0.0;
#pragma omp simd reduction(+ : s)
      for (int k = 0; k < d; ++k) s += g[k] * v[k];
      Y[(long)c * d + i] = s;
    }
  }
}

// W = V S for V column-major d x p and S row-major p x p; W column-major d x q
// (first q columns of the product).
void times_small(const double* V, int d, int p, const std::vector<double>& S,
                 int q, double* W) {
#pragma omp parallel for schedule(static)
  for (int i = 0; i < d; ++i)
    for (int c = 0; c < q; ++c) {
      double s = 0.0;
      for (int k = 0; k < p; ++k) s += V[(long)k * d + i] * S[(size_t)k * p + c];
      W[(long)c * d + i] = s;
    }
}

}  // namespace

int top_singular(const double* A, int K, int N, int nsv, int r_out,
                 double* sigma, double* L1, double* L2) {
  const bool rows_side = K <= N;   // Gram of the rows of W~ (K x K)
  const int d = rows_side ? K : N;
  const long D = rows_side ? N : K;
  if (nsv < 1 || nsv > d) return -1;
  std::vector<double> At;
  const double* B = A;
  if (!rows_side) {   // B = A^T, N x K row-major
    At.resize((size_t)N * K);
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n)
      for (int k = 0; k < K; ++k) At[(size_t)n * K + k] = A[(size_t)k * N + n];
    B = At.data();
  }
  std::vector<double> G((size_t)d * d);
  gram_rows(B, d, D, G.data());

  const int p = std::min(d, std::max(nsv + 16, 2 * nsv));
  std::vector<double> V((size_t)d * p), Y((size_t)d * p), U((size_t)d * p),
      GU((size_t)d * p);
  random_fill(V.data(), (long)d * p, 0x5D5Full);
  orthonormalize(V.data(), d, p, 1234);
  std::vector<double> H((size_t)p * p), theta, S;
  double best = 1e300;
  int stall = 0;
  for (int it = 0; it < 4000; ++it) {
    gemm_gv(G.data(), V.data(), d, p, Y.data());
    // H = V^T Y (p x p), symmetrised
#pragma omp parallel for schedule(static)
    for (int a = 0; a < p; ++a)
      for (int b = 0; b < p; ++b) {
        double s = 0.0;
        for (long i = 0; i < d; ++i) s += V[(long)a * d + i] * Y[(long)b * d + i];
        H[(size_t)a * p + b] = s;
      }
    for (int a = 0; a < p; ++a)
      for (int b = a + 1; b < p; ++b) {
        const double m = 0.5 * (H[(size_t)a * p + b] + H[(size_t)b * p + a]);
        H[(size_t)a * p + b] = H[(size_t)b * p + a] = m;
      }
    jacobi_eig(H, p, theta, S);
    times_small(V.data(), d, p, S, p, U.data());    // Ritz vectors
    times_small(Y.data(), d, p, S, p, GU.data());   // G times them
    double worst = 0.0;
    for (int j = 0; j < nsv; ++j) {
      double r2 = 0.0;
      for (long i = 0; i < d; ++i) {
        const double e = GU[(long)j * d + i] - theta[j] * U[(long)j * d + i];
        r2 += e * e;
      }
      worst = std::max(worst, std::sqrt(r2));
    }
    const double scale = std::max(std::fabs(theta[0]), 1e-300);
    if (worst <= 1e-13 * scale) break;
    if (worst < 0.5 * best) { best = worst; stall = 0; }
    else if (++stall > 60) break;   // at the rounding floor
    V.swap(GU);
    orthonormalize(V.data(), d, p, 99 + it);
  }
  // U holds the Ritz vectors, theta the Ritz values.
  for (int j = 0; j < nsv; ++j) sigma[j] = std::sqrt(std::max(theta[j], 0.0));
  const int r = std::min(r_out, nsv);
  if (r <= 0) return 0;
  const double tiny = 1e-300;
  if (rows_side) {
    // L1 = U_r S_r (K x r); L2 = S_r^-1 U_r^T A (r x N)
    for (int k = 0; k < K; ++k)
      for (int j = 0; j < r; ++j) L1[(size_t)k * r + j] = U[(long)j * K + k] * sigma[j];
#pragma omp parallel for schedule(static)
    for (int j = 0; j < r; ++j) {
      double* row = L2 + (size_t)j * N;
      for (int n = 0; n < N; ++n) row[n] = 0.0;
      for (int k = 0; k < K; ++k) {
        const double u = U[(long)j * K + k];
        const double* a = A + (size_t)k * N;
        for (int n = 0; n < N; ++n) row[n] += u * a[n];
      }
      const double inv = sigma[j] > tiny ? 1.0 / sigma[j] : 0.0;
      for (int n = 0; n < N; ++n) row[n] *= inv;
      if (sigma[j] <= tiny)
        for (int k = 0; k < K; ++k) L1[(size_t)k * r + j] = 0.0;
    }
  } else {
    // L2 = V_r^T (r x N); L1 = A V_r (K x r)
    for (int j = 0; j < r; ++j)
      for (int n = 0; n < N; ++n) L2[(size_t)j * N + n] = U[(long)j * N + n];
#pragma omp parallel for schedule(static)
    for (int k = 0; k < K; ++k) {
      const double* a = A + (size_t)k * N;
      for (int j = 0; j < r; ++j) {
        double s = 0.0;
        const double* v = U.data() + (long)j * N;
        for (int n = 0; n < N; ++n) s += a[n] * v[n];
        L1[(size_t)k * r + j] = s;
      }
    }
  }
  return 0;
}

}  // namespace svdq
