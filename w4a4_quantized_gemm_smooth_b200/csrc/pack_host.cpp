// Host side of the C ABI: the offline pack (SVDQuant review section 5: the
// offline procedure, with or without the calibrated alpha search and the
// alternating factor refinement), handle management, export, save/load.
//
// Exactness contract with the checks: every rounding below is a single IEEE
// rounding of a value that both sides define the same way, so the codes and
// scales of the quantised residual are reproducible bit for bit:
//   lambda (eq. 4, alpha = 0.5) = sqrt(a) / sqrt(w)   (fp64, correctly rounded)
//   inv_lambda = fl32(1 / lambda)
//   W~ = lambda_k * W[k][n]                           (fp64, eq. 3)
//   R = W~ - sum_j L1b[k][j] L2b[j][n], j ascending   (fp64; the products of
//       two bf16 values are exact, each subtraction is rounded once)
//   s = fl32(max|fl32(R)| / 7), codes = rne of the exact quotient  (eq. 1)
//   W8A8 comparator: s = fl32(max|fl32(R)| / 127) per output column over
//   all K, codes rne of the exact quotient clamped to [-128, 127]
//   NVFP4 variant: s = fl32(max|fl32(R)| / 2688) per output column,
//   b = e4m3(fl32(max|group of 16| / fl32(6 s))), codes e2m1 of the exact
//   quotient z / (b s), nearest with ties to even
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "svdq_internal.h"

namespace {

uint32_t f32_bits(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }
float bits_f32(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }

double bf16_to_f64(uint16_t b) { return (double)bits_f32((uint32_t)b << 16); }

// One round-to-nearest-even rounding of an fp64 value to bf16 (8 significant
// bits, fp32's exponent range, subnormal quantum 2^-133).
uint16_t f64_to_bf16(double x) {
  if (std::isnan(x)) return 0x7FC0;
  const double ax = std::fabs(x);
  if (ax == 0.0) return std::signbit(x) ? 0x8000 : 0x0000;
  double y;
  if (ax < 0x1p-126) {
    y = std::nearbyint(x * 0x1p133) * 0x1p-133;   // exact scalings
  } else {
    uint64_t u;
    std::memcpy(&u, &x, 8);
    const uint64_t keep = (u >> 45) & 1u;          // lsb of the kept part
    u += ((uint64_t)1 << 44) - 1 + keep;
    u &= ~(((uint64_t)1 << 45) - 1);
    std::memcpy(&y, &u, 8);
    if (std::fabs(y) >= 0x1p128) return std::signbit(x) ? 0xFF80 : 0x7F80;
  }
  return (uint16_t)(f32_bits((float)y) >> 16);     // exact conversion
}

// Eq. 1 on one group of 64 fp32 values: scale and codes.
float quantize_group(const float* z, int stride, int8_t* q) {
  float m = 0.0f;
  for (int i = 0; i < 64; ++i) m = std::fmax(m, std::fabs(z[(long)i * stride]));
  const float s = m / 7.0f;    // IEEE fp32 division
  if (s == 0.0f) {
    for (int i = 0; i < 64; ++i) q[i] = 0;
    return 0.0f;
  }
  const double sd = s;
  for (int i = 0; i < 64; ++i) {
    const double zd = z[(long)i * stride];
    double c = std::nearbyint(zd / sd);
    for (int it = 0; it < 2; ++it) {
      const double d2 = 2.0 * (zd - c * sd);          // exact
      if (d2 > sd) c += 1.0;
      else if (d2 < -sd) c -= 1.0;
    }
    const double d2 = 2.0 * (zd - c * sd);
    if (std::fabs(d2) == sd && std::fmod(c, 2.0) != 0.0) c += (d2 > 0 ? 1.0 : -1.0);
    if (c > 7.0) c = 7.0;
    if (c < -8.0) c = -8.0;
    q[i] = (int8_t)c;
  }
  return s;
}

// The comparator's int8 quantiser: one scale for n fp32 values.
float quantize_row_int8(const float* z, int n, long stride, int8_t* q) {
  float m = 0.0f;
  for (int i = 0; i < n; ++i) m = std::fmax(m, std::fabs(z[(long)i * stride]));
  const float s = m / 127.0f;  // IEEE fp32 division
  if (s == 0.0f) {
    for (int i = 0; i < n; ++i) q[i] = 0;
    return 0.0f;
  }
  const double sd = s;
  for (int i = 0; i < n; ++i) {
    const double zd = z[(long)i * stride];
    double c = std::nearbyint(zd / sd);
    for (int it = 0; it < 2; ++it) {
      const double d2 = 2.0 * (zd - c * sd);          // exact (c s has <= 31 bits)
      if (d2 > sd) c += 1.0;
      else if (d2 < -sd) c -= 1.0;
    }
    const double d2 = 2.0 * (zd - c * sd);
    if (std::fabs(d2) == sd && std::fmod(c, 2.0) != 0.0) c += (d2 > 0 ? 1.0 : -1.0);
    if (c > 127.0) c = 127.0;
    if (c < -128.0) c = -128.0;
    q[i] = (int8_t)c;
  }
  return s;
}

// FP8 E4M3 rounding of a non-negative value: 4 significant bits, exponent
// bias 7, subnormal quantum 2^-9, nearest with ties to even, saturating at
// 448 (the largest finite value).
double round_e4m3(double t) {
  if (!(t > 0.0)) return 0.0;
  int e = 0;
  std::frexp(t, &e);                                  // t = f 2^e, 0.5 <= f < 1
  const int qexp = e - 4 > -9 ? e - 4 : -9;
  const double v = std::ldexp(std::nearbyint(std::ldexp(t, -qexp)), qexp);
  return v < 448.0 ? v : 448.0;
}

uint8_t e4m3_bits(double v) {
  if (!(v > 0.0)) return 0;
  if (v < 0x1p-6) return (uint8_t)std::nearbyint(v * 512.0);   // subnormal: m 2^-9
  int e = 0;
  const double f = std::frexp(v, &e);
  return (uint8_t)(((e - 1 + 7) << 3) | (int)std::nearbyint((2.0 * f - 1.0) * 8.0));
}

// FP4 E2M1 code of the exact quotient z / d (d > 0): index into
// {0, .5, 1, 1.5, 2, 3, 4, 6} by exact comparisons with the midpoints times
// d (each product has at most 31 significant bits), ties to the even index,
// saturating at 6; bit 3 is the sign of a nonzero magnitude.
uint8_t e2m1_code(double z, double d) {
  static const double mids[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
  const double a = std::fabs(z);
  int idx = 0;
  while (idx < 7 && mids[idx] * d < a) ++idx;
  if (idx < 7 && mids[idx] * d == a && (idx & 1)) ++idx;
  return (uint8_t)(idx | ((z < 0.0 && idx > 0) ? 8 : 0));
}

// The NVFP4 rule on one row of K fp32 values (stride between elements):
// packed codes (K/2 bytes, even k in the low nibble), E4M3 group scale bits
// (K/16 bytes), and the row scale.
float quantize_row_nvfp4(const float* z, int K, long stride, uint8_t* codes, uint8_t* sf) {
  float m = 0.0f;
  for (int i = 0; i < K; ++i) m = std::fmax(m, std::fabs(z[(long)i * stride]));
  const float srow = m / 2688.0f;                      // IEEE fp32 division
  const float d6 = 6.0f * srow;                        // IEEE fp32 product
  for (int g = 0; g < K / 16; ++g) {
    float mg = 0.0f;
    for (int i = 0; i < 16; ++i) mg = std::fmax(mg, std::fabs(z[(long)(16 * g + i) * stride]));
    const double b = d6 > 0.0f ? round_e4m3((double)(mg / d6)) : 0.0;
    sf[g] = e4m3_bits(b);
    const double d = b * (double)srow;                 // exact
    for (int i = 0; i < 16; i += 2) {
      const uint8_t c0 = d > 0.0 ? e2m1_code(z[(long)(16 * g + i) * stride], d) : 0;
      const uint8_t c1 = d > 0.0 ? e2m1_code(z[(long)(16 * g + i + 1) * stride], d) : 0;
      codes[8 * g + i / 2] = (uint8_t)(c0 | (c1 << 4));
    }
  }
  return srow;
}

template <class T>
svdq_status dev_alloc_copy(T** dst, const T* src, size_t n, cudaStream_t st) {
  if (n == 0) n = 1;
  if (cudaMalloc((void**)dst, n * sizeof(T)) != cudaSuccess) return SVDQ_ERR_OOM;
  if (src && cudaMemcpyAsync(*dst, src, n * sizeof(T), cudaMemcpyHostToDevice, st) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return SVDQ_OK;
}

void free_device(svdq_weights* w) {
  cudaFree(w->d_inv_lambda); cudaFree(w->d_wq); cudaFree(w->d_sw); cudaFree(w->d_wcs);
  cudaFree(w->d_L1T); cudaFree(w->d_L2); cudaFree(w->d_L2T); cudaFree(w->d_bias);
  cudaFree(w->d_wq8); cudaFree(w->d_sw8);
  cudaFree(w->d_wq4); cudaFree(w->d_sfb4); cudaFree(w->d_sw4);
  cudaFree(w->d_err);
  w->d_wq8 = nullptr; w->d_sw8 = nullptr;
  w->d_wq4 = nullptr; w->d_sfb4 = nullptr; w->d_sw4 = nullptr;
  w->d_inv_lambda = nullptr; w->d_wq = nullptr; w->d_sw = nullptr; w->d_wcs = nullptr;
  w->d_L1T = nullptr;
  w->d_L2 = nullptr; w->d_L2T = nullptr; w->d_bias = nullptr; w->d_err = nullptr;
}

}  // namespace

namespace svdq {

svdq_status upload(svdq_weights* w, cudaStream_t st) {
  if (cudaGetDevice(&w->device) != cudaSuccess) return SVDQ_ERR_CUDA;
  const int K = w->K, N = w->N, G = w->G, rp = w->rank_pad;
  w->rank_pad32 = (w->rank + 31) / 32 * 32;
  w->N_pad = (N + 255) / 256 * 256;
  const int rp32 = w->rank_pad32;
  std::vector<uint16_t> L1T((size_t)rp * K, 0), L2p((size_t)rp * N, 0),
      L2T((size_t)w->N_pad * (rp32 > 0 ? rp32 : 1), 0);
  for (int j = 0; j < w->rank; ++j)
    for (int n = 0; n < N; ++n) L2T[(size_t)n * rp32 + j] = w->L2[(size_t)j * N + n];
  for (int j = 0; j < w->rank; ++j)
    for (int k = 0; k < K; ++k) L1T[(size_t)j * K + k] = w->L1[(size_t)k * w->rank + j];
  for (int j = 0; j < w->rank; ++j)
    std::memcpy(&L2p[(size_t)j * N], &w->L2[(size_t)j * N], (size_t)N * 2);
  svdq_status s;
  if ((s = dev_alloc_copy(&w->d_inv_lambda, w->inv_lambda.data(), (size_t)K, st))) return s;
  w->N16 = (N + 15) / 16 * 16;
  if (w->format == SVDQ_FORMAT_NVFP4) {
    std::vector<float> swp((size_t)w->N_pad, 0.0f);
    std::memcpy(swp.data(), w->sw4.data(), (size_t)N * 4);
    std::vector<uint8_t> sfb(svdq::nvfp4_sf_bytes(N, K), 0);
    for (int n = 0; n < N; ++n)
      for (int g = 0; g < K / 16; ++g)
        sfb[svdq::nvfp4_sf_offset(n, g, K)] = w->sf4[(size_t)n * (K / 16) + g];
    if ((s = dev_alloc_copy(&w->d_wq4, w->wq4.data(), (size_t)N * K / 2, st))) return s;
    if ((s = dev_alloc_copy(&w->d_sfb4, sfb.data(), sfb.size(), st))) return s;
    if ((s = dev_alloc_copy(&w->d_sw4, swp.data(), swp.size(), st))) return s;
  } else if (w->format == SVDQ_FORMAT_W8A8) {
    std::vector<float> sw8p((size_t)w->N_pad, 0.0f);
    std::memcpy(sw8p.data(), w->sw8.data(), (size_t)N * 4);
    if ((s = dev_alloc_copy(&w->d_wq8, w->wq8.data(), (size_t)N * K, st))) return s;
    if ((s = dev_alloc_copy(&w->d_sw8, sw8p.data(), sw8p.size(), st))) return s;
  } else {
    // device codes: sign-magnitude nibbles unless some code is -8
    const size_t nb = (size_t)N * K / 2;
    w->wq_twos = false;
    for (size_t i = 0; i < nb && !w->wq_twos; ++i)
      w->wq_twos = (w->wq[i] & 0x0F) == 0x08 || (w->wq[i] & 0xF0) == 0x80;
    std::vector<uint8_t> wqd(w->wq);
    if (!w->wq_twos) {
      for (size_t i = 0; i < nb; ++i) {
        uint8_t out = 0;
        for (int h = 0; h < 2; ++h) {
          const int q = (int)(int8_t)(uint8_t)(((w->wq[i] >> (4 * h)) & 0x0F) << 4) >> 4;
          const uint8_t n = (uint8_t)((q < 0 ? 8 : 0) | (q < 0 ? -q : q));
          out |= (uint8_t)(n << (4 * h));
        }
        wqd[i] = out;
      }
    }
    if ((s = dev_alloc_copy(&w->d_wq, wqd.data(), nb, st))) return s;
    std::vector<float> swp((size_t)G * w->N16, 0.0f);
    for (int g = 0; g < G; ++g)
      for (int n = 0; n < N; ++n) {
        const int c = n & 15, pos = (n & ~15) + 4 * ((c & 7) >> 1) + 2 * (c >> 3) + (c & 1);
        const double v = (double)w->sw[(size_t)g * N + n];
        if (!(v < SVDQ_SW_LIMIT)) return SVDQ_ERR_NUMERIC;
        swp[(size_t)g * w->N16 + pos] = (float)std::ldexp(v, 18);   // exact
      }
    if ((s = dev_alloc_copy(&w->d_sw, swp.data(), swp.size(), st))) return s;
    // per group and column: -sum_k q_w = d0 + 8 d1 + 64 d2 with d0, d1 in
    // [-4, 3] (balanced base 8) and |d2| <= 8, each as the E4M3 byte of d 2^-9
    std::vector<uint32_t> wcs((size_t)G * w->N_pad, 0u);
    auto e4m3_int = [](int d) -> uint32_t { return (uint32_t)((d < 0 ? 0x80 : 0) | (d < 0 ? -d : d)); };
    for (int n = 0; n < N; ++n)
      for (int g = 0; g < G; ++g) {
        int cs = 0;
        for (int k = 64 * g; k < 64 * g + 64; ++k) {
          const uint8_t b = w->wq[(size_t)n * (K / 2) + k / 2];
          cs += (int)(int8_t)(uint8_t)(((b >> (4 * (k & 1))) & 0x0F) << 4) >> 4;
        }
        const int v = -cs;
        const int d0 = ((v % 8) + 8 + 4) % 8 - 4;
        const int v1 = (v - d0) / 8;
        const int d1 = ((v1 % 8) + 8 + 4) % 8 - 4;
        const int d2 = (v1 - d1) / 8;
        if (d0 + 8 * d1 + 64 * d2 != v || d2 < -8 || d2 > 8) return SVDQ_ERR_NUMERIC;   // |cs| <= 512
        wcs[(size_t)g * w->N_pad + n] = e4m3_int(d0) | (e4m3_int(d1) << 8) | (e4m3_int(d2) << 16);
      }
    if ((s = dev_alloc_copy(&w->d_wcs, wcs.data(), wcs.size(), st))) return s;
  }
  if ((s = dev_alloc_copy(&w->d_L1T, L1T.data(), L1T.size(), st))) return s;
  if ((s = dev_alloc_copy(&w->d_L2, L2p.data(), L2p.size(), st))) return s;
  if ((s = dev_alloc_copy(&w->d_L2T, L2T.data(), L2T.size(), st))) return s;
  if ((s = dev_alloc_copy(&w->d_bias, w->bias.data(), (size_t)N, st))) return s;
  if ((s = dev_alloc_copy<int>(&w->d_err, nullptr, 1, st))) return s;
  if (cudaMemsetAsync(w->d_err, 0, sizeof(int), st) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SVDQ_ERR_CUDA;
  return SVDQ_OK;
}

}  // namespace svdq

namespace {

// One candidate of the offline pack: smoothing, protected factors and the
// quantised residual (math layout: K input channels x N output channels).
struct Candidate {
  std::vector<double> lam, Wt;     // lambda [K]; W~ = diag(lambda) W [K][N]
  std::vector<float> inv_lambda;   // fl32(1 / lambda)
  std::vector<double> sigma;       // leading singular values [rank + 1]
  std::vector<uint16_t> L1, L2;    // bf16 factors [K][rank], [rank][N]
  std::vector<uint8_t> wq;         // packed residual codes [N][K/2]
  std::vector<float> sw;           // residual scales [G][N]
  std::vector<int8_t> wq8;         // W8A8 comparator: codes [N][K]
  std::vector<float> sw8;          //                  scales [N]
  std::vector<uint8_t> wq4;        // NVFP4: packed codes [N][K/2]
  std::vector<uint8_t> sf4;        //        E4M3 group scales [N][K/16]
  std::vector<float> sw4;          //        row scales [N]
};

// eqs. 3-4: lambda from the activation statistic and the weight's per-channel
// absmax (lambda = 1 where either is 0), then W~.
svdq_status smooth(int K, int N, const uint16_t* W, const float* act_absmax, double alpha,
                   Candidate& c) {
  for (int k = 0; k < K; ++k) {
    const double a = act_absmax[k];
    if (!std::isfinite(a) || a < 0) return SVDQ_ERR_NUMERIC;
  }
  std::vector<double> wmax(K, 0.0);
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) {
      const double v = bf16_to_f64(W[(size_t)n * K + k]);
      if (!std::isfinite(v)) return SVDQ_ERR_NUMERIC;
      wmax[k] = std::fmax(wmax[k], std::fabs(v));
    }
  c.lam.assign(K, 1.0);
  c.inv_lambda.resize(K);
  for (int k = 0; k < K; ++k) {
    const double a = act_absmax[k], m = wmax[k];
    double l = 1.0;
    if (a > 0.0 && m > 0.0)
      l = (alpha == 0.5) ? std::sqrt(a) / std::sqrt(m)
                         : std::pow(a, alpha) / std::pow(m, 1.0 - alpha);
    c.lam[k] = l;
    c.inv_lambda[k] = (float)(1.0 / l);
  }
  c.Wt.resize((size_t)K * N);
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k)
      c.Wt[(size_t)k * N + n] = c.lam[k] * bf16_to_f64(W[(size_t)n * K + k]);
  return SVDQ_OK;
}

// eq. 10: the rank-r factors of T (stored as bf16) and T's leading singular
// values.
svdq_status fit_factors(const double* T, int K, int N, int rank, Candidate& c) {
  const int nsv = std::min(rank + 1, std::min(K, N));
  std::vector<double> sig(nsv), L1((size_t)K * (rank > 0 ? rank : 1)),
      L2((size_t)(rank > 0 ? rank : 1) * N);
  if (svdq::top_singular(T, K, N, nsv, rank, sig.data(), L1.data(), L2.data()))
    return SVDQ_ERR_NUMERIC;
  c.sigma.assign(rank + 1, 0.0);
  for (int j = 0; j < nsv; ++j) c.sigma[j] = sig[j];
  c.L1.assign((size_t)K * rank, 0);
  c.L2.assign((size_t)rank * N, 0);
  for (int k = 0; k < K; ++k)
    for (int j = 0; j < rank; ++j) c.L1[(size_t)k * rank + j] = f64_to_bf16(L1[(size_t)k * rank + j]);
  for (int j = 0; j < rank; ++j)
    for (int n = 0; n < N; ++n) c.L2[(size_t)j * N + n] = f64_to_bf16(L2[(size_t)j * N + n]);
  return SVDQ_OK;
}

// fl32(R), R = W~ - L1b L2b against the stored factors (j ascending, fp64),
// [K][N].
std::vector<float> residual_f32(int K, int N, int rank, const Candidate& c) {
  std::vector<float> R32((size_t)K * N);
#pragma omp parallel for schedule(static)
  for (int k = 0; k < K; ++k) {
    std::vector<double> row(c.Wt.begin() + (size_t)k * N, c.Wt.begin() + (size_t)(k + 1) * N);
    for (int j = 0; j < rank; ++j) {
      const double a = bf16_to_f64(c.L1[(size_t)k * rank + j]);
      const uint16_t* l2 = &c.L2[(size_t)j * N];
      for (int n = 0; n < N; ++n) row[n] -= a * bf16_to_f64(l2[n]);
    }
    for (int n = 0; n < N; ++n) R32[(size_t)k * N + n] = (float)row[n];
  }
  return R32;
}

// The residual, then eq. 1 per (output column, group of 64 input channels).
void quantize_residual(int K, int N, int rank, Candidate& c) {
  const std::vector<float> R32 = residual_f32(K, N, rank, c);
  const int G = K / SVDQ_GROUP;
  c.sw.assign((size_t)G * N, 0.0f);
  c.wq.assign((size_t)N * K / 2, 0);
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    int8_t q[64];
    for (int g = 0; g < G; ++g) {
      c.sw[(size_t)g * N + n] = quantize_group(&R32[(size_t)g * 64 * N + n], N, q);
      uint8_t* dst = &c.wq[(size_t)n * (K / 2) + g * 32];
      for (int b = 0; b < 32; ++b)
        dst[b] = (uint8_t)((q[2 * b] & 0xF) | ((q[2 * b + 1] & 0xF) << 4));
    }
  }
}

// The residual, then the comparator's int8 quantiser per output column.
void quantize_residual_w8(int K, int N, int rank, Candidate& c) {
  const std::vector<float> R32 = residual_f32(K, N, rank, c);
  c.sw8.assign(N, 0.0f);
  c.wq8.assign((size_t)N * K, 0);
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n)
    c.sw8[n] = quantize_row_int8(&R32[n], K, N, &c.wq8[(size_t)n * K]);
}

// The residual, then the NVFP4 rule per output column.
void quantize_residual_nvfp4(int K, int N, int rank, Candidate& c) {
  const std::vector<float> R32 = residual_f32(K, N, rank, c);
  c.sw4.assign(N, 0.0f);
  c.wq4.assign((size_t)N * K / 2, 0);
  c.sf4.assign((size_t)N * K / 16, 0);
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n)
    c.sw4[n] = quantize_row_nvfp4(&R32[n], K, N, &c.wq4[(size_t)n * K / 2], &c.sf4[(size_t)n * K / 16]);
}

int8_t code_at(const std::vector<uint8_t>& wq, int K, int n, int k) {
  const uint8_t b = wq[(size_t)n * (K / 2) + k / 2];
  const int v = (k & 1) ? (b >> 4) : (b & 0xF);
  return (int8_t)(v >= 8 ? v - 16 : v);
}

// ---------------------------------------------------------------- GPTQ
// The residual rounded by GPTQ (the review's offline procedure: "residual
// weights use GPTQ"; the published algorithm of Frantar et al.) on the
// Hessian H = X~^T X~ of the calibration tokens in smoothed coordinates.

// Exact round-half-even of zd / sd (sd > 0), clamped to [-8, 7].
int code_of(double zd, double sd) {
  double c = std::nearbyint(zd / sd);
  for (int it = 0; it < 2; ++it) {
    const double d2 = 2.0 * (zd - c * sd);          // exact
    if (d2 > sd) c += 1.0;
    else if (d2 < -sd) c -= 1.0;
  }
  const double d2 = 2.0 * (zd - c * sd);
  if (std::fabs(d2) == sd && std::fmod(c, 2.0) != 0.0) c += (d2 > 0 ? 1.0 : -1.0);
  return (int)std::fmax(-8.0, std::fmin(7.0, c));
}

// In-place lower Cholesky factor of the symmetric positive definite n x n
// row-major A (only the lower triangle is read and written).
bool cholesky_lower(std::vector<double>& A, int n) {
  for (int j = 0; j < n; ++j) {
    double d = A[(size_t)j * n + j];
    for (int k = 0; k < j; ++k) d -= A[(size_t)j * n + k] * A[(size_t)j * n + k];
    if (!(d > 0.0)) return false;
    d = std::sqrt(d);
    A[(size_t)j * n + j] = d;
#pragma omp parallel for schedule(static)
    for (int i = j + 1; i < n; ++i) {
      double v = A[(size_t)i * n + j];
      for (int k = 0; k < j; ++k) v -= A[(size_t)i * n + k] * A[(size_t)j * n + k];
      A[(size_t)i * n + j] = v / d;
    }
  }
  return true;
}

// U (upper, row-major) with H^-1 = U^T U for the dampened Hessian: H + damp
// mean(diag H) I, a channel the calibration never activates given H_kk = 1.
svdq_status gptq_factor(std::vector<double> H, int K, std::vector<double>& U) {
  double mean = 0.0;
  for (int k = 0; k < K; ++k) {
    if (H[(size_t)k * K + k] == 0.0) H[(size_t)k * K + k] = 1.0;
    mean += H[(size_t)k * K + k];
  }
  mean /= K;
  for (int k = 0; k < K; ++k) H[(size_t)k * K + k] += 0.01 * mean;
  if (!cholesky_lower(H, K)) return SVDQ_ERR_NUMERIC;         // H = L L^T
  // Linv = L^-1 (lower), column by column by forward substitution; stored
  // transposed (LinvT[c][i] = Linv[i][c]) so that every inner sum below runs
  // over contiguous memory
  std::vector<double> LinvT((size_t)K * K, 0.0);
#pragma omp parallel for schedule(dynamic)
  for (int c = 0; c < K; ++c) {
    double* lc = &LinvT[(size_t)c * K];
    for (int i = c; i < K; ++i) {
      double v = (i == c) ? 1.0 : 0.0;
      const double* hi = &H[(size_t)i * K];
      for (int k = c; k < i; ++k) v -= hi[k] * lc[k];
      lc[i] = v / hi[i];
    }
  }
  // Hinv = Linv^T Linv (symmetric; lower triangle suffices for the next factor)
  std::vector<double> Hinv((size_t)K * K, 0.0);
#pragma omp parallel for schedule(dynamic)
  for (int i = 0; i < K; ++i) {
    const double* li = &LinvT[(size_t)i * K];
    for (int j = 0; j <= i; ++j) {
      const double* lj = &LinvT[(size_t)j * K];
      double v = 0.0;
      for (int k = i; k < K; ++k) v += li[k] * lj[k];
      Hinv[(size_t)i * K + j] = v;
    }
  }
  if (!cholesky_lower(Hinv, K)) return SVDQ_ERR_NUMERIC;       // Hinv = L2 L2^T
  U.assign((size_t)K * K, 0.0);
  for (int i = 0; i < K; ++i)
    for (int j = 0; j <= i; ++j) U[(size_t)j * K + i] = Hinv[(size_t)i * K + j];   // U = L2^T
  return SVDQ_OK;
}

// H = X~^T X~ in fp64 over the calibration tokens, X~ = fl32(x inv_lambda).
std::vector<double> gptq_hessian(int K, const uint16_t* X, int M, int ldx,
                                 const std::vector<float>& inv_lambda) {
  std::vector<double> XT((size_t)K * M);
  for (int m = 0; m < M; ++m)
    for (int k = 0; k < K; ++k)
      XT[(size_t)k * M + m] = (double)(float)(bf16_to_f64(X[(size_t)m * ldx + k]) * (double)inv_lambda[k]);
  std::vector<double> H((size_t)K * K);
#pragma omp parallel for schedule(dynamic)
  for (int i = 0; i < K; ++i)
    for (int j = 0; j <= i; ++j) {
      double v = 0.0;
      for (int m = 0; m < M; ++m) v += XT[(size_t)i * M + m] * XT[(size_t)j * M + m];
      H[(size_t)i * K + j] = v;
      H[(size_t)j * K + i] = v;
    }
  return H;
}

// The residual R = W~ - L1b L2b, then GPTQ per output column (the columns
// are independent): on entering a group of 64 the eq. 1 scale comes from the
// updated group; channel k's error (w - q s) / U_kk moves the later channels
// by U_kj.  Columns are taken in batches of GPTQ_NB so that each row of U is
// read once per batch (the loop over a batch's columns is innermost); every
// column sees exactly the operations, in the same order, of a column-by-
// column loop.
constexpr int GPTQ_NB = 16;
void gptq_residual(int K, int N, int rank, const std::vector<double>& U, Candidate& c) {
  const int G = K / SVDQ_GROUP;
  c.sw.assign((size_t)G * N, 0.0f);
  c.wq.assign((size_t)N * K / 2, 0);
  const int nbat = (N + GPTQ_NB - 1) / GPTQ_NB;
#pragma omp parallel for schedule(dynamic)
  for (int bi = 0; bi < nbat; ++bi) {
    const int n0 = bi * GPTQ_NB;
    const int nb = N - n0 < GPTQ_NB ? N - n0 : GPTQ_NB;
    std::vector<double> r((size_t)K * GPTQ_NB, 0.0);    // r[k][b]
    for (int k = 0; k < K; ++k)
      for (int b = 0; b < nb; ++b) {
        double v = c.Wt[(size_t)k * N + n0 + b];
        for (int j = 0; j < rank; ++j)
          v -= bf16_to_f64(c.L1[(size_t)k * rank + j]) * bf16_to_f64(c.L2[(size_t)j * N + n0 + b]);
        r[(size_t)k * GPTQ_NB + b] = v;
      }
    std::vector<int8_t> q((size_t)GPTQ_NB * K);
    float s[GPTQ_NB] = {};
    double err[GPTQ_NB] = {};
    for (int k = 0; k < K; ++k) {
      if (k % SVDQ_GROUP == 0) {
        for (int b = 0; b < nb; ++b) {
          float m = 0.0f;
          for (int i = 0; i < SVDQ_GROUP; ++i)
            m = std::fmax(m, std::fabs((float)r[(size_t)(k + i) * GPTQ_NB + b]));
          s[b] = m / 7.0f;
          c.sw[(size_t)(k / SVDQ_GROUP) * N + n0 + b] = s[b];
        }
      }
      const double ukk = U[(size_t)k * K + k];
      for (int b = 0; b < nb; ++b) {
        const double rk = r[(size_t)k * GPTQ_NB + b];
        const int qk = s[b] > 0.0f ? code_of((double)(float)rk, (double)s[b]) : 0;
        q[(size_t)b * K + k] = (int8_t)qk;
        err[b] = (rk - (double)qk * (double)s[b]) / ukk;
      }
      for (int b = nb; b < GPTQ_NB; ++b) err[b] = 0.0;
      const double* urow = &U[(size_t)k * K];
      for (int j = k + 1; j < K; ++j) {
        const double u = urow[j];
        double* rj = &r[(size_t)j * GPTQ_NB];
#pragma omp simd
        for (int b = 0; b < GPTQ_NB; ++b) rj[b] -= u * err[b];
      }
    }
    for (int b = 0; b < nb; ++b) {
      uint8_t* dst = &c.wq[(size_t)(n0 + b) * (K / 2)];
      const int8_t* qb = &q[(size_t)b * K];
      for (int t = 0; t < K / 2; ++t)
        dst[t] = (uint8_t)((qb[2 * t] & 0xF) | ((qb[2 * t + 1] & 0xF) << 4));
    }
  }
}

// One alternating refinement: the factors of W~ - deq(Q(R)), then R again.
svdq_status refine(int K, int N, int rank, Candidate& c, const std::vector<double>* U) {
  std::vector<double> T(c.Wt);
#pragma omp parallel for schedule(static)
  for (int k = 0; k < K; ++k)
    for (int n = 0; n < N; ++n)
      T[(size_t)k * N + n] -= (double)code_at(c.wq, K, n, k) * (double)c.sw[(size_t)(k / 64) * N + n];
  const svdq_status s = fit_factors(T.data(), K, N, rank, c);
  if (s != SVDQ_OK) return s;
  if (U) gptq_residual(K, N, rank, *U, c);
  else quantize_residual(K, N, rank, c);
  return SVDQ_OK;
}

// X W in fp64 on M tokens, [M][N] (the reference of layer_error).
std::vector<double> dense_reference(int K, int N, const uint16_t* W, const uint16_t* X, int M,
                                    int ldx) {
  std::vector<double> ref((size_t)M * N);
#pragma omp parallel for schedule(dynamic)
  for (int m = 0; m < M; ++m) {
    std::vector<double> x(K);
    for (int k = 0; k < K; ++k) x[k] = bf16_to_f64(X[(size_t)m * ldx + k]);
    for (int n = 0; n < N; ++n) {
      const uint16_t* wr = &W[(size_t)n * K];
      double t = 0.0;
      for (int k = 0; k < K; ++k) t += x[k] * bf16_to_f64(wr[k]);
      ref[(size_t)m * N + n] = t;
    }
  }
  return ref;
}

// Relative Frobenius error, in fp64, of the quantised layer (both branches,
// no bias, before the bf16 output rounding) against ref = X W on M tokens.
double layer_error(int K, int N, int rank, const Candidate& c, const std::vector<double>& refm,
                   const uint16_t* X, int M, int ldx) {
  const int G = K / SVDQ_GROUP;
  std::vector<int8_t> wc((size_t)N * K);
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) wc[(size_t)n * K + k] = code_at(c.wq, K, n, k);
  double num = 0.0, den = 0.0;
#pragma omp parallel for schedule(dynamic) reduction(+ : num, den)
  for (int m = 0; m < M; ++m) {
    std::vector<float> xh(K);
    std::vector<double> x(K), z(rank > 0 ? rank : 1, 0.0);
    std::vector<int8_t> xc(K);
    std::vector<float> sx(G);
    for (int k = 0; k < K; ++k) {
      x[k] = bf16_to_f64(X[(size_t)m * ldx + k]);
      xh[k] = (float)(x[k] * (double)c.inv_lambda[k]);     // one rounding of an exact product
    }
    for (int g = 0; g < G; ++g) sx[g] = quantize_group(&xh[(size_t)g * 64], 1, &xc[(size_t)g * 64]);
    for (int j = 0; j < rank; ++j) {
      double t = 0.0;
      for (int k = 0; k < K; ++k)
        t += bf16_to_f64(f64_to_bf16((double)xh[k])) * bf16_to_f64(c.L1[(size_t)k * rank + j]);
      z[j] = bf16_to_f64(f64_to_bf16(t));
    }
    for (int n = 0; n < N; ++n) {
      double y = 0.0, ref = 0.0;
      const int8_t* wn = &wc[(size_t)n * K];
      for (int g = 0; g < G; ++g) {
        int p = 0;
        for (int i = 0; i < 64; ++i) p += (int)xc[g * 64 + i] * (int)wn[g * 64 + i];
        y += (double)sx[g] * (double)c.sw[(size_t)g * N + n] * (double)p;
      }
      for (int j = 0; j < rank; ++j) y += z[j] * bf16_to_f64(c.L2[(size_t)j * N + n]);
      ref = refm[(size_t)m * N + n];
      num += (y - ref) * (y - ref);
      den += ref * ref;
    }
  }
  return den > 0.0 ? std::sqrt(num / den) : 0.0;
}

svdq_status check_pack_args(int K, int N, int rank, int group, const uint16_t* W, int lora_rank,
                            const uint16_t* lora_A, const uint16_t* lora_B, float lora_scale,
                            svdq_weights** out) {
  if (!out) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (!W) return SVDQ_ERR_INVALID_ARG;
  if (group != SVDQ_GROUP) return SVDQ_ERR_UNSUPPORTED;
  if (K < SVDQ_GROUP || N < 1 || K % SVDQ_GROUP) return SVDQ_ERR_SHAPE;
  if (rank < 0 || lora_rank < 0 || rank > (K < N ? K : N)) return SVDQ_ERR_INVALID_ARG;
  if (rank + lora_rank > SVDQ_MAX_RANK || (rank + lora_rank) % 8 != 0) return SVDQ_ERR_UNSUPPORTED;
  if (lora_rank > 0 && (!lora_A || !lora_B)) return SVDQ_ERR_INVALID_ARG;
  if (!std::isfinite(lora_scale)) return SVDQ_ERR_NUMERIC;
  return SVDQ_OK;
}

// The handle from a finished candidate: eq. 13 (LoRA joins the 16-bit branch
// in smoothed coordinates), bias, optional upload.
svdq_status finish(int K, int N, int rank, Candidate& c, const uint16_t* bias, int lora_rank,
                   const uint16_t* lora_A, const uint16_t* lora_B, float lora_scale,
                   bool to_device, cudaStream_t stream, svdq_weights** out) {
  svdq_weights* w = new (std::nothrow) svdq_weights();
  if (!w) return SVDQ_ERR_OOM;
  w->K = K; w->N = N; w->G = K / SVDQ_GROUP;
  w->svd_rank = rank; w->lora_rank = lora_rank; w->rank = rank + lora_rank;
  w->rank_pad = (w->rank + 15) / 16 * 16;
  w->inv_lambda = std::move(c.inv_lambda);
  w->sigma = std::move(c.sigma);
  w->wq = std::move(c.wq);
  w->sw = std::move(c.sw);
  w->wq8 = std::move(c.wq8);
  w->sw8 = std::move(c.sw8);
  w->wq4 = std::move(c.wq4);
  w->sf4 = std::move(c.sf4);
  w->sw4 = std::move(c.sw4);
  w->format = !w->wq8.empty() ? SVDQ_FORMAT_W8A8
                              : !w->wq4.empty() ? SVDQ_FORMAT_NVFP4 : SVDQ_FORMAT_W4A4;
  const int rt = w->rank;
  w->L1.assign((size_t)K * rt, 0);
  w->L2.assign((size_t)rt * N, 0);
  for (int k = 0; k < K; ++k)
    for (int j = 0; j < rank; ++j) w->L1[(size_t)k * rt + j] = c.L1[(size_t)k * rank + j];
  for (int j = 0; j < rank; ++j)
    std::memcpy(&w->L2[(size_t)j * N], &c.L2[(size_t)j * N], (size_t)N * 2);
  for (int k = 0; k < K; ++k)
    for (int j = 0; j < lora_rank; ++j) {
      const double a = bf16_to_f64(lora_A[(size_t)k * lora_rank + j]);
      w->L1[(size_t)k * rt + rank + j] = f64_to_bf16((c.lam[k] * a) * (double)lora_scale);
    }
  for (int j = 0; j < lora_rank; ++j)
    std::memcpy(&w->L2[(size_t)(rank + j) * N], &lora_B[(size_t)j * N], (size_t)N * 2);
  w->bias.assign(N, 0);
  if (bias) std::memcpy(w->bias.data(), bias, (size_t)N * 2);
  if (to_device) {
    const svdq_status st = svdq::upload(w, stream);
    if (st != SVDQ_OK) { free_device(w); delete w; return st; }
  }
  *out = w;
  return SVDQ_OK;
}

}  // namespace

extern "C" {

const char* svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_SHAPE: return "unsupported shape (K must be a multiple of 64)";
    case SVDQ_ERR_ALIGNMENT: return "pointer or row not 16-byte aligned";
    case SVDQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case SVDQ_ERR_NUMERIC: return "non-finite input";
    case SVDQ_ERR_CUDA: return "CUDA runtime error";
    case SVDQ_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case SVDQ_ERR_OOM: return "out of memory";
    case SVDQ_ERR_IO: return "file I/O error";
    default: return "unknown status";
  }
}

int svdq_version(void) { return 100; }

svdq_status svdq_calib_absmax(int M, int K, const uint16_t* X, int ldx, float* absmax) {
  if (M < 0 || K < 1 || ldx < K) return SVDQ_ERR_SHAPE;
  if ((M > 0 && !X) || !absmax) return SVDQ_ERR_INVALID_ARG;
  for (int i = 0; i < M; ++i)
    for (int k = 0; k < K; ++k) {
      const float v = std::fabs(bits_f32((uint32_t)X[(size_t)i * ldx + k] << 16));
      if (std::isnan(v)) return SVDQ_ERR_NUMERIC;
      if (v > absmax[k]) absmax[k] = v;
    }
  return SVDQ_OK;
}


static svdq_status pack_impl(int K, int N, int rank, int group, const uint16_t* W,
                             const float* act_absmax, double alpha, const uint16_t* bias,
                             int lora_rank, const uint16_t* lora_A, const uint16_t* lora_B,
                             float lora_scale, bool to_device, cudaStream_t stream,
                             svdq_weights** out) {
  svdq_status s = check_pack_args(K, N, rank, group, W, lora_rank, lora_A, lora_B, lora_scale, out);
  if (s != SVDQ_OK) return s;
  if (!act_absmax || !(alpha > 0.0 && alpha < 1.0)) return SVDQ_ERR_INVALID_ARG;
  Candidate c;
  if ((s = smooth(K, N, W, act_absmax, alpha, c)) != SVDQ_OK) return s;
  if ((s = fit_factors(c.Wt.data(), K, N, rank, c)) != SVDQ_OK) return s;
  quantize_residual(K, N, rank, c);
  return finish(K, N, rank, c, bias, lora_rank, lora_A, lora_B, lora_scale, to_device, stream, out);
}

static svdq_status pack_calibrated_impl(int K, int N, int rank, int group, const uint16_t* W,
                                        const uint16_t* X, int M, int ldx, int n_alpha,
                                        const double* alphas, int iters, int gptq,
                                        const uint16_t* bias,
                                        int lora_rank, const uint16_t* lora_A,
                                        const uint16_t* lora_B, float lora_scale,
                                        bool to_device, cudaStream_t stream, double* errors,
                                        svdq_weights** out) {
  svdq_status s = check_pack_args(K, N, rank, group, W, lora_rank, lora_A, lora_B, lora_scale, out);
  if (s != SVDQ_OK) return s;
  if (!X || M < 1 || ldx < K || n_alpha < 1 || !alphas || iters < 0) return SVDQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_alpha; ++i)
    if (!(alphas[i] > 0.0 && alphas[i] < 1.0)) return SVDQ_ERR_INVALID_ARG;
  std::vector<float> a(K, 0.0f);
  if ((s = svdq_calib_absmax(M, K, X, ldx, a.data())) != SVDQ_OK) return s;
  const std::vector<double> ref = dense_reference(K, N, W, X, M, ldx);
  Candidate best;
  double best_err = 0.0;
  for (int i = 0; i < n_alpha; ++i) {
    Candidate c;
    if ((s = smooth(K, N, W, a.data(), alphas[i], c)) != SVDQ_OK) return s;
    if ((s = fit_factors(c.Wt.data(), K, N, rank, c)) != SVDQ_OK) return s;
    std::vector<double> U;
    if (gptq && (s = gptq_factor(gptq_hessian(K, X, M, ldx, c.inv_lambda), K, U)) != SVDQ_OK)
      return s;
    if (gptq) gptq_residual(K, N, rank, U, c);
    else quantize_residual(K, N, rank, c);
    for (int it = 0; it < iters; ++it)
      if ((s = refine(K, N, rank, c, gptq ? &U : nullptr)) != SVDQ_OK) return s;
    const double e = layer_error(K, N, rank, c, ref, X, M, ldx);
    if (errors) errors[i] = e;
    if (i == 0 || e < best_err) {
      best = std::move(c);
      best_err = e;
    }
  }
  return finish(K, N, rank, best, bias, lora_rank, lora_A, lora_B, lora_scale, to_device, stream,
                out);
}

svdq_status svdq_pack_weights(int K, int N, int rank, int group, const uint16_t* W,
                              const float* act_absmax, double alpha, const uint16_t* bias,
                              int lora_rank, const uint16_t* lora_A, const uint16_t* lora_B,
                              float lora_scale, cudaStream_t stream, svdq_weights** out) {
  return pack_impl(K, N, rank, group, W, act_absmax, alpha, bias, lora_rank, lora_A,
                   lora_B, lora_scale, true, stream, out);
}

svdq_status svdq_pack_weights_host(int K, int N, int rank, int group, const uint16_t* W,
                                   const float* act_absmax, double alpha,
                                   const uint16_t* bias, int lora_rank,
                                   const uint16_t* lora_A, const uint16_t* lora_B,
                                   float lora_scale, svdq_weights** out) {
  return pack_impl(K, N, rank, group, W, act_absmax, alpha, bias, lora_rank, lora_A,
                   lora_B, lora_scale, false, nullptr, out);
}

svdq_status svdq_pack_weights_calibrated(int K, int N, int rank, int group, const uint16_t* W,
                                         const uint16_t* X_cal, int M_cal, int ldx,
                                         int n_alpha, const double* alphas, int refine_iters,
                                         int gptq, const uint16_t* bias, int lora_rank,
                                         const uint16_t* lora_A, const uint16_t* lora_B,
                                         float lora_scale, int to_device, cudaStream_t stream,
                                         double* errors, svdq_weights** out) {
  return pack_calibrated_impl(K, N, rank, group, W, X_cal, M_cal, ldx, n_alpha, alphas,
                              refine_iters, gptq, bias, lora_rank, lora_A, lora_B, lora_scale,
                              to_device != 0, stream, errors, out);
}

svdq_status svdq_pack_weights_w8a8(int K, int N, int rank, const uint16_t* W,
                                   const float* act_absmax, double alpha, const uint16_t* bias,
                                   int to_device, cudaStream_t stream, svdq_weights** out) {
  svdq_status s = check_pack_args(K, N, rank, SVDQ_GROUP, W, 0, nullptr, nullptr, 1.0f, out);
  if (s != SVDQ_OK) return s;
  if (!act_absmax || !(alpha > 0.0 && alpha < 1.0)) return SVDQ_ERR_INVALID_ARG;
  Candidate c;
  if ((s = smooth(K, N, W, act_absmax, alpha, c)) != SVDQ_OK) return s;
  if ((s = fit_factors(c.Wt.data(), K, N, rank, c)) != SVDQ_OK) return s;
  quantize_residual_w8(K, N, rank, c);
  return finish(K, N, rank, c, bias, 0, nullptr, nullptr, 1.0f, to_device != 0, stream, out);
}

svdq_status svdq_weights_export_w8a8(const svdq_weights* w, int8_t* wq8, float* s_w8) {
  if (!w || w->format != SVDQ_FORMAT_W8A8) return SVDQ_ERR_INVALID_ARG;
  if (wq8) std::memcpy(wq8, w->wq8.data(), w->wq8.size());
  if (s_w8) std::memcpy(s_w8, w->sw8.data(), w->sw8.size() * 4);
  return SVDQ_OK;
}

int svdq_weights_format(const svdq_weights* w) { return w ? w->format : -1; }

svdq_status svdq_pack_weights_nvfp4(int K, int N, int rank, const uint16_t* W,
                                    const float* act_absmax, double alpha, const uint16_t* bias,
                                    int to_device, cudaStream_t stream, svdq_weights** out) {
  svdq_status s = check_pack_args(K, N, rank, SVDQ_GROUP, W, 0, nullptr, nullptr, 1.0f, out);
  if (s != SVDQ_OK) return s;
  if (!act_absmax || !(alpha > 0.0 && alpha < 1.0)) return SVDQ_ERR_INVALID_ARG;
  Candidate c;
  if ((s = smooth(K, N, W, act_absmax, alpha, c)) != SVDQ_OK) return s;
  if ((s = fit_factors(c.Wt.data(), K, N, rank, c)) != SVDQ_OK) return s;
  quantize_residual_nvfp4(K, N, rank, c);
  return finish(K, N, rank, c, bias, 0, nullptr, nullptr, 1.0f, to_device != 0, stream, out);
}

svdq_status svdq_weights_export_nvfp4(const svdq_weights* w, uint8_t* codes, uint8_t* sf,
                                      float* s_w) {
  if (!w || w->format != SVDQ_FORMAT_NVFP4) return SVDQ_ERR_INVALID_ARG;
  if (codes) std::memcpy(codes, w->wq4.data(), w->wq4.size());
  if (sf) std::memcpy(sf, w->sf4.data(), w->sf4.size());
  if (s_w) std::memcpy(s_w, w->sw4.data(), w->sw4.size() * 4);
  return SVDQ_OK;
}

size_t svdq_nvfp4_sf_bytes(int rows, int K) {
  return rows > 0 && K > 0 && K % 64 == 0 ? svdq::nvfp4_sf_bytes(rows, K) : 0;
}

svdq_status svdq_weights_info(const svdq_weights* w, int* K, int* N, int* rank,
                              int* svd_rank, int* lora_rank) {
  if (!w) return SVDQ_ERR_INVALID_ARG;
  if (K) *K = w->K;
  if (N) *N = w->N;
  if (rank) *rank = w->rank;
  if (svd_rank) *svd_rank = w->svd_rank;
  if (lora_rank) *lora_rank = w->lora_rank;
  return SVDQ_OK;
}

svdq_status svdq_weights_export(const svdq_weights* w, float* inv_lambda, uint8_t* wq,
                                float* s_w, uint16_t* L1, uint16_t* L2, uint16_t* bias,
                                double* sigma) {
  if (!w) return SVDQ_ERR_INVALID_ARG;
  if (inv_lambda) std::memcpy(inv_lambda, w->inv_lambda.data(), w->inv_lambda.size() * 4);
  if (wq) std::memcpy(wq, w->wq.data(), w->wq.size());
  if (s_w) std::memcpy(s_w, w->sw.data(), w->sw.size() * 4);
  if (L1 && !w->L1.empty()) std::memcpy(L1, w->L1.data(), w->L1.size() * 2);
  if (L2 && !w->L2.empty()) std::memcpy(L2, w->L2.data(), w->L2.size() * 2);
  if (bias) std::memcpy(bias, w->bias.data(), w->bias.size() * 2);
  if (sigma) std::memcpy(sigma, w->sigma.data(), w->sigma.size() * 8);
  return SVDQ_OK;
}

static const char kMagic[8] = {'S', 'V', 'D', 'Q', 'W', '0', '0', '1'};

svdq_status svdq_weights_save(const svdq_weights* w, const char* path) {
  if (!w || !path) return SVDQ_ERR_INVALID_ARG;
  if (w->format != SVDQ_FORMAT_W4A4) return SVDQ_ERR_UNSUPPORTED;
  FILE* f = std::fopen(path, "wb");
  if (!f) return SVDQ_ERR_IO;
  int32_t hdr[6] = {w->K, w->N, w->svd_rank, w->lora_rank, SVDQ_GROUP, 0};
  bool ok = std::fwrite(kMagic, 1, 8, f) == 8 && std::fwrite(hdr, 4, 6, f) == 6;
  auto put = [&](const void* p, size_t bytes) {
    if (ok && bytes) ok = std::fwrite(p, 1, bytes, f) == bytes;
  };
  put(w->inv_lambda.data(), w->inv_lambda.size() * 4);
  put(w->wq.data(), w->wq.size());
  put(w->sw.data(), w->sw.size() * 4);
  put(w->L1.data(), w->L1.size() * 2);
  put(w->L2.data(), w->L2.size() * 2);
  put(w->bias.data(), w->bias.size() * 2);
  put(w->sigma.data(), w->sigma.size() * 8);
  ok = (std::fclose(f) == 0) && ok;
  return ok ? SVDQ_OK : SVDQ_ERR_IO;
}

svdq_status svdq_weights_load(const char* path, cudaStream_t stream, svdq_weights** out) {
  if (!path || !out) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  FILE* f = std::fopen(path, "rb");
  if (!f) return SVDQ_ERR_IO;
  char magic[8];
  int32_t hdr[6];
  if (std::fread(magic, 1, 8, f) != 8 || std::memcmp(magic, kMagic, 8) != 0 ||
      std::fread(hdr, 4, 6, f) != 6) {
    std::fclose(f);
    return SVDQ_ERR_IO;
  }
  const int K = hdr[0], N = hdr[1], r = hdr[2], lr = hdr[3];
  if (hdr[4] != SVDQ_GROUP || K < 64 || K % 64 || N < 1 || r < 0 || lr < 0 ||
      r + lr > SVDQ_MAX_RANK || (r + lr) % 8 != 0 || K > (1 << 20) || N > (1 << 20)) {
    std::fclose(f);
    return SVDQ_ERR_IO;
  }
  svdq_weights* w = new (std::nothrow) svdq_weights();
  if (!w) { std::fclose(f); return SVDQ_ERR_OOM; }
  w->K = K; w->N = N; w->G = K / 64; w->svd_rank = r; w->lora_rank = lr;
  w->rank = r + lr; w->rank_pad = (w->rank + 15) / 16 * 16;
  w->inv_lambda.resize(K); w->wq.resize((size_t)N * K / 2); w->sw.resize((size_t)w->G * N);
  w->L1.resize((size_t)K * w->rank); w->L2.resize((size_t)w->rank * N);
  w->bias.resize(N); w->sigma.resize(r + 1);
  bool ok = true;
  auto get = [&](void* p, size_t bytes) {
    if (ok && bytes) ok = std::fread(p, 1, bytes, f) == bytes;
  };
  get(w->inv_lambda.data(), (size_t)K * 4);
  get(w->wq.data(), w->wq.size());
  get(w->sw.data(), w->sw.size() * 4);
  get(w->L1.data(), w->L1.size() * 2);
  get(w->L2.data(), w->L2.size() * 2);
  get(w->bias.data(), w->bias.size() * 2);
  get(w->sigma.data(), w->sigma.size() * 8);
  std::fclose(f);
  if (!ok) { delete w; return SVDQ_ERR_IO; }
  const svdq_status st = svdq::upload(w, stream);
  if (st != SVDQ_OK) { free_device(w); delete w; return st; }
  *out = w;
  return SVDQ_OK;
}

void svdq_weights_free(svdq_weights* w) {
  if (!w) return;
  free_device(w);
  delete w;
}

svdq_status svdq_get_device_error(const svdq_weights* w, cudaStream_t stream) {
  if (!w || !w->d_err) return SVDQ_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SVDQ_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, w->d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  if (h != SVDQ_DEVERR_NONE) {
    if (cudaMemset(w->d_err, 0, sizeof(int)) != cudaSuccess) return SVDQ_ERR_CUDA;
    return SVDQ_ERR_DEVICE_TIMEOUT;
  }
  return SVDQ_OK;
}

}  // extern "C"
