// The activation quantiser of the W4A4 path (SVDQuant review section 2.2,
// eq. 1, applied per token and group of 64 channels), shared by the
// activation pass and by the GEMM epilogue that quantises its own output
// for the next layer.
//
// s = fl32(m / 7) (IEEE division) for the group absmax m of x~, and the code
// is round-half-even of the exact quotient x~/s, clamped to [-8, 7]: a
// first guess from the correctly rounded reciprocal, with an exact
// fma-residual path where the guess is within 2^-20 of a half or the scale
// is tiny.  A lane holds 16 values of a token's group; the group spans the
// four lanes of a quad (absmax with two xor-shuffles).
#pragma once

#include <cstdint>

namespace svdq {
namespace {   // internal linkage: each kernel file keeps its own copy

constexpr float RN_MAGIC = 12582912.0f;   // 1.5 * 2^23: adding it rounds to an integer

// Two's-complement nibble of round-half-even(x / s), clamped to [-8, 7]; s > 0.
// `ss`, `rcp` are s (possibly scaled by 2^64 when s is tiny) and its
// correctly rounded reciprocal; `scale` is the same power of two for x.
// Branch-free: q0 = rne(x * rcp) by the magic-number add (|x/s| < 8, far
// inside its exact range); the exact residual x - q0 s (an fma, exact here)
// moves q0 by one where the rounded quotient crossed a half, and an exact
// tie goes to the even neighbour.  The nibble is read from the low bits of
// the magic-biased float, whose integer bits are 0x4B400000 + q.
__device__ __forceinline__ uint32_t quant_nibble(float x, float ss, float rcp, float scale) {
  const float xx = __fmul_rn(x, scale);              // exact (power of two)
  const float b0 = __fadd_rn(__fmul_rn(xx, rcp), RN_MAGIC);
  float q = __fsub_rn(b0, RN_MAGIC);                 // rne(xx * rcp)
  const float d2 = 2.0f * __fmaf_rn(-q, ss, xx);     // exact residual, doubled
  const uint32_t odd = __float_as_uint(b0) & 1u;
  float adj = (d2 > ss) ? 1.0f : ((d2 < -ss) ? -1.0f : 0.0f);
  adj = (fabsf(d2) == ss && odd) ? copysignf(1.0f, d2) : adj;
  q = fminf(fmaxf(__fadd_rn(q, adj), -8.0f), 7.0f);
  return __float_as_uint(__fadd_rn(q, RN_MAGIC)) & 0xFu;
}

// Value j = 4 ks + e of a lane's row (16-column step ks; e: columns 2q, 2q+1,
// 2q+8, 2q+9) goes to byte ks of word e / 2, low nibble for even e.
__device__ __forceinline__ void place(uint32_t nib, int j, uint32_t& u0, uint32_t& u1) {
  const uint32_t v = nib << (8 * (j >> 2) + 4 * (j & 1));
  if ((j >> 1) & 1) u1 |= v; else u0 |= v;
}

// All 16 codes of a lane's row by the exact path (rare; kept out of line).
__device__ __noinline__ void quant16_exact(const float* v, float ssc, float rcp, float scale,
                                           uint32_t* u) {
  uint32_t u0 = 0u, u1 = 0u;
#pragma unroll
  for (int j = 0; j < 16; ++j) place(quant_nibble(v[j], ssc, rcp, scale), j, u0, u1);
  u[0] = u0;
  u[1] = u1;
}

// One token's group of 64: the lane's 16 values v[4 ks + e] (layout of
// `place`), the quad's lanes holding the rest.  Returns s = fl32(m / 7) and
// the lane's codes as two words (byte ks of word h: the two codes of columns
// 16 ks + 8 h + 2q and + 1, low nibble first).  Every lane of the warp must
// call it (shuffles).
__device__ __forceinline__ float quant_group16(const float* v, uint32_t (&u)[2]) {
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) m = fmaxf(m, fabsf(v[j]));
  m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
  const float sc = __fdiv_rn(m, 7.0f);
  u[0] = 0u;
  u[1] = 0u;
  if (sc > 0.0f) {
    const bool tiny = sc < 0x1p-64f;     // s subnormal or nearly: exact path
    bool near = tiny;
    const float scale = tiny ? 0x1p64f : 1.0f;
    const float ssc = __fmul_rn(sc, scale);
    const float rcp = __frcp_rn(ssc);
    if (!tiny) {
      // Fast path for a normal scale: t = fl(x * fl(1/s)) is within
      // |x/s| 2^-23 <= 2^-20 of the exact quotient, so rne(t) = rne(x/s)
      // unless t lies within 2^-20 of a half-integer.
      // Pairs (j, j+1) are the two codes of one byte; t = x * fl(1/s),
      // rne(t) by the magic add, f = t - rne(t) exact; the row is near
      // a half somewhere iff max |f| >= 1/2 - 2^-20
      const float2 rc2 = make_float2(rcp, rcp), mg2 = make_float2(RN_MAGIC, RN_MAGIC);
      const float2 nmg2 = make_float2(-RN_MAGIC, -RN_MAGIC);
      float fmx = 0.0f;
      uint32_t by[8];
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float2 t = __fmul2_rn(make_float2(v[j], v[j + 1]), rc2);
        const float2 b = __fadd2_rn(t, mg2);
        const float2 r = __fadd2_rn(b, nmg2);
        const float2 f = __fadd2_rn(t, make_float2(-r.x, -r.y));
        fmx = fmaxf(fmx, fmaxf(fabsf(f.x), fabsf(f.y)));
        // |rne(t)| <= 7: the low nibble of the biased word is the code
        by[j >> 1] = (__float_as_uint(b.x) & 0xFu) | ((__float_as_uint(b.y) << 4) & 0xF0u);
      }
      near = fmx >= 0.5f - 0x1p-20f;
      // byte of pair j/2 = 2 ks + h goes to byte ks of word h
      u[0] = __byte_perm(__byte_perm(by[0], by[2], 0x0040), __byte_perm(by[4], by[6], 0x0040), 0x5410);
      u[1] = __byte_perm(__byte_perm(by[1], by[3], 0x0040), __byte_perm(by[5], by[7], 0x0040), 0x5410);
    }
    if (near) {                          // rare: exact residual
      float tmp[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) tmp[j] = v[j];
      quant16_exact(tmp, ssc, rcp, scale, u);
    }
  }
  return sc;
}

// 4 x 4 byte transpose across the lanes of a quad: lane q holds bytes
// b[q][0..3] (byte j destined for lane j) and returns b[0..3][q].
__device__ __forceinline__ uint32_t quad_transpose(uint32_t x, int q) {
  uint32_t p = __shfl_xor_sync(0xFFFFFFFFu, x, 2);
  const uint32_t y = (q & 2) ? __byte_perm(p, x, 0x7632) : __byte_perm(x, p, 0x5410);
  p = __shfl_xor_sync(0xFFFFFFFFu, y, 1);
  return __byte_perm(y, p, (q & 1) ? 0x3715 : 0x6240);
}

}  // namespace
}  // namespace svdq
