// Fused activation pass (SVDQuant review section 6.1, activation side): read
// X once, smooth it (eq. 3), quantise it per token and group of 64 (eq. 1)
// and, from the same registers, compute the 16-bit down-projection
// Z = bf16(x~) L1 on the tensor cores (mma.sync bf16, fp32 accumulation).
//
// Layout: a CTA owns 32 consecutive tokens and walks K in stages of eight
// groups (512 channels; four for branch ranks above 64).  A producer warp
// streams each stage by TMA into a shared-memory ring: the 32 x 64 bf16 tile
// of X of every group (128-byte swizzled), the matching 64-column slice of
// L1^T (all branch rows, also swizzled) and the stage's smoothing factors,
// all on one mbarrier.  Sixteen compute warps (eight for the largest ranks)
// each own one 16-token x 64-channel block of a stage (two token halves x
// the stage's groups), read it with ldmatrix in the mma.sync A
// fragment layout and, without any CTA-wide barrier, smooth, quantise,
// store codes and scales, and multiply the same fragments (as bf16) with
// L1 fragments read by ldmatrix.  A warp releases the stage with an mbarrier
// arrive; the producer refills it.  The warps' partial Z (different groups,
// same tokens) are summed in shared memory at the end.
//
// Quantiser: x~ = fl32(x * inv_lambda) (one IEEE multiply), s = fl32(m / 7)
// (IEEE division) for the group absmax m, and the code is round-half-even of
// the exact quotient x~/s: a first guess from the correctly rounded
// reciprocal, with an exact fma-residual path where the guess is within
// 2^-20 of a half or the scale is tiny.  A lane holds 16 values of each of
// two tokens; a token's group spans the four lanes of a quad (absmax with
// two xor-shuffles; codes regrouped into 8-byte stores by a 4 x 4 byte
// transpose across the quad).
//
// Few tokens: when the 32-token blocks cannot fill the GPU, K is split over
// a cluster of up to eight CTAs per token block (one K range each).  Codes
// and scales are per group, so they need nothing more; each CTA sums its
// warps' partial Z in shared memory, and after a cluster barrier CTA c sums,
// for its share of the 32 rows, the partials of CTAs 0, 1, .. in order
// through distributed shared memory (deterministic).
//
// The W8A8 comparator (review section 8, the eight-bit setting) runs the
// same kernel with one int8 scale per token: the CTA streams its tokens
// twice.  The first sweep takes each token's absmax of x~ and the
// down-projection Z; the compute warps then combine their row maxima in
// shared memory (one named barrier among them) into s = fl32(m / 127); the
// second sweep (X only, which the first sweep has just brought into L2)
// quantises and stores 16 contiguous int8 codes per lane and token.
//
// The NVFP4 variant (review section 8: groups of 16 with FP8 scales) takes
// the same two sweeps with s = fl32(m / 2688) per token.  The second sweep
// needs no Z, so it leaves the fragment layout: each lane reads 32
// contiguous columns of one token from the swizzled tile, takes the two
// 16-column group maxima in-thread (E4M3 group scale b), decides each E2M1
// code from one reciprocal per group (exact comparisons |x| <> mid_j b s,
// one fma each, only near a midpoint), and writes its 32 codes with one
// 16-byte store and its two group scales into the tensor-core scale atom.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "gemm_common.cuh"
#include "ptx.cuh"
#include "quant_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int AQ_ROWS = 32;                 // tokens per CTA
constexpr int AQ_XTILE = AQ_ROWS * 128;     // one group of X: 32 rows x 64 bf16
constexpr uint64_t AQ_LIMIT_NS = 2000000000ull;

// Stage layout: X tiles of the GPS groups, then their L1^T slices
// (NT * 8 rows x 128 B each), then the 64 GPS smoothing factors.  Eight
// groups (16 compute warps) per stage while the L1 slices are small, four
// (8 warps) for the largest ranks.
template <int NT>
struct AqStage {
  static constexpr int GPS = NT <= 8 ? 8 : 4;
  static constexpr int WARPS = 2 * GPS;                               // compute warps
  static constexpr int THREADS = (WARPS + 1) * 32;                    // + the producer warp
  static constexpr int L1_TILE = NT * 8 * 128;
  static constexpr int OFF_L1 = GPS * AQ_XTILE;
  static constexpr int OFF_IL = OFF_L1 + GPS * L1_TILE;
  static constexpr int BYTES = OFF_IL + GPS * 64 * 4;                 // multiple of 1024
  static constexpr int STAGES = (200 * 1024) / BYTES < 4 ? (200 * 1024) / BYTES : 4;
  static constexpr int RED = WARPS * 16 * NT * 8 * 4;                 // Z partials at the end
  static constexpr int ZC = AQ_ROWS * NT * 8 * 4;                     // a CTA's partial Z (split K)
  static_assert(STAGES >= 2, "stage too large");
  static_assert(RED + ZC <= STAGES * BYTES, "reduction buffers alias the ring");
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of every CTA of the cluster (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// fp32 at the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ float ld_cluster_f32(uint32_t saddr, uint32_t rank) {
  uint32_t ra;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(saddr), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

__device__ __forceinline__ float2 lds64(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
// Two floats -> packed bf16x2 bits (round to nearest even), a in the low half.
__device__ __forceinline__ uint32_t bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// int8 code of round-half-even(x / s), clamped to [-128, 127]: the exact
// path of quant_nibble with the comparator's range; |x/s| <= 127.5 keeps the
// magic-number rounding and the fma residual exact.
__device__ __forceinline__ uint32_t quant_byte(float x, float ss, float rcp, float scale) {
  const float xx = __fmul_rn(x, scale);
  const float b0 = __fadd_rn(__fmul_rn(xx, rcp), RN_MAGIC);
  float q = __fsub_rn(b0, RN_MAGIC);
  const float d2 = 2.0f * __fmaf_rn(-q, ss, xx);
  const uint32_t odd = __float_as_uint(b0) & 1u;
  float adj = (d2 > ss) ? 1.0f : ((d2 < -ss) ? -1.0f : 0.0f);
  adj = (fabsf(d2) == ss && odd) ? copysignf(1.0f, d2) : adj;
  q = fminf(fmaxf(__fadd_rn(q, adj), -128.0f), 127.0f);
  return __float_as_uint(__fadd_rn(q, RN_MAGIC)) & 0xFFu;
}

// The 16 int8 codes of one lane's token in a group, as four words: word ks
// holds columns 16ks + 2q, 2q+1, 2q+8, 2q+9 (bytes 0..3).  Rare exact path.
__device__ __noinline__ void quant16_byte_exact(const float* v, float ssc, float rcp, float scale,
                                                uint32_t* wd) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    uint32_t x = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) x |= quant_byte(v[4 * ks + e], ssc, rcp, scale) << (8 * e);
    wd[ks] = x;
  }
}

// Word transpose across a quad: lane q holds w[0..3] (word ks destined for
// lane ks) and returns, in o[p], word q of lane p.
__device__ __forceinline__ void quad_transpose_words(const uint32_t (&w)[4], int q,
                                                     uint32_t (&o)[4]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) o[k] = (k == q) ? w[k] : 0u;
#pragma unroll
  for (int i = 1; i < 4; ++i) {
    const int p = q ^ i;
    const uint32_t send = p == 0 ? w[0] : p == 1 ? w[1] : p == 2 ? w[2] : w[3];
    const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, send, i);   // lane p's word q
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] = (k == p) ? got : o[k];
  }
}

// FP8 E4M3 value of a non-negative fp32 t (nearest, ties to even, saturating
// at 448) and its bit pattern.
__device__ __forceinline__ float e4m3_round(float t) {
  if (!(t > 0.0f)) return 0.0f;
  if (t >= 448.0f) return 448.0f;
  const int ex = (int)((__float_as_uint(t) >> 23) & 0xFF) - 127;   // floor(log2 t) for a normal t
  const int qexp = ex - 3 > -9 ? ex - 3 : -9;                      // in [-9, 5]
  // 2^-qexp and 2^qexp as floats (normal exponents): exact scalings
  const float up = __uint_as_float((uint32_t)(127 - qexp) << 23);
  const float dn = __uint_as_float((uint32_t)(127 + qexp) << 23);
  const float v = rintf(t * up) * dn;
  return v < 448.0f ? v : 448.0f;
}
__device__ __forceinline__ uint32_t e4m3_byte(float v) {
  if (!(v > 0.0f)) return 0u;
  if (v < 0x1p-6f) return (uint32_t)rintf(v * 512.0f);
  const uint32_t u = __float_as_uint(v);
  return ((((u >> 23) & 0xFF) - 120u) << 3) | ((u >> 20) & 7u);
}

// E2M1 code of the exact quotient x / (b s): bd_j = mid_j b (exact in fp32),
// the sign of fma(bd_j, s, -|x|) is that of mid_j b s - |x| (exact).
__device__ __forceinline__ uint32_t e2m1_code(float x, float b, float s) {
  const float a = fabsf(x);
  const float mids[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
  int idx = 0;
  bool tie = false;
#pragma unroll
  for (int j = 0; j < 7; ++j) {
    const float c = __fmaf_rn(mids[j] * b, s, -a);
    idx += c < 0.0f ? 1 : 0;
    tie = (c == 0.0f && idx == j) ? true : tie;
  }
  if (tie && (idx & 1)) ++idx;
  return (uint32_t)idx | ((x < 0.0f && idx > 0) ? 8u : 0u);
}

// E2M1 code from u = |x| fl(1/fl(b s)), within 2^-22 (relative) of the exact
// quotient, without branches: the grid {0, .5, 1, 1.5, 2, 3, 4, 6} maps onto
// the integers 0..7 under the concave piecewise-linear c(u) = min(2u, u + 2,
// u/2 + 4), so the code is rne(c) (its ties are the grid's midpoints, and
// rne's even choice is the even code), capped at 7.  `near` is raised when
// c lies within 2^-18 of a half below 7 (the exact path decides).
__device__ __forceinline__ uint32_t e2m1_fast(float x, float r, bool& near) {
  const float u = fabsf(x) * r;
  const float c = fminf(2.0f * u, fminf(u + 2.0f, __fmaf_rn(0.5f, u, 4.0f)));
  const float rc = rintf(c);
  near |= (fabsf(c - rc) > 0.5f - 0x1p-18f) && (c < 7.25f);
  const uint32_t k = (uint32_t)fminf(rc, 7.0f);
  return k | ((x < 0.0f && k > 0u) ? 8u : 0u);
}

// NVFP4 second sweep, one lane = 32 contiguous columns (two groups of 16) of
// one token, read straight from the 128-byte-swizzled X tile: group maxima
// in-thread, codes packed in column order (one 16-byte store), the two group
// scales as one 16-bit store into the scale atom.
// rs: token scale (x 2^64 when tiny); d6 = fl32(6 s); sc = 2^64 or 1.
__device__ __forceinline__ void nvfp4_row32(uint32_t xrow, int rl, int hh, uint32_t ilt, float rs,
                                            float d6, float sc, bool tiny, uint8_t* xq_dst,
                                            uint8_t* sf_dst) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 raw = lds128u(xrow + (((4 * hh + i) ^ (rl & 7)) << 4));
    const float4 i0 = lds128(ilt + 4 * (32 * hh + 8 * i));
    const float4 i1 = lds128(ilt + 4 * (32 * hh + 8 * i + 4));
    const float2 p0 = __fmul2_rn(make_float2(bf16lo(raw.x), bf16hi(raw.x)), make_float2(i0.x, i0.y));
    const float2 p1 = __fmul2_rn(make_float2(bf16lo(raw.y), bf16hi(raw.y)), make_float2(i0.z, i0.w));
    const float2 p2 = __fmul2_rn(make_float2(bf16lo(raw.z), bf16hi(raw.z)), make_float2(i1.x, i1.y));
    const float2 p3 = __fmul2_rn(make_float2(bf16lo(raw.w), bf16hi(raw.w)), make_float2(i1.z, i1.w));
    v[8 * i + 0] = p0.x; v[8 * i + 1] = p0.y; v[8 * i + 2] = p1.x; v[8 * i + 3] = p1.y;
    v[8 * i + 4] = p2.x; v[8 * i + 5] = p2.y; v[8 * i + 6] = p3.x; v[8 * i + 7] = p3.y;
  }
  float bs[2];
#pragma unroll
  for (int bk = 0; bk < 2; ++bk) {
    float mg = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) mg = fmaxf(mg, fabsf(v[16 * bk + j]));
    bs[bk] = d6 > 0.0f ? e4m3_round(__fdiv_rn(mg, d6)) : 0.0f;
  }
  uint32_t w[4];
  bool near = tiny;
  if (!near) {
    const float r0 = bs[0] > 0.0f ? __frcp_rn(__fmul_rn(bs[0], rs)) : 0.0f;
    const float r1 = bs[1] > 0.0f ? __frcp_rn(__fmul_rn(bs[1], rs)) : 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t x = 0u;
#pragma unroll
      for (int e = 0; e < 8; ++e) x |= e2m1_fast(v[8 * i + e], i < 2 ? r0 : r1, near) << (4 * e);
      w[i] = x;
    }
  }
  if (near) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t x = 0u;
      const float bb = bs[i >> 1];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        x |= (bb > 0.0f ? e2m1_code(v[8 * i + e] * sc, bb, rs) : 0u) << (4 * e);
      w[i] = x;
    }
  }
  if (xq_dst) *reinterpret_cast<uint4*>(xq_dst) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint16_t*>(sf_dst) = (uint16_t)(e4m3_byte(bs[0]) | (e4m3_byte(bs[1]) << 8));
}



// FMT: 0 W4A4 groups of 64; 1 W8A8 comparator; 2 NVFP4 variant.
template <int NT, int FMT>
__global__ void __launch_bounds__(AqStage<NT>::THREADS, 1)
act_quant_kernel(const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_l,   // L1^T [NT*8][K] bf16
                 const float* __restrict__ inv_lambda,
                 int M, int K, int rank,
                 uint8_t* __restrict__ xq, float* __restrict__ s_x,
                 uint16_t* __restrict__ Z, uint8_t* __restrict__ sfa,
                 int* __restrict__ err, int ksplit) {
  constexpr bool W8 = FMT != 0;                // two sweeps, one scale per token
  using ST = AqStage<NT>;
  constexpr int S = ST::STAGES;
  constexpr int AQ_GPS = ST::GPS, AQ_WARPS = ST::WARPS, AQ_THREADS = ST::THREADS;
  __shared__ __align__(8) uint64_t full_bar[S], empty_bar[S];
  __shared__ int abort_sh;
  __shared__ float rowmax_sh[W8 ? AqStage<NT>::GPS : 1][AQ_ROWS];   // W8: per-warp token maxima
  extern __shared__ uint8_t aq_dyn_raw[];
  uint8_t* ring_p = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(aq_dyn_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t ring = smem_u32(ring_p);

  const int tid = threadIdx.x, warp = tid >> 5, l = tid & 31;
  // token block and K range (groups [g0, g1)) of this CTA; ksplit > 1 only
  // for W4A4, and then, with a branch, the CTAs of a block form a cluster
  const int row0 = (blockIdx.x / ksplit) * AQ_ROWS;
  const int sp = blockIdx.x % ksplit;
  const int G = K / 64;
  const int g0 = (int)((long long)sp * G / ksplit), g1 = (int)((long long)(sp + 1) * G / ksplit);
  const int nstages = (g1 - g0 + AQ_GPS - 1) / AQ_GPS;
  const int nsweep = W8 ? 2 * nstages : nstages;      // W8: quantising sweep after the first

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), AQ_WARPS);
    }
    abort_sh = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  float zacc[NT > 0 ? NT : 1][4];
#pragma unroll
  for (int a = 0; a < (NT > 0 ? NT : 1); ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) zacc[a][b] = 0.0f;

  if (warp == AQ_WARPS) {
    // ------------------------------------------------------------ producer
    if (l == 0) {
      int c = 0;
      for (; c < nsweep; ++c) {
        const int s = c % S;
        if (c >= S && !mbar_wait_bounded(smem_u32(&empty_bar[s]), ((c / S) - 1) & 1, AQ_LIMIT_NS)) {
          atomicExch(err, SVDQ_DEVERR_TIMEOUT);
          abort_sh = 1;
          break;
        }
        if (*reinterpret_cast<volatile int*>(&abort_sh)) break;
        const bool second = c >= nstages;              // no L1 slices needed
        const int cc = second ? c - nstages : c;
        const int gb = g0 + AQ_GPS * cc;               // first group of the stage
        const int ng = min(AQ_GPS, g1 - gb);
        const uint32_t fb = smem_u32(&full_bar[s]);
        const bool with_l1 = NT > 0 && !second;
        mbar_arrive_expect_tx(fb, ng * (AQ_XTILE + (with_l1 ? ST::L1_TILE : 0) + 256));
        const uint32_t st = ring + s * ST::BYTES;
        for (int g = 0; g < ng; ++g) {
          const int col = (gb + g) * 64;
          tma_load_2d(st + g * AQ_XTILE, &tm_x, col, row0, fb);
          if (with_l1) tma_load_2d(st + ST::OFF_L1 + g * ST::L1_TILE, &tm_l, col, 0, fb);
        }
        bulk_load(st + ST::OFF_IL, inv_lambda + 64 * gb, ng * 256, fb);
      }
      // every issued copy lands before the CTA moves on
      for (int k = (c > S ? c - S : 0); k < c; ++k)
        mbar_wait_bounded(smem_u32(&full_bar[k % S]), (k / S) & 1, AQ_LIMIT_NS);
    }
  } else {
    // ------------------------------------------------------- compute warps
    const int rb = warp & 1, gi = warp >> 1, q = l & 3, g8 = l >> 2;
    float rmax[2] = {0.0f, 0.0f};     // W8: running absmax of the lane's two tokens
    float wsc[2] = {0.0f, 0.0f}, wss[2] = {0.0f, 0.0f}, wrcp[2] = {0.0f, 0.0f};
    // NVFP4 second sweep: this lane's token rl4 = 16 rb + l / 2 and its scales
    const int rl4 = rb * 16 + (l >> 1), hh4 = l & 1;
    float f4s = 0.0f, f4d6 = 0.0f, f4sc = 1.0f;
    bool f4tiny = false;
    float wscale[2] = {1.0f, 1.0f};
    bool wtiny[2] = {false, false};
    // One stage: the warp's 16 x 64 block of group AQ_GPS * cc + gi.
    // second: the comparator's quantising sweep (W8 only).
    auto stage = [&](int c, int cc, bool second) -> bool {
      const int s = c % S;
      if (!mbar_wait_bounded(smem_u32(&full_bar[s]), (c / S) & 1, AQ_LIMIT_NS)) {
        atomicExch(err, SVDQ_DEVERR_TIMEOUT);
        abort_sh = 1;
        return false;
      }
      if (*reinterpret_cast<volatile int*>(&abort_sh)) return false;
      const int grp = g0 + AQ_GPS * cc + gi;
      if (FMT == 2 && second && grp < g1) {
        const uint32_t st = ring + s * ST::BYTES;
        const int row = row0 + rl4, a = row >> 7, r = row & 127;
        nvfp4_row32(st + gi * AQ_XTILE + rl4 * 128, rl4, hh4, st + ST::OFF_IL + gi * 256, f4s, f4d6,
                    f4sc, f4tiny, row < M ? xq + (size_t)row * (K / 2) + grp * 32 + 16 * hh4 : nullptr,
                    sfa + ((size_t)a * G + grp) * 512 + 16 * (r & 31) + 4 * (r >> 5) + 2 * hh4);
      } else if (grp < g1) {
        const uint32_t st = ring + s * ST::BYTES;
        const uint32_t xt = st + gi * AQ_XTILE;
        // raw X in the A fragment layout: a[ks][0] row g8, cols 16ks+2q (+1);
        // [1] row g8+8; [2] row g8, cols 16ks+8+2q (+1); [3] row g8+8
        uint32_t a[4][4];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const int rr = rb * 16 + (l & 15), ch = 2 * ks + (l >> 4);
          ldmatrix_x4(xt + rr * 128 + ((ch ^ (rr & 7)) << 4), a[ks]);
        }
        const uint32_t ilt = st + ST::OFF_IL + gi * 256;
        float v[2][16];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const float2 i0 = lds64(ilt + 4 * (16 * ks + 2 * q));
          const float2 i1 = lds64(ilt + 4 * (16 * ks + 8 + 2 * q));
#pragma unroll
          for (int ri = 0; ri < 2; ++ri) {
            const float2 p0 = __fmul2_rn(make_float2(bf16lo(a[ks][ri]), bf16hi(a[ks][ri])), i0);
            const float2 p1 = __fmul2_rn(make_float2(bf16lo(a[ks][2 + ri]), bf16hi(a[ks][2 + ri])), i1);
            v[ri][4 * ks + 0] = p0.x;
            v[ri][4 * ks + 1] = p0.y;
            v[ri][4 * ks + 2] = p1.x;
            v[ri][4 * ks + 3] = p1.y;
          }
        }
        if constexpr (W8) {
          if (!second) {
#pragma unroll
            for (int ri = 0; ri < 2; ++ri)
#pragma unroll
              for (int j = 0; j < 16; ++j) rmax[ri] = fmaxf(rmax[ri], fabsf(v[ri][j]));
          } else {
#pragma unroll
            for (int ri = 0; ri < 2; ++ri) {
              uint32_t wd[4] = {0u, 0u, 0u, 0u};
              if (wsc[ri] > 0.0f) {
                bool near = wtiny[ri];
                if (!near) {
                  // t = x * fl(1/s) is within |x/s| 2^-23 < 2^-16 of the exact
                  // quotient: rne(t) = rne(x/s) unless t is within 2^-15 of a half
                  const float2 rc2 = make_float2(wrcp[ri], wrcp[ri]);
                  const float2 mg2 = make_float2(RN_MAGIC, RN_MAGIC);
                  const float2 nmg2 = make_float2(-RN_MAGIC, -RN_MAGIC);
                  float fmx = 0.0f;
#pragma unroll
                  for (int j = 0; j < 16; j += 2) {
                    const float2 t = __fmul2_rn(make_float2(v[ri][j], v[ri][j + 1]), rc2);
                    const float2 b = __fadd2_rn(t, mg2);
                    const float2 r = __fadd2_rn(b, nmg2);
                    const float2 f = __fadd2_rn(t, make_float2(-r.x, -r.y));
                    fmx = fmaxf(fmx, fmaxf(fabsf(f.x), fabsf(f.y)));
                    // |rne(t)| <= 127: the low byte of the biased word is the code
                    const uint32_t two = (__float_as_uint(b.x) & 0xFFu) |
                                         ((__float_as_uint(b.y) & 0xFFu) << 8);
                    wd[j >> 2] |= two << (16 * ((j >> 1) & 1));
                  }
                  near = fmx >= 0.5f - 0x1p-15f;
                }
                if (near) {
                  float tmp[16];
#pragma unroll
                  for (int j = 0; j < 16; ++j) tmp[j] = v[ri][j];
                  quant16_byte_exact(tmp, wss[ri], wrcp[ri], wscale[ri], wd);
                }
              }
              // lane q gets columns 16q .. 16q+15 of the group: from lane p the
              // bytes of columns 16q + {2p, 2p+1, 2p+8, 2p+9}
              uint32_t o[4];
              quad_transpose_words(wd, q, o);
              const uint4 out = make_uint4(__byte_perm(o[0], o[1], 0x5410), __byte_perm(o[2], o[3], 0x5410),
                                           __byte_perm(o[0], o[1], 0x7632), __byte_perm(o[2], o[3], 0x7632));
              const int row = row0 + rb * 16 + g8 + 8 * ri;
              if (row < M)
                *reinterpret_cast<uint4*>(xq + (size_t)row * K + grp * 64 + 16 * q) = out;
            }
          }
        } else {
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
          uint32_t u[2];
          const float sc = quant_group16(v[ri], u);
          const uint32_t w0 = quad_transpose(u[0], q), w1 = quad_transpose(u[1], q);
          const int row = row0 + rb * 16 + g8 + 8 * ri;
          if (row < M) {
            *reinterpret_cast<uint2*>(xq + (size_t)row * (K / 2) + grp * 32 + 8 * q) = make_uint2(w0, w1);
            if (q == 0) s_x[(size_t)grp * M + row] = sc;
          }
        }
        }
        if constexpr (NT > 0) {
          if (!second) {
            const uint32_t lt = st + ST::OFF_L1 + gi * ST::L1_TILE;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              uint32_t af[4];
              af[0] = bf16x2(v[0][4 * ks + 0], v[0][4 * ks + 1]);
              af[1] = bf16x2(v[1][4 * ks + 0], v[1][4 * ks + 1]);
              af[2] = bf16x2(v[0][4 * ks + 2], v[0][4 * ks + 3]);
              af[3] = bf16x2(v[1][4 * ks + 2], v[1][4 * ks + 3]);
#pragma unroll
              for (int j = 0; j < NT / 2; ++j) {
                // matrices: n-tile 2j (k 0-7, 8-15), n-tile 2j+1 (k 0-7, 8-15)
                const int mi = l >> 3, n = 16 * j + 8 * (mi >> 1) + (l & 7), ch = 2 * ks + (mi & 1);
                uint32_t b[4];
                ldmatrix_x4(lt + n * 128 + ((ch ^ (n & 7)) << 4), b);
                mma_bf16_16816(zacc[2 * j], af, b[0], b[1]);
                mma_bf16_16816(zacc[2 * j + 1], af, b[2], b[3]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (l == 0) mbar_arrive(smem_u32(&empty_bar[s]));
      return true;
    };
    bool alive = true;
    for (int c = 0; c < nstages && alive; ++c) alive = stage(c, c, false);
    if constexpr (W8) {
      // per-token scales: quad, then the group-warps of each token half.
      // Every compute warp reaches this barrier exactly once.
#pragma unroll
      for (int ri = 0; ri < 2; ++ri) {
        rmax[ri] = fmaxf(rmax[ri], __shfl_xor_sync(0xFFFFFFFFu, rmax[ri], 1));
        rmax[ri] = fmaxf(rmax[ri], __shfl_xor_sync(0xFFFFFFFFu, rmax[ri], 2));
        if (q == 0) rowmax_sh[gi][rb * 16 + g8 + 8 * ri] = rmax[ri];
      }
      asm volatile("bar.sync 1, %0;" ::"r"(AQ_WARPS * 32) : "memory");
#pragma unroll
      for (int ri = 0; ri < 2; ++ri) {
        const int rl = rb * 16 + g8 + 8 * ri;
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < AQ_GPS; ++j) m = fmaxf(m, rowmax_sh[j][rl]);
        if constexpr (FMT == 2) {
          // s = fl32(m / 2688); wss = fl32(6 s); the codes are decided on
          // x 2^64 against s 2^64 when s is tiny (exact power-of-two scaling)
          const float sr = __fdiv_rn(m, 2688.0f);
          wss[ri] = __fmul_rn(6.0f, sr);
          wtiny[ri] = sr < 0x1p-64f;
          wscale[ri] = wtiny[ri] ? 0x1p64f : 1.0f;
          wsc[ri] = __fmul_rn(sr, wscale[ri]);
          if (gi == 0 && q == 0 && row0 + rl < M) s_x[row0 + rl] = sr;
          if (ri == 0) {                       // the row-contiguous sweep's token
            float m4 = 0.0f;
#pragma unroll
            for (int j = 0; j < AQ_GPS; ++j) m4 = fmaxf(m4, rowmax_sh[j][rl4]);
            const float s4 = __fdiv_rn(m4, 2688.0f);
            f4d6 = __fmul_rn(6.0f, s4);
            f4tiny = s4 < 0x1p-64f;
            f4sc = f4tiny ? 0x1p64f : 1.0f;
            f4s = __fmul_rn(s4, f4sc);
          }
        } else {
          wsc[ri] = __fdiv_rn(m, 127.0f);
          wtiny[ri] = wsc[ri] < 0x1p-64f;
          wscale[ri] = wtiny[ri] ? 0x1p64f : 1.0f;
          wss[ri] = __fmul_rn(wsc[ri], wscale[ri]);
          wrcp[ri] = wsc[ri] > 0.0f ? __frcp_rn(wss[ri]) : 0.0f;
          if (gi == 0 && q == 0 && row0 + rl < M) s_x[row0 + rl] = wsc[ri];
        }
      }
      for (int c = nstages; c < 2 * nstages && alive; ++c) alive = stage(c, c - nstages, true);
    }
  }
  __syncthreads();
  // Every thread reaches the cluster barriers below, also after an expired
  // wait (the partials are then not used: the error word is raised).
  const bool aborted = *reinterpret_cast<volatile int*>(&abort_sh) != 0;
  if (aborted && (NT == 0 || ksplit == 1)) return;

  if constexpr (NT > 0) {
    // sum the group-warps of each token half; Z rows in bf16
    constexpr int RP = NT * 8;
    float* red = reinterpret_cast<float*>(ring_p);
    if (!aborted && warp < AQ_WARPS) {
      float* rw = red + (size_t)warp * 16 * RP;
      const int q = l & 3, g8 = l >> 2;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int cc = nt * 8 + 2 * q;
        rw[g8 * RP + cc] = zacc[nt][0];
        rw[g8 * RP + cc + 1] = zacc[nt][1];
        rw[(g8 + 8) * RP + cc] = zacc[nt][2];
        rw[(g8 + 8) * RP + cc + 1] = zacc[nt][3];
      }
    }
    __syncthreads();
    if (ksplit == 1) {
      for (int idx = tid; idx < AQ_ROWS * rank; idx += AQ_THREADS) {
        const int r = idx / rank, j = idx % rank, hb = r >> 4, r16 = r & 15;
        float sum = 0.0f;
#pragma unroll
        for (int gw = 0; gw < AQ_GPS; ++gw) sum += red[(size_t)(2 * gw + hb) * 16 * RP + r16 * RP + j];
        if (row0 + r < M)
          Z[(size_t)(row0 + r) * rank + j] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
      }
    } else {
      // this CTA's partial [32][rank], then the cluster's sum in CTA order
      float* zc = red + ST::RED / 4;
      if (!aborted) {
        for (int idx = tid; idx < AQ_ROWS * rank; idx += AQ_THREADS) {
          const int r = idx / rank, j = idx % rank, hb = r >> 4, r16 = r & 15;
          float sum = 0.0f;
#pragma unroll
          for (int gw = 0; gw < AQ_GPS; ++gw) sum += red[(size_t)(2 * gw + hb) * 16 * RP + r16 * RP + j];
          zc[idx] = sum;
        }
      }
      cluster_barrier();
      if (!aborted) {
        const uint32_t me = cluster_ctarank();
        const int ra = (int)me * AQ_ROWS / ksplit, rb2 = ((int)me + 1) * AQ_ROWS / ksplit;
        const uint32_t zc_s = smem_u32(zc);
        for (int idx = ra * rank + tid; idx < rb2 * rank; idx += AQ_THREADS) {
          const int r = idx / rank, j = idx % rank;
          float sum = 0.0f;
          for (int c = 0; c < ksplit; ++c) sum += ld_cluster_f32(zc_s + 4u * idx, (uint32_t)c);
          if (row0 + r < M)
            Z[(size_t)(row0 + r) * rank + j] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
        }
      }
      cluster_barrier();    // no CTA leaves while others read its partial
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 aq_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) ==
            cudaSuccess && qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2D bf16 map with a 64-column (128-byte), 128-byte-swizzled box.
bool aq_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch,
            uint32_t box_rows) {
  auto fn = aq_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NT, int FMT>
cudaError_t launch_aq(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                      uint8_t* xq, float* s_x, uint16_t* Z, uint8_t* sfa, cudaStream_t st) {
  using ST = AqStage<NT>;
  const size_t dyn = (size_t)ST::STAGES * ST::BYTES + 1024;
  static bool attr[64] = {};          // per device: the shared-memory limit is per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(act_quant_kernel<NT, FMT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e != cudaSuccess) return e;
    attr[dev] = true;
  }
  CUtensorMap tx, tl;
  if (!aq_map(&tx, X, (uint64_t)w->K, (uint64_t)M, (uint64_t)ldx * 2, AQ_ROWS))
    return cudaErrorInvalidValue;
  tl = tx;
  if (NT > 0 && !aq_map(&tl, w->d_L1T, (uint64_t)w->K, (uint64_t)NT * 8, (uint64_t)w->K * 2, NT * 8))
    return cudaErrorInvalidValue;
  // NVFP4: cover whole 128-row blocks, so that every scale-atom row is written
  const int rows = FMT == 2 ? (M + 127) / 128 * 128 : M;
  const int nrb = (rows + AQ_ROWS - 1) / AQ_ROWS;
  // W4A4 with few token blocks: split K over up to eight CTAs per block
  int ks = 1;
  if (FMT == 0) {
    ks = num_sms() / nrb;
    ks = ks < 1 ? 1 : (ks > 8 ? 8 : ks);
    if (ks > w->K / 64) ks = w->K / 64;
  }
  if (NT == 0 || ks == 1) {
    act_quant_kernel<NT, FMT><<<dim3(nrb * ks), ST::THREADS, dyn, st>>>(
        tx, tl, w->d_inv_lambda, M, w->K, w->rank, xq, s_x, Z, sfa, w->d_err, ks);
    return cudaGetLastError();
  }
  // the CTAs of a token block form a cluster (their Z partials meet in
  // distributed shared memory)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nrb * ks);
  cfg.blockDim = dim3(ST::THREADS);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = st;
  cudaLaunchAttribute attr_c[1];
  attr_c[0].id = cudaLaunchAttributeClusterDimension;
  attr_c[0].val.clusterDim.x = ks;
  attr_c[0].val.clusterDim.y = 1;
  attr_c[0].val.clusterDim.z = 1;
  cfg.attrs = attr_c;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, act_quant_kernel<NT, FMT>, tx, tl, (const float*)w->d_inv_lambda, M,
                            w->K, w->rank, xq, s_x, Z, sfa, (int*)w->d_err, ks);
}

template <int FMT>
cudaError_t launch_act(const svdq_weights* w, int M, const uint16_t* X, int ldx, uint8_t* xq,
                       float* s_x, uint16_t* Z, uint8_t* sfa, cudaStream_t st) {
  switch (w->rank_pad / 8) {
    case 0: return launch_aq<0, FMT>(w, M, X, ldx, xq, s_x, Z, sfa, st);
    case 2: return launch_aq<2, FMT>(w, M, X, ldx, xq, s_x, Z, sfa, st);
    case 4: return launch_aq<4, FMT>(w, M, X, ldx, xq, s_x, Z, sfa, st);
    case 6: return launch_aq<6, FMT>(w, M, X, ldx, xq, s_x, Z, sfa, st);
    case 8: return launch_aq<8, FMT>(w, M, X, ldx, xq, s_x, Z, sfa, st);
    case 10: return launch_aq<10, FMT>(w, M, X, ldx, xq, s_x, Z, sfa, st);
    case 12: return launch_aq<12, FMT>(w, M, X, ldx, xq, s_x, Z, sfa, st);
    case 14: return launch_aq<14, FMT>(w, M, X, ldx, xq, s_x, Z, sfa, st);
    case 16: return launch_aq<16, FMT>(w, M, X, ldx, xq, s_x, Z, sfa, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_act_quant(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                             uint8_t* xq, float* s_x, uint16_t* Z, cudaStream_t st) {
  return launch_act<0>(w, M, X, ldx, xq, s_x, Z, nullptr, st);
}

cudaError_t launch_act_quant_w8a8(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                                  int8_t* xq, float* s_x, uint16_t* Z, cudaStream_t st) {
  return launch_act<1>(w, M, X, ldx, reinterpret_cast<uint8_t*>(xq), s_x, Z, nullptr, st);
}

cudaError_t launch_act_quant_nvfp4(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                                   uint8_t* xq, uint8_t* sfa, float* s_x, uint16_t* Z,
                                   cudaStream_t st) {
  return launch_act<2>(w, M, X, ldx, xq, s_x, Z, sfa, st);
}

}  // namespace svdq
