// Fused activation pass (SVDQuant review section 6.1, activation side):
// read X once, smooth it (eq. 3), quantise it per token and group of 64
// (eq. 1) and, from the same tile, compute the 16-bit down-projection
// Z = bf16(x~) L1 on the tensor cores (mma.sync bf16, fp32 accumulation).
//
// Layout: one CTA of 8 warps owns 16 consecutive tokens and walks K in
// chunks of 256 channels (several CTAs per SM).  TMA streams 16 x 256 bf16
// tiles of X into a 6-stage shared-memory ring, so X is read from HBM
// exactly once with full-width transactions.  A warp reads one token's 256
// channels from the ring (16 bytes per lane); the 8 lanes holding one group
// of 64 find its absmax with three xor-shuffles.  bf16(x~) is staged in
// shared memory for the MMA; the scale tile is staged so that s_x[g][m] is
// written with contiguous stores.
//
// Bit-exact quantiser: x~ = fl32(x * inv_lambda) (one IEEE multiply),
// s = fl32(m / 7) (IEEE division), and the code is round-half-even of the
// exact quotient x~/s: a first guess from the correctly rounded reciprocal
// is corrected with the exact residual x~ - q s computed by an fma.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int AQ_ROWS = 16;
constexpr int AQ_CH = 256;
constexpr int AQ_THREADS = 256;
constexpr int AQ_STAGES = 6;
constexpr int AQ_STAGE_BYTES = AQ_ROWS * AQ_CH * 2;     // 8 KB
constexpr uint64_t AQ_LIMIT_NS = 2000000000ull;

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
// Two floats -> packed bf16x2 bits (round to nearest even), a in the low half.
__device__ __forceinline__ uint32_t bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

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

// All 8 codes of a lane by the exact path (rare; kept out of line).
__device__ __noinline__ uint32_t quant8_exact(const float* xh, float ssc, float rcp, float scale) {
  uint32_t packed = 0u;
#pragma unroll
  for (int j = 0; j < 8; ++j) packed |= quant_nibble(xh[j], ssc, rcp, scale) << (4 * j);
  return packed;
}

// Fast path of the same rounding for a normal scale s: t = fl(x * fl(1/s))
// is within |x/s| 2^-23 <= 2^-20 of the exact quotient (|x/s| <= 7 + 2^-21),
// so unless t lies within 2^-20 of a half-integer, rne(t) = rne(x/s).  Sets
// `near` when that margin is not met (the caller then takes the exact path).
__device__ __forceinline__ uint32_t quant_nibble_fast(float x, float rcp, bool& near) {
  const float t = __fmul_rn(x, rcp);
  const float b0 = __fadd_rn(t, RN_MAGIC);
  const float f = __fsub_rn(t, __fsub_rn(b0, RN_MAGIC));     // t - rne(t), exact
  near |= fabsf(fabsf(f) - 0.5f) <= 0x1p-20f;
  return __float_as_uint(b0) & 0xFu;                          // |rne(t)| <= 7
}

template <int NT>
__global__ void __launch_bounds__(AQ_THREADS)
act_quant_kernel(const __grid_constant__ CUtensorMap tm_x, int box_cols,
                 const float* __restrict__ inv_lambda,
                 const uint16_t* __restrict__ L1T,   // [NT*8][K] bf16
                 int M, int K, int rank,
                 uint8_t* __restrict__ xq, float* __restrict__ s_x,
                 uint16_t* __restrict__ Z, int* __restrict__ err) {
  __shared__ __align__(16) uint16_t xs[AQ_ROWS][AQ_CH + 8];
  __shared__ float ss_tile[AQ_CH / 64][AQ_ROWS];
  __shared__ __align__(8) uint64_t full_bar[AQ_STAGES];
  __shared__ int abort_sh;
  // dynamic: [AQ_STAGES][32 rows][box_cols] bf16 ring (1024-B aligned),
  // then [8][AQ_ROWS][NT*8] fp32 reduction buffer when NT > 0
  extern __shared__ uint8_t aq_dyn_raw[];
  uint8_t* aq_dyn = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(aq_dyn_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = aq_dyn;
  float* red = reinterpret_cast<float*>(aq_dyn + AQ_STAGES * AQ_STAGE_BYTES);

  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  const int row0 = blockIdx.x * AQ_ROWS;
  const int G = K / 64;
  const int nchunks = (K + AQ_CH - 1) / AQ_CH;

  float zacc[1][NT > 0 ? NT : 1][4];
#pragma unroll
  for (int a = 0; a < 1; ++a)
#pragma unroll
    for (int b = 0; b < (NT > 0 ? NT : 1); ++b)
#pragma unroll
      for (int c = 0; c < 4; ++c) zacc[a][b][c] = 0.0f;

  const uint32_t stage_bytes = (uint32_t)box_cols * AQ_ROWS * 2;
  if (tid == 0) {
    for (int s = 0; s < AQ_STAGES; ++s) mbar_init(smem_u32(&full_bar[s]), 1);
    abort_sh = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int c = 0; c < AQ_STAGES && c < nchunks; ++c) {
      mbar_arrive_expect_tx(smem_u32(&full_bar[c]), stage_bytes);
      tma_load_2d(smem_u32(ring + c * AQ_STAGE_BYTES), &tm_x, c * AQ_CH, row0,
                  smem_u32(&full_bar[c]));
    }
  }

  // L1 fragments of the chunk's two k16 steps; for NT <= 8 the next chunk's
  // are prefetched while this chunk is quantised
  constexpr bool PF = NT > 0 && NT <= 8;
  constexpr int NTB = NT > 0 ? NT : 1;
  uint32_t bfr[2][NTB][2], bnx[2][NTB][2];
  auto load_frags = [&](int c, uint32_t (&dst)[2][NTB][2]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int kglob = c * AQ_CH + (w + 8 * h) * 16;
#pragma unroll
      for (int nt = 0; nt < NTB; ++nt) {
        if (NT > 0 && kglob < K) {
          const uint16_t* bp = L1T + (size_t)(nt * 8 + (l >> 2)) * K + kglob + 2 * (l & 3);
          dst[h][nt][0] = __ldg(reinterpret_cast<const uint32_t*>(bp));
          dst[h][nt][1] = __ldg(reinterpret_cast<const uint32_t*>(bp + 8));
        } else {
          dst[h][nt][0] = dst[h][nt][1] = 0u;
        }
      }
    }
  };
  if (PF) load_frags(0, bfr);
  // smoothing factors of the lane's 8 channels, prefetched one chunk ahead
  auto load_il = [&](int c, float (&dst)[8]) {
    const int col = c * AQ_CH + l * 8;
    if (col < K) {
      const float4 i0 = __ldg(reinterpret_cast<const float4*>(inv_lambda + col));
      const float4 i1 = __ldg(reinterpret_cast<const float4*>(inv_lambda + col + 4));
      dst[0] = i0.x; dst[1] = i0.y; dst[2] = i0.z; dst[3] = i0.w;
      dst[4] = i1.x; dst[5] = i1.y; dst[6] = i1.z; dst[7] = i1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) dst[j] = 0.0f;
    }
  };
  float il[8], il_nx[8];
  load_il(0, il);

  for (int c = 0; c < nchunks; ++c) {
    const int st = c % AQ_STAGES;
    if (PF && c + 1 < nchunks) load_frags(c + 1, bnx);
    if (c + 1 < nchunks) load_il(c + 1, il_nx);
    if (!mbar_wait_bounded(smem_u32(&full_bar[st]), (c / AQ_STAGES) & 1, AQ_LIMIT_NS)) {
      atomicExch(err, SVDQ_DEVERR_TIMEOUT);
      abort_sh = 1;
    }
    __syncthreads();
    if (abort_sh) break;
    uint4 cur[2];
    const uint8_t* stage = ring + st * AQ_STAGE_BYTES;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
      cur[rr] = (l * 8 < box_cols)
                    ? *reinterpret_cast<const uint4*>(stage + (w + 8 * rr) * box_cols * 2 + l * 16)
                    : make_uint4(0u, 0u, 0u, 0u);
    const int col = c * AQ_CH + l * 8;
    const bool colok = col < K;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int lr = w + 8 * rr;
      const int row = row0 + lr;
      const uint32_t u[4] = {cur[rr].x, cur[rr].y, cur[rr].z, cur[rr].w};
      float xh[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xh[2 * j] = __fmul_rn(bf16lo(u[j]), il[2 * j]);
        xh[2 * j + 1] = __fmul_rn(bf16hi(u[j]), il[2 * j + 1]);
      }
      float m = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(xh[j]));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
      const float s = __fdiv_rn(m, 7.0f);
      uint32_t packed = 0u;
      if (s > 0.0f) {
        const bool tiny = s < 0x1p-64f;         // s subnormal or nearly: exact path
        bool near = tiny;
        const float scale = tiny ? 0x1p64f : 1.0f;
        const float ssc = __fmul_rn(s, scale);
        const float rcp = __frcp_rn(ssc);
        if (!tiny) {
#pragma unroll
          for (int j = 0; j < 8; ++j) packed |= quant_nibble_fast(xh[j], rcp, near) << (4 * j);
        }
        if (near) packed = quant8_exact(xh, ssc, rcp, scale);   // rare: exact residual
      }
      if (colok && row < M)
        *reinterpret_cast<uint32_t*>(xq + (size_t)row * (K / 2) + col / 2) = packed;
      if ((l & 7) == 0) ss_tile[l >> 3][lr] = s;
      uint4 hv;
      hv.x = bf16x2(xh[0], xh[1]);
      hv.y = bf16x2(xh[2], xh[3]);
      hv.z = bf16x2(xh[4], xh[5]);
      hv.w = bf16x2(xh[6], xh[7]);
      *reinterpret_cast<uint4*>(&xs[lr][l * 8]) = hv;
    }
    __syncthreads();
    if (tid < (AQ_CH / 64) * AQ_ROWS) {
      const int g = c * (AQ_CH / 64) + tid / AQ_ROWS;
      const int row = row0 + tid % AQ_ROWS;
      if (g < G && row < M) s_x[(size_t)g * M + row] = ss_tile[tid / AQ_ROWS][tid % AQ_ROWS];
    }
    if constexpr (NT > 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int kc = (w + 8 * h) * 16;          // k16 step inside the chunk
        const int kglob = c * AQ_CH + kc;
        if (kglob < K) {
          uint32_t a[1][4];
          ldmatrix_x4(smem_u32(&xs[l & 15][kc + (l >> 4) * 8]), a[0]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            uint32_t b0, b1;
            if (PF) {
              b0 = bfr[h][nt][0];
              b1 = bfr[h][nt][1];
            } else {
              const uint16_t* bp = L1T + (size_t)(nt * 8 + (l >> 2)) * K + kglob + 2 * (l & 3);
              b0 = __ldg(reinterpret_cast<const uint32_t*>(bp));
              b1 = __ldg(reinterpret_cast<const uint32_t*>(bp + 8));
            }
            mma_bf16_16816(zacc[0][nt], a[0], b0, b1);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) il[j] = il_nx[j];
    if (PF) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int nt = 0; nt < NTB; ++nt) {
          bfr[h][nt][0] = bnx[h][nt][0];
          bfr[h][nt][1] = bnx[h][nt][1];
        }
    }
    __syncthreads();
    if (tid == 0 && c + AQ_STAGES < nchunks) {
      mbar_arrive_expect_tx(smem_u32(&full_bar[st]), stage_bytes);
      tma_load_2d(smem_u32(ring + st * AQ_STAGE_BYTES), &tm_x, (c + AQ_STAGES) * AQ_CH, row0,
                  smem_u32(&full_bar[st]));
    }
  }
  if (abort_sh) {
    // let every issued copy land before the CTA exits
    if (tid == 0)
      for (int c = 0; c < AQ_STAGES && c < nchunks; ++c)
        mbar_wait_bounded(smem_u32(&full_bar[c]), 0, AQ_LIMIT_NS);
    return;
  }

  if constexpr (NT > 0) {
    constexpr int RP = NT * 8;
    float* rw = red + (size_t)w * AQ_ROWS * RP;
#pragma unroll
    for (int mt = 0; mt < 1; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int r = mt * 16 + (l >> 2);
        const int cc = nt * 8 + 2 * (l & 3);
        rw[r * RP + cc] = zacc[mt][nt][0];
        rw[r * RP + cc + 1] = zacc[mt][nt][1];
        rw[(r + 8) * RP + cc] = zacc[mt][nt][2];
        rw[(r + 8) * RP + cc + 1] = zacc[mt][nt][3];
      }
    __syncthreads();
    for (int idx = tid; idx < AQ_ROWS * rank; idx += AQ_THREADS) {
      const int r = idx / rank, j = idx % rank;
      float sum = 0.0f;
#pragma unroll
      for (int ww = 0; ww < 8; ++ww) sum += red[(size_t)ww * AQ_ROWS * RP + r * RP + j];
      if (row0 + r < M)
        Z[(size_t)(row0 + r) * rank + j] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 aq_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

template <int NT>
cudaError_t launch_aq(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                      uint8_t* xq, float* s_x, uint16_t* Z, cudaStream_t st) {
  const size_t red_bytes = NT > 0 ? (size_t)8 * AQ_ROWS * NT * 8 * sizeof(float) : 0;
  const size_t dyn = (size_t)AQ_STAGES * AQ_STAGE_BYTES + red_bytes + 1024;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(act_quant_kernel<NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  auto fn = aq_encode_fn();
  if (!fn) return cudaErrorInvalidValue;
  const int box_cols = w->K < AQ_CH ? w->K : AQ_CH;
  CUtensorMap tm;
  const cuuint64_t dims[2] = {(cuuint64_t)w->K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)AQ_ROWS};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides,
         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const dim3 grid((M + AQ_ROWS - 1) / AQ_ROWS);
  act_quant_kernel<NT><<<grid, AQ_THREADS, dyn, st>>>(
      tm, box_cols, w->d_inv_lambda, w->d_L1T, M, w->K, w->rank, xq, s_x, Z, w->d_err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_act_quant(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                             uint8_t* xq, float* s_x, uint16_t* Z, cudaStream_t st) {
  switch (w->rank_pad / 8) {
    case 0: return launch_aq<0>(w, M, X, ldx, xq, s_x, Z, st);
    case 2: return launch_aq<2>(w, M, X, ldx, xq, s_x, Z, st);
    case 4: return launch_aq<4>(w, M, X, ldx, xq, s_x, Z, st);
    case 6: return launch_aq<6>(w, M, X, ldx, xq, s_x, Z, st);
    case 8: return launch_aq<8>(w, M, X, ldx, xq, s_x, Z, st);
    case 10: return launch_aq<10>(w, M, X, ldx, xq, s_x, Z, st);
    case 12: return launch_aq<12>(w, M, X, ldx, xq, s_x, Z, st);
    case 14: return launch_aq<14>(w, M, X, ldx, xq, s_x, Z, st);
    case 16: return launch_aq<16>(w, M, X, ldx, xq, s_x, Z, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace svdq
