// W4A4 product with the 16-bit up-projection fused into the epilogue
// (SVDQuant review section 6.1, Algorithm 2 steps 4-8; eq. 7).
//
// sm_100a tensor cores have no 4-bit integer kind, so the packed codes are
// expanded to int8 in shared memory and multiplied with
// tcgen05.mma.kind::i8 (int32 accumulation in TMEM).  Each group of 64 K
// gets its own int32 partial P_g (two K=32 MMAs), which the epilogue threads
// read back with tcgen05.ld and fold into an fp32 accumulator with the
// group's scales s_x[g][m] s_w[g][n].  Finally Z L2 and the bias are added
// and Y is written once as bf16.
//
// This is the straightforward form of the kernel: one 128 x 128 output tile
// per CTA of 4 warps; per group every thread expands one row of A and one
// row of B, thread 0 issues the MMAs, and all threads rescale their TMEM
// lane (= output row).
//
// Expanded operand layout (K-major, no swizzle): a 64-byte K row is four
// 16-byte core-matrix rows; the core matrix (row group r/8, K chunk c) sits
// at (r/8)*512 + c*128, row r%8 at +16*(r%8).  Within every 8 codes the
// expansion stores the even-k codes first and the odd-k codes after them;
// A and B use the same order, so each group's dot product is unchanged.
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int LIN_THREADS = 128;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s per wait

// Expand the 32 packed bytes (64 codes) of one row-group into the shared
// memory layout above.
__device__ __forceinline__ void expand_row(const uint8_t* __restrict__ src, bool valid,
                                           uint8_t* dst_row_base) {
  uint4 p0 = make_uint4(0u, 0u, 0u, 0u), p1 = p0;
  if (valid) {
    p0 = __ldg(reinterpret_cast<const uint4*>(src));
    p1 = __ldg(reinterpret_cast<const uint4*>(src + 16));
  }
  const uint32_t wds[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 o;
    const uint32_t w0 = wds[2 * c], w1 = wds[2 * c + 1];
    o.x = sext_nibbles(w0 & 0x0F0F0F0Fu);
    o.y = sext_nibbles((w0 >> 4) & 0x0F0F0F0Fu);
    o.z = sext_nibbles(w1 & 0x0F0F0F0Fu);
    o.w = sext_nibbles((w1 >> 4) & 0x0F0F0F0Fu);
    *reinterpret_cast<uint4*>(dst_row_base + c * 128) = o;
  }
}

__device__ __forceinline__ float gelu_f(float y) {
  return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f));
}

template <bool DUMP>
__global__ void __launch_bounds__(LIN_THREADS)
linear_kernel(const uint8_t* __restrict__ xq, const float* __restrict__ s_x,
              const uint16_t* __restrict__ Z, const uint8_t* __restrict__ wq,
              const float* __restrict__ s_w, const uint16_t* __restrict__ L2,
              const uint16_t* __restrict__ bias, uint16_t* __restrict__ Y, int ldy,
              int M, int N, int K, int rank, int epilogue, int* __restrict__ err,
              int32_t* __restrict__ P, int row0, int nrows, int col0, int ncols,
              int tile_m0, int tile_n0) {
  __shared__ __align__(128) uint8_t sA[BM * 64];
  __shared__ __align__(128) uint8_t sB[BN * 64];
  __shared__ float sw_s[BN];
  __shared__ __align__(8) uint64_t mbar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int m0 = (tile_m0 + blockIdx.y) * BM;
  const int n0 = (tile_n0 + blockIdx.x) * BN;
  const int G = K / 64;
  const int KB = K / 2;

  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base_sh), BN);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(smem_u32(&mbar), 1);
    fence_mbarrier_init();
    abort_sh = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t tmem_warp = tmem + ((uint32_t)(warp * 32) << 16);

  const int row = m0 + tid;               // this thread's A row and output row
  const int brow = n0 + tid;              // this thread's B row
  uint8_t* a_dst = sA + (tid >> 3) * 512 + (tid & 7) * 16;
  uint8_t* b_dst = sB + (tid >> 3) * 512 + (tid & 7) * 16;
  const uint32_t idesc = idesc_i8(BM, BN);
  const uint64_t adesc = sdesc_kmajor_noswizzle(smem_u32(sA), 128, 512);
  const uint64_t bdesc = sdesc_kmajor_noswizzle(smem_u32(sB), 128, 512);

  float acc[BN];
#pragma unroll
  for (int j = 0; j < BN; ++j) acc[j] = 0.0f;

  for (int g = 0; g < G; ++g) {
    expand_row(xq + (size_t)row * KB + g * 32, row < M, a_dst);
    expand_row(wq + (size_t)brow * KB + g * 32, brow < N, b_dst);
    if (!DUMP) sw_s[tid] = (brow < N) ? s_w[(size_t)g * N + brow] : 0.0f;
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      mma_i8(tmem, adesc, bdesc, idesc, 0u);
      mma_i8(tmem, adesc + (256 >> 4), bdesc + (256 >> 4), idesc, 1u);
      mma_commit(smem_u32(&mbar));
    }
    if (!mbar_wait_bounded(smem_u32(&mbar), (uint32_t)(g & 1), WAIT_LIMIT_NS)) {
      atomicExch(err, SVDQ_DEVERR_TIMEOUT);
      abort_sh = 1;
    }
    tc_fence_after();
    if (DUMP) {
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_warp + c0, r);
        tmem_wait_ld();
        const int i = row - row0;
        if (i >= 0 && i < nrows) {
          for (int j = 0; j < 32; ++j) {
            const int jj = n0 + c0 + j - col0;
            if (jj >= 0 && jj < ncols)
              P[((size_t)g * nrows + i) * ncols + jj] = (int32_t)r[j];
          }
        }
      }
    } else {
      const float sx = (row < M) ? s_x[(size_t)g * M + row] : 0.0f;
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_warp + c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          acc[c0 + j] = fmaf(sx * sw_s[c0 + j], (float)(int32_t)r[j], acc[c0 + j]);
      }
    }
    tc_fence_before();
    __syncthreads();
    if (abort_sh) break;
  }

  if (!DUMP && !abort_sh && row < M) {
    for (int j = 0; j < rank; ++j) {
      const float z = __uint_as_float((uint32_t)Z[(size_t)row * rank + j] << 16);
      const uint16_t* l2 = L2 + (size_t)j * N + n0;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        const float v = (n0 + c < N) ? __uint_as_float((uint32_t)__ldg(l2 + c) << 16) : 0.0f;
        acc[c] = fmaf(z, v, acc[c]);
      }
    }
#pragma unroll
    for (int c = 0; c < BN; ++c) {
      const int n = n0 + c;
      if (n < N) {
        float y = acc[c] + __uint_as_float((uint32_t)__ldg(bias + n) << 16);
        if (epilogue == SVDQ_EPI_GELU) y = gelu_f(y);
        Y[(size_t)row * ldy + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

}  // namespace

cudaError_t launch_linear(const svdq_weights* w, int M, const uint8_t* xq, const float* s_x,
                          const uint16_t* Z, uint16_t* Y, int ldy, int epilogue,
                          cudaStream_t st) {
  const dim3 grid((w->N + BN - 1) / BN, (M + BM - 1) / BM);
  linear_kernel<false><<<grid, LIN_THREADS, 0, st>>>(
      xq, s_x, Z, w->d_wq, w->d_sw, w->d_L2, w->d_bias, Y, ldy, M, w->N, w->K, w->rank,
      epilogue, w->d_err, nullptr, 0, 0, 0, 0, 0, 0);
  return cudaGetLastError();
}

cudaError_t launch_partials(const svdq_weights* w, int M, const uint8_t* xq, int row0,
                            int nrows, int col0, int ncols, int32_t* P, cudaStream_t st) {
  const int tm0 = row0 / BM, tm1 = (row0 + nrows - 1) / BM;
  const int tn0 = col0 / BN, tn1 = (col0 + ncols - 1) / BN;
  const dim3 grid(tn1 - tn0 + 1, tm1 - tm0 + 1);
  linear_kernel<true><<<grid, LIN_THREADS, 0, st>>>(
      xq, nullptr, nullptr, w->d_wq, nullptr, nullptr, nullptr, nullptr, 0, M, w->N, w->K,
      0, 0, w->d_err, P, row0, nrows, col0, ncols, tm0, tn0);
  return cudaGetLastError();
}

}  // namespace svdq
