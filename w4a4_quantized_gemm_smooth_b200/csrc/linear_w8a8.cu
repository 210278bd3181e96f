// W8A8 comparator product (SVDQuant review section 8: the eight-bit
// setting with per-token activation and per-channel weight scales; its INT8
// rows in section 9.3), warp-specialised for sm_100a:
//
//   Y = bf16(epi(s_x[m] s_w[n] sum_k q_x[m][k] q_w[n][k] + Z L2 + b))
//
// With one scale per token and per output channel the integer product needs
// no per-group rescale: the int8 codes are copied by TMA straight into the
// tensor-core operand layout (no expansion step; 64-byte K rows with the
// 64-byte swizzle, one TMA box per operand and stage) and tcgen05.mma.kind::i8
// accumulates the whole K range of a 128 x 256 output tile into one int32
// TMEM accumulator (|sum| <= 127^2 K < 2^31 for K <= 2^17).  The epilogue
// converts it once (int32 -> fp32, exact below 2^24, one rounding above),
// scales it by s_x s_w, adds the low-rank product Z L2 (a kind::f16 stage
// into the other TMEM buffer, as in the W4A4 kernel), the bias and GELU,
// and stores Y by TMA.
//
// Persistent CTAs (one per SM), static round-robin tiles; 16 warps:
//   warp 0      TMA producer: 64-K stages of A (128 x 64 B) and B (256 x
//               64 B), each one box of 64-byte rows; per-tile scales;
//               low-rank slices (16-byte-wide boxes, no swizzle);
//   warp 1      TMEM owner and MMA issuer (one thread);
//   warps 2-7   idle (they keep the warp-to-TMEM-lane mapping of the
//               epilogue warps and the register split of the W4A4 kernel);
//   warps 8-15  epilogue: warp w owns TMEM lanes 32 (w % 4).. and 128
//               columns.  Two 256-column TMEM buffers alternate between a
//               tile's integer product and its low-rank product, so a tile's
//               low-rank stage runs while its product is drained.
// Every wait is bounded (the handle's error word is raised on expiry).
#include "gemm_common.cuh"

namespace svdq {
namespace {

constexpr int W8_BM = 128, W8_BN = 256;
constexpr int W8_THREADS = 512;
constexpr int W8_EPI0 = 8;        // epilogue warps 8-15
constexpr int W8_NEPI = 8;
constexpr int W8_REG_LO = 56, W8_REG_HI = 200;
constexpr int W8_REG_NEED = (256 * W8_REG_LO + 256 * W8_REG_HI + W8_THREADS - 1) / W8_THREADS;

__device__ __forceinline__ float2 lds64f(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

// Shared-memory descriptor of a K-major operand stored as 64-byte rows with
// the 64-byte swizzle (8-row atoms of 512 B, as TMA writes them): the stride
// between 8-row groups is 512 B; the leading offset is unused for this layout
// (encoded as 1).  Layout type 4 = 64-byte swizzle, version 1.  Advancing the
// start address by 32 B selects the second K half of the row.
__device__ __forceinline__ uint64_t sdesc_kmajor_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(512 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)4 << 61;
  return d;
}

struct W8Args {
  const float* s_x;
  const float* s_w;
  const uint16_t* bias;
  int M, N, K, G;
  int n_lr;                  // 16-wide low-rank slices, ceil(rank / 16)
  int epilogue;
  int tiles_n, num_tiles;
  int* err;
};

struct W8Lay {
  static constexpr int BM = W8_BM, BN = W8_BN;
  static constexpr int CW = BN / 2;                       // columns per epilogue warp
  static constexpr int Y_BOX = 32 * 64 * 2;               // 32 rows x 64 bf16
  static constexpr int Y_WARP = (CW / 64) * Y_BOX;
  static constexpr int ST_A = BM * 64, ST_B = BN * 64, STAGE = ST_A + ST_B;   // 64 K of int8
  static constexpr int NST = 5;
  static constexpr int NLR = 2;
  static constexpr int LR_SA = BM * 32, LR_SB = BN * 32, LR_SLOT = LR_SA + LR_SB;
  static constexpr int SC_SLOT = (BM + BN) * 4;          // s_x[128], then s_w[256]
  static constexpr int OFF_Y = 0;
  static constexpr int OFF_ST = OFF_Y + W8_NEPI * Y_WARP;
  static constexpr int OFF_LR = OFF_ST + NST * STAGE;
  static constexpr int OFF_SC = OFF_LR + NLR * LR_SLOT;
  static constexpr int OFF_BIAS = OFF_SC + 2 * SC_SLOT;
  static constexpr int OFF_BAR = OFF_BIAS + W8_NEPI * CW * 4;
  // st_full[NST], st_empty[NST], tm_full[2], tm_empty[2], lr_full[NLR],
  // lr_empty[NLR], sc_full[2], sc_empty[2]
  static constexpr int N_BARS = 2 * NST + 4 + 2 * NLR + 4;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

__global__ void __launch_bounds__(W8_THREADS, 1)
linear_w8a8_kernel(const __grid_constant__ CUtensorMap tm_a,
                   const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_y,
                   const __grid_constant__ CUtensorMap tm_z,
                   const __grid_constant__ CUtensorMap tm_l2,
                   const __grid_constant__ CUtensorMap tm_sx,
                   const __grid_constant__ CUtensorMap tm_sw, const W8Args p) {
  using L = W8Lay;
  constexpr int BM = L::BM, BN = L::BN, CW = L::CW, NST = L::NST, NLR = L::NLR;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::OFF_BAR;
  auto st_full = [&](int s) { return bar0 + 8u * s; };
  auto st_empty = [&](int s) { return bar0 + 8u * (NST + s); };
  auto tm_full = [&](int b) { return bar0 + 8u * (2 * NST + b); };
  auto tm_empty = [&](int b) { return bar0 + 8u * (2 * NST + 2 + b); };
  auto lr_full = [&](int s) { return bar0 + 8u * (2 * NST + 4 + s); };
  auto lr_empty = [&](int s) { return bar0 + 8u * (2 * NST + 4 + NLR + s); };
  auto sc_full = [&](int s) { return bar0 + 8u * (2 * NST + 4 + 2 * NLR + s); };
  auto sc_empty = [&](int s) { return bar0 + 8u * (2 * NST + 4 + 2 * NLR + 2 + s); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.G;

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) { mbar_init(st_full(s), 1); mbar_init(st_empty(s), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tm_full(b), 1); mbar_init(tm_empty(b), W8_NEPI); }
    for (int s = 0; s < NLR; ++s) { mbar_init(lr_full(s), 1); mbar_init(lr_empty(s), 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(sc_full(s), 1); mbar_init(sc_empty(s), W8_NEPI); }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < W8_EPI0) {
    regs_dec<W8_REG_LO>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------- TMA producer
      uint32_t it = 0, il = 0, ti = 0;
      bool alive = true;
      for (int t = blockIdx.x; t < p.num_tiles && alive; t += gridDim.x, ++ti) {
        const int m0 = (t / p.tiles_n) * BM, n0 = (t % p.tiles_n) * BN;
        const int sc = ti & 1;
        if (!wait_or_abort(sc_empty(sc), ((ti >> 1) & 1) ^ 1, abort_flag, p.err)) break;
        const uint32_t slot = sbase + L::OFF_SC + sc * L::SC_SLOT;
        mbar_arrive_expect_tx(sc_full(sc), L::SC_SLOT);
        tma_load_2d(slot, &tm_sx, m0, 0, sc_full(sc));
        tma_load_2d(slot + 4 * BM, &tm_sw, n0, 0, sc_full(sc));
        for (int g = 0; g < G; ++g, ++it) {
          const int s = it % NST;
          if (!wait_or_abort(st_empty(s), ((it / NST) & 1) ^ 1, abort_flag, p.err)) { alive = false; break; }
          mbar_arrive_expect_tx(st_full(s), L::STAGE);
          const uint32_t dst = sbase + L::OFF_ST + s * L::STAGE;
          tma_load_2d(dst, &tm_a, g * 64, m0, st_full(s));
          tma_load_2d(dst + L::ST_A, &tm_b, g * 64, n0, st_full(s));
        }
        for (int j = 0; j < p.n_lr && alive; ++j, ++il) {
          const int ls = il % NLR;
          if (!wait_or_abort(lr_empty(ls), ((il / NLR) & 1) ^ 1, abort_flag, p.err)) { alive = false; break; }
          mbar_arrive_expect_tx(lr_full(ls), L::LR_SLOT);
          const uint32_t dst = sbase + L::OFF_LR + ls * L::LR_SLOT;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tma_load_2d(dst + c * (BM * 16), &tm_z, 16 * j + 8 * c, m0, lr_full(ls));
            tma_load_2d(dst + L::LR_SA + c * (BN * 16), &tm_l2, 16 * j + 8 * c, n0, lr_full(ls));
          }
        }
      }
      // every issued copy has landed before the CTA exits
      for (uint32_t k = (it > NST ? it - NST : 0); k < it; ++k)
        mbar_wait_bounded(st_full(k % NST), (k / NST) & 1, LIMIT_NS);
      for (uint32_t k = (il > NLR ? il - NLR : 0); k < il; ++k)
        mbar_wait_bounded(lr_full(k % NLR), (k / NLR) & 1, LIMIT_NS);
      for (uint32_t k = (ti > 2 ? ti - 2 : 0); k < ti; ++k)
        mbar_wait_bounded(sc_full(k & 1), (k >> 1) & 1, LIMIT_NS);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------- MMA issuer
      const uint32_t id_i8 = idesc_i8(BM, BN), id_bf = idesc_bf16(BM, BN);
      uint32_t it = 0, tb = 0, il = 0;
      for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
        int b = tb & 1;
        if (!wait_or_abort(tm_empty(b), ((tb >> 1) & 1) ^ 1, abort_flag, p.err)) break;
        uint32_t d = tmem + b * BN;
        bool ok = true;
        for (int g = 0; g < G; ++g, ++it) {
          const int s = it % NST;
          if (!wait_or_abort(st_full(s), (it / NST) & 1, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = sbase + L::OFF_ST + s * L::STAGE, sb = sa + L::ST_A;
#pragma unroll
          for (int h = 0; h < 2; ++h) {     // K = 32 each: bytes 32h .. 32h+31 of the rows
            const uint64_t ad = sdesc_kmajor_sw64(sa + 32 * h);
            const uint64_t bd = sdesc_kmajor_sw64(sb + 32 * h);
            mma_i8(d, ad, bd, id_i8, (g > 0 || h > 0) ? 1u : 0u);
          }
          mma_commit(st_empty(s));
        }
        if (!ok) break;
        mma_commit(tm_full(b));
        ++tb;
        if (p.n_lr > 0) {
          b = tb & 1;
          if (!wait_or_abort(tm_empty(b), ((tb >> 1) & 1) ^ 1, abort_flag, p.err)) break;
          d = tmem + b * BN;
          for (int j = 0; j < p.n_lr; ++j, ++il) {
            const int ls = il % NLR;
            if (!wait_or_abort(lr_full(ls), (il / NLR) & 1, abort_flag, p.err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t la = sbase + L::OFF_LR + ls * L::LR_SLOT;
            const uint64_t ad = sdesc_kmajor_noswizzle(la, BM * 16, 128);
            const uint64_t bd = sdesc_kmajor_noswizzle(la + L::LR_SA, BN * 16, 128);
            mma_bf16(d, ad, bd, id_bf, j > 0 ? 1u : 0u);
            mma_commit(lr_empty(ls));
          }
          if (!ok) break;
          mma_commit(tm_full(b));
          ++tb;
        }
      }
    }
    __syncwarp();
  } else {
    regs_inc<W8_REG_HI>();
    // ------------------------------------------------------ epilogue
    // .16x256b loads: this thread owns rows r0 + 8i (i < 4) of the warp's
    // quarter and, in each 16-column chunk c, the column pairs
    // 16c + 8b + 2pq (+1), b < 2; acc[i][2c + b] holds that pair.
    const int rw = warp - W8_EPI0, q = warp & 3, h = rw >> 2;
    const int pq = lane & 3, r0 = lane >> 2;
    float* bb = reinterpret_cast<float*>(smem + L::OFF_BIAS) + rw * CW;
    uint8_t* ystage = smem + L::OFF_Y + rw * L::Y_WARP;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    uint32_t tb = 0, ti = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++ti) {
      const int m0 = (t / p.tiles_n) * BM, n0 = (t % p.tiles_n) * BN;
      const int ncol0 = n0 + h * CW;
      constexpr int PER = CW / 32;
      float bias_n[PER];
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int n = ncol0 + lane * PER + e;
        bias_n[e] = n < p.N ? __uint_as_float((uint32_t)__ldg(p.bias + n) << 16) : 0.0f;
      }
      float2 acc[4][CW / 8];
      // integer product: one conversion and one scaling per output
      {
        const int sc = ti & 1;
        if (!wait_or_abort(sc_full(sc), (ti >> 1) & 1, abort_flag, p.err)) { ok = false; break; }
        const uint32_t slot = sbase + L::OFF_SC + sc * L::SC_SLOT;
        float2 sx2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float v = lds32(slot + 4u * (32 * q + r0 + 8 * i));
          sx2[i] = make_float2(v, v);
        }
        const int b = tb & 1;
        if (!wait_or_abort(tm_full(b), (tb >> 1) & 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ta = tmem + b * BN + h * CW + lane_off;
        const uint32_t swa = slot + 4u * (BM + h * CW) + 8u * pq;
        uint32_t rb[2][16];
        tmem_ld16x256b_x2(ta, &rb[0][0]);
        tmem_ld16x256b_x2(ta + (16u << 16), &rb[0][8]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < CW / 16; ++c) {
          if (c + 1 < CW / 16) {
            tmem_ld16x256b_x2(ta + 16 * (c + 1), &rb[(c + 1) & 1][0]);
            tmem_ld16x256b_x2(ta + 16 * (c + 1) + (16u << 16), &rb[(c + 1) & 1][8]);
          }
          const uint32_t* r = rb[c & 1];
#pragma unroll
          for (int b2 = 0; b2 < 2; ++b2) {
            const float2 sw2 = lds64f(swa + 64u * c + 32u * b2);    // columns 16c + 8b2 + 2pq (+1)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t* wv = r + 8 * (i >> 1) + 4 * b2 + 2 * (i & 1);
              const float2 pv = make_float2(__int2float_rn((int)wv[0]), __int2float_rn((int)wv[1]));
              acc[i][2 * c + b2] = __fmul2_rn(__fmul2_rn(sx2[i], sw2), pv);
            }
          }
          if (c + 1 < CW / 16) tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(tm_empty(b));
          mbar_arrive(sc_empty(sc));
        }
        ++tb;
      }
      if (p.n_lr > 0) {
        const int b = tb & 1;
        if (!wait_or_abort(tm_full(b), (tb >> 1) & 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ta = tmem + b * BN + h * CW + lane_off;
        uint32_t rb[2][16];
        tmem_ld16x256b_x2(ta, &rb[0][0]);
        tmem_ld16x256b_x2(ta + (16u << 16), &rb[0][8]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < CW / 16; ++c) {
          if (c + 1 < CW / 16) {
            tmem_ld16x256b_x2(ta + 16 * (c + 1), &rb[(c + 1) & 1][0]);
            tmem_ld16x256b_x2(ta + 16 * (c + 1) + (16u << 16), &rb[(c + 1) & 1][8]);
          }
          const uint32_t* r = rb[c & 1];
#pragma unroll
          for (int b2 = 0; b2 < 2; ++b2)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t* wv = r + 8 * (i >> 1) + 4 * b2 + 2 * (i & 1);
              acc[i][2 * c + b2] = __fadd2_rn(acc[i][2 * c + b2],
                                              make_float2(__uint_as_float(wv[0]), __uint_as_float(wv[1])));
            }
          if (c + 1 < CW / 16) tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tm_empty(b));
        ++tb;
      }
      // epilogue: bias, GELU, bf16, swizzled staging, TMA store
#pragma unroll
      for (int e = 0; e < PER; ++e) bb[lane * PER + e] = bias_n[e];
      if (lane == 0) tma_store_wait_read0();
      __syncwarp();
      const bool gelu = p.epilogue == SVDQ_EPI_GELU;
#pragma unroll
      for (int c = 0; c < CW / 16; ++c) {
#pragma unroll
        for (int b2 = 0; b2 < 2; ++b2) {
          const int col = 16 * c + 8 * b2 + 2 * pq;
          const float2 bv = *reinterpret_cast<const float2*>(bb + col);
          uint8_t* yb = ystage + (c >> 2) * L::Y_BOX + 4 * pq;
          const int ch = (2 * c + b2) & 7;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float2 v = __fadd2_rn(acc[i][2 * c + b2], bv);
            if (gelu) v = make_float2(gelu_f(v.x), gelu_f(v.y));
            const int row = r0 + 8 * i;
            *reinterpret_cast<uint32_t*>(yb + row * 128 + ((ch ^ (row & 7)) * 16)) = bf16x2_bits(v);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int box = 0; box < CW / 64; ++box)
          tma_store_2d(&tm_y, ncol0 + box * 64, m0 + 32 * q, smem_u32(ystage + box * L::Y_BOX));
        tma_store_commit();
      }
      __syncwarp();
    }
    if (lane == 0) tma_store_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_linear_w8a8(const svdq_weights* w, int M, const int8_t* xq, const float* s_x,
                               const uint16_t* Z, uint16_t* Y, int ldy, int epilogue,
                               cudaStream_t st) {
  using L = W8Lay;
  static bool attr[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (!attr[dev]) {
    cudaFuncAttributes fa;
    cudaError_t e0 = cudaFuncGetAttributes(&fa, linear_w8a8_kernel);
    if (e0 != cudaSuccess) return e0;
    if (fa.numRegs < W8_REG_NEED) return cudaErrorInvalidConfiguration;   // split would not fit
    cudaError_t e = cudaFuncSetAttribute(linear_w8a8_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    attr[dev] = true;
  }
  CUtensorMap ta, tb, ty, tz, tl, tsx, tsw;
  const uint64_t sx_pitch = ((uint64_t)M * 4 + 15) / 16 * 16;
  const uint64_t sw_pitch = ((uint64_t)w->N_pad * 4 + 15) / 16 * 16;
  if (!make_map(&ta, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->K, M, w->K, 64, L::BM,
                CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map(&tb, w->d_wq8, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->K, w->N, w->K, 64, L::BN,
                CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map(&ty, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->N, M, (uint64_t)ldy * 2, 64, 32,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tsx, s_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, M, 1, sx_pitch, L::BM, 1,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map(&tsw, w->d_sw8, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w->N, 1, sw_pitch, L::BN, 1,
                CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  tz = ta;
  tl = ta;
  if (w->rank > 0 &&
      (!make_map(&tz, Z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->rank, M, (uint64_t)w->rank * 2, 8,
                 L::BM, CU_TENSOR_MAP_SWIZZLE_NONE) ||
       !make_map(&tl, w->d_L2T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->rank_pad32, w->N,
                 (uint64_t)w->rank_pad32 * 2, 8, L::BN, CU_TENSOR_MAP_SWIZZLE_NONE)))
    return cudaErrorInvalidValue;
  W8Args a{};
  a.s_x = s_x; a.s_w = w->d_sw8; a.bias = w->d_bias;
  a.M = M; a.N = w->N; a.K = w->K; a.G = w->K / 64;
  a.n_lr = (w->rank + 15) / 16;
  a.epilogue = epilogue;
  a.tiles_n = (w->N + L::BN - 1) / L::BN;
  a.num_tiles = ((M + L::BM - 1) / L::BM) * a.tiles_n;
  a.err = w->d_err;
  const int grid = a.num_tiles < num_sms() ? a.num_tiles : num_sms();
  linear_w8a8_kernel<<<grid, W8_THREADS, L::ALLOC, st>>>(ta, tb, ty, tz, tl, tsx, tsw, a);
  return cudaGetLastError();
}

}  // namespace svdq
