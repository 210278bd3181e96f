// NVFP4 product (SVDQuant review section 8: NVFP4 uses groups of 16 with
// FP8 scales; section 9.1), warp-specialised for sm_100a:
//
//   Y = bf16(epi(s_x[m] s_w[n] sum_k (q_x b_x)(q_w b_w) + Z L2 + b))
//
// The tensor cores apply the E4M3 group scales themselves
// (tcgen05.mma.kind::mxf4nvf4.block_scale, 16-element blocks): the packed
// E2M1 codes go from TMA straight into the operand tiles, the group scales
// are copied from shared memory into TMEM with tcgen05.cp, and the fp32 sum
// over all of K stays in one TMEM accumulator.  The low-rank product Z L2
// runs on the tensor cores (kind::f16, bf16 operands) into a separate TMEM
// buffer; the epilogue computes s_x s_w acc + Z L2 + b (and GELU) per output
// and stores Y by TMA.
//
// Persistent CTAs (one per SM), 128 x 128 tiles, static round-robin; 8 warps:
//   warp 0    TMA producer: 256-K stages of A and B (one 128-byte-swizzled
//             box each: 128 rows x 128 B) and the four 512-byte group-scale
//             atoms of A and of B (bulk copies); low-rank slices at tile end;
//   warp 1    TMEM owner and MMA issuer: per stage four tcgen05.cp of each
//             operand's atoms into TMEM and four block-scaled MMAs (K = 64);
//   warps 2-3 idle;
//   warps 4-7 epilogue: warp w owns TMEM lanes 32 (w % 4)..; two 128-column
//             accumulator buffers let tile t+1 accumulate while tile t is
//             drained (the low-rank buffer is single: its stage comes at the
//             end of a tile, after the previous tile's epilogue has read it).
// The operand stream is bound by the L2 -> SM path (about 2700 cycles from
// a stage's copy to its arrival at the measured rate): the widest rows the
// copy engine takes (128 B) and four 36 KB stages in flight, with the
// 256-K stage halving the per-stage round trips of a 128-K one.
// TMEM: accumulators [0, 256), low-rank [256, 384), and one 32-column slot
// of group scales per shared-memory stage [384, 512) (A: 4 columns per K
// block, then B), so the scale copies of a stage never wait for the MMAs of
// an earlier one: a slot is refilled only after its stage's MMAs have
// completed (the stage's empty barrier).
// Every wait is bounded (the handle's error word is raised on expiry).
#include "gemm_common.cuh"

namespace svdq {
namespace {

constexpr int F4_BM = 128, F4_BN = 128;
constexpr int F4_THREADS = 256;
constexpr int F4_EPI0 = 4;         // epilogue warps 4-7

struct F4Args {
  const float* s_x;
  const float* s_w;
  const uint16_t* bias;
  const uint8_t* sfa;      // activation group scales, atom layout
  const uint8_t* sfb;      // weight group scales, atom layout
  int M, N, K;
  int nkb;                 // K blocks of 64
  int n_lr;                // 16-wide low-rank slices
  int epilogue;
  int tiles_n, num_tiles;
  int* err;
};

struct F4Lay {
  static constexpr int BM = F4_BM, BN = F4_BN;
  static constexpr int KB = 4;                                // 64-K blocks per stage
  static constexpr int ST_A = BM * 128, ST_B = BN * 128;     // 256 K of packed FP4
  static constexpr int ST_SFA = KB * 512, ST_SFB = KB * 512;  // one 512-byte atom per K block
  static constexpr int STAGE = ST_A + ST_B + ST_SFA + ST_SFB;
  static constexpr int NST = 4;          // also the TMEM scale slots (4 x 32 columns)
  static constexpr int SF_COLS = 32;
  static constexpr int NLR = 2;
  static constexpr int LR_SA = BM * 32, LR_SB = BN * 32, LR_SLOT = LR_SA + LR_SB;
  static constexpr int Y_BOX = 32 * 64 * 2;                   // 32 rows x 64 bf16
  static constexpr int Y_WARP = 2 * Y_BOX;                    // 128 columns
  static constexpr int OFF_ST = 0;
  static constexpr int OFF_LR = OFF_ST + NST * STAGE;
  static constexpr int OFF_Y = OFF_LR + NLR * LR_SLOT;
  // per epilogue warp: the tile's 128 weight scales, then its 128 biases (fp32)
  static constexpr int OFF_EPS = OFF_Y + 4 * Y_WARP;
  static constexpr int OFF_BAR = OFF_EPS + 4 * 1024;
  // st_full[NST], st_empty[NST], tm_full[2], tm_empty[2], lr_full[NLR], lr_empty[NLR],
  // lrb_empty (low-rank TMEM buffer read by the epilogue)
  static constexpr int N_BARS = 2 * NST + 4 + 2 * NLR + 1;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static_assert(ALLOC <= 227 * 1024, "shared memory");
  static_assert(STAGE % 1024 == 0 && OFF_Y % 1024 == 0, "alignment");
};

// True in one lane of the (converged) calling warp: the issuing lane of
// single-thread tcgen05 instructions in warp-uniform code.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "elect.sync _|P, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}\n"
      : "=r"(pred));
  return pred != 0;
}

constexpr uint32_t TM_LR = 256;                    // low-rank accumulator
constexpr uint32_t TM_SF = 384;                    // group-scale slots, 32 columns per stage

// Instruction descriptor of the block-scaled FP4 MMA: E2M1 A and B (K-major),
// UE4M3 scales, fp32 D, M = 128, N = 128, K = 64, scale ids 0.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10)                 // A, B: E2M1
         | ((uint32_t)(N >> 3) << 17)           // N / 8
         | (0u << 23)                           // scale format UE4M3
         | ((uint32_t)(M >> 4) << 24);          // M / 16
}

// K-major operand as 128-byte rows with the 128-byte swizzle (8-row atoms of
// 1 KB, stride 1 KB); the K block j of a row starts 32 j bytes in, i.e. the
// descriptor's start address advances by 2 (16-byte units).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
      "}\n" ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
      "r"(sfb_tmem));
}

// 32 rows x 128 bits from shared memory (a 512-byte scale atom, 16 bytes per
// row) into TMEM, replicated to the four lane quarters.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint32_t satom) {
  const uint64_t d = sdesc_kmajor_noswizzle(satom, 128, 128);
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d));
}

__global__ void __launch_bounds__(F4_THREADS, 1)
linear_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_y,
                    const __grid_constant__ CUtensorMap tm_z,
                    const __grid_constant__ CUtensorMap tm_l2, const F4Args p) {
  using L = F4Lay;
  constexpr int BM = L::BM, BN = L::BN, NST = L::NST, NLR = L::NLR;
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
  const uint32_t lrb_empty = bar0 + 8u * (2 * NST + 4 + 2 * NLR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int KB = L::KB;
  const int nst = (p.nkb + KB - 1) / KB;      // 256-K stages per tile

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) { mbar_init(st_full(s), 1); mbar_init(st_empty(s), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tm_full(b), 1); mbar_init(tm_empty(b), 4); }
    for (int s = 0; s < NLR; ++s) { mbar_init(lr_full(s), 1); mbar_init(lr_empty(s), 1); }
    mbar_init(lrb_empty, 4);
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

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      uint32_t it = 0, il = 0;
      bool alive = true;
      for (int t = blockIdx.x; t < p.num_tiles && alive; t += gridDim.x) {
        const int mb = t / p.tiles_n, nb = t % p.tiles_n;
        const int m0 = mb * BM, n0 = nb * BN;
        for (int s = 0; s < nst; ++s, ++it) {
          const int st = it % NST;
          if (!wait_or_abort(st_empty(st), ((it / NST) & 1) ^ 1, abort_flag, p.err)) { alive = false; break; }
          // K blocks [kb0, kb0 + nk); the boxes read zeros past the end of K
          const int kb0 = KB * s, nk = p.nkb - kb0 < KB ? p.nkb - kb0 : KB;
          mbar_arrive_expect_tx(st_full(st), L::ST_A + L::ST_B + 2 * nk * 512);
          const uint32_t dst = sbase + L::OFF_ST + st * L::STAGE;
          tma_load_2d(dst, &tm_a, s * 128, m0, st_full(st));
          tma_load_2d(dst + L::ST_A, &tm_b, s * 128, n0, st_full(st));
          bulk_load(dst + L::ST_A + L::ST_B, p.sfa + ((size_t)mb * p.nkb + kb0) * 512, nk * 512,
                    st_full(st));
          bulk_load(dst + L::ST_A + L::ST_B + L::ST_SFA, p.sfb + ((size_t)(n0 / 128) * p.nkb + kb0) * 512,
                    nk * 512, st_full(st));
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
      for (uint32_t k = (it > NST ? it - NST : 0); k < it; ++k)
        mbar_wait_bounded(st_full(k % NST), (k / NST) & 1, LIMIT_NS);
      for (uint32_t k = (il > NLR ? il - NLR : 0); k < il; ++k)
        mbar_wait_bounded(lr_full(k % NLR), (k / NLR) & 1, LIMIT_NS);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    // The whole warp walks the loop with warp-uniform operands (lane 0
    // waits, the result is broadcast); one elected lane issues the tcgen05
    // instructions.  Issuing from a lane-0-only branch cost ~100 cycles per
    // tcgen05 instruction, more than the MMAs themselves.
    const uint32_t id_f4 = idesc_nvf4(BM, BN), id_bf = idesc_bf16(BM, BN);
    const uint32_t tm = __shfl_sync(0xFFFFFFFFu, tmem, 0);
    auto wait_warp = [&](uint32_t bar, uint32_t parity) -> bool {
      int ok = 1;
      if (lane == 0) ok = wait_or_abort(bar, parity, abort_flag, p.err) ? 1 : 0;
      return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
    };
    uint32_t it = 0, tb = 0, il = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++tb) {
      const int b = tb & 1;
      if (!wait_warp(tm_empty(b), ((tb >> 1) & 1) ^ 1)) break;
      const uint32_t d = tm + b * BN;
      bool ok = true;
      for (int s = 0; s < nst; ++s, ++it) {
        const int st = it % NST;
        if (!wait_warp(st_full(st), (it / NST) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = sbase + L::OFF_ST + st * L::STAGE;
        const uint32_t sb = sa + L::ST_A, ssfa = sb + L::ST_B, ssfb = ssfa + L::ST_SFA;
        const int nk = p.nkb - KB * s < KB ? p.nkb - KB * s : KB;
        const uint32_t sf = tm + TM_SF + L::SF_COLS * st;   // A: +4h, B: +16+4h
        if (elect_one()) {
          for (int h = 0; h < nk; ++h) {
            // this K block's scales: 4 TMEM columns per operand
            tmem_cp_sf(sf + 4 * h, ssfa + 512 * h);
            tmem_cp_sf(sf + 4 * KB + 4 * h, ssfb + 512 * h);
          }
          const uint64_t ad = sdesc_sw128(sa), bd = sdesc_sw128(sb);
          for (int h = 0; h < nk; ++h)
            mma_nvf4(d, ad + 2 * h, bd + 2 * h, id_f4, sf + 4 * h, sf + 4 * KB + 4 * h,
                     (s > 0 || h > 0) ? 1u : 0u);
          mma_commit(st_empty(st));
        }
        __syncwarp();
      }
      if (!ok) break;
      // the low-rank buffer: free once the previous tile's epilogue read it
      if (p.n_lr > 0 && !wait_warp(lrb_empty, (tb & 1) ^ 1)) break;
      for (int j = 0; j < p.n_lr; ++j, ++il) {
        const int ls = il % NLR;
        if (!wait_warp(lr_full(ls), (il / NLR) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t la = sbase + L::OFF_LR + ls * L::LR_SLOT;
        if (elect_one()) {
          mma_bf16(tm + TM_LR, sdesc_kmajor_noswizzle(la, BM * 16, 128),
                   sdesc_kmajor_noswizzle(la + L::LR_SA, BN * 16, 128), id_bf, j > 0 ? 1u : 0u);
          mma_commit(lr_empty(ls));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) mma_commit(tm_full(b));
      __syncwarp();
    }
  } else if (warp >= F4_EPI0) {
    // ------------------------------------------------------ epilogue
    // thread = one row of the warp's quarter; 32-column TMEM loads
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    uint8_t* ystage = smem + L::OFF_Y + q * L::Y_WARP;
    // the tile's weight scales and biases, staged once per tile (zeros past N)
    float* eps = reinterpret_cast<float*>(smem + L::OFF_EPS + q * 1024);
    const uint32_t eps_sw = smem_u32(eps), eps_b = eps_sw + 512;
    const bool gelu = p.epilogue == SVDQ_EPI_GELU;
    uint32_t tb = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++tb) {
      const int m0 = (t / p.tiles_n) * BM, n0 = (t % p.tiles_n) * BN;
      const int row = m0 + 32 * q + lane;
      const float sx = row < p.M ? __ldg(p.s_x + row) : 0.0f;
      // columns n0 + 4 lane .. + 3, loaded before the accumulator is ready
      const int nl = n0 + 4 * lane;
      float4 w4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f), b4 = w4;
      if (nl + 3 < p.N) {
        w4 = __ldg(reinterpret_cast<const float4*>(p.s_w + nl));
        const uint2 bb = __ldg(reinterpret_cast<const uint2*>(p.bias + nl));
        b4 = make_float4(__uint_as_float(bb.x << 16), __uint_as_float(bb.x & 0xFFFF0000u),
                         __uint_as_float(bb.y << 16), __uint_as_float(bb.y & 0xFFFF0000u));
      } else {
        float* wv = &w4.x;
        float* bv = &b4.x;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (nl + e < p.N) {
            wv[e] = __ldg(p.s_w + nl + e);
            bv[e] = __uint_as_float((uint32_t)__ldg(p.bias + nl + e) << 16);
          }
      }
      const int b = tb & 1;
      if (!wait_or_abort(tm_full(b), (tb >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      if (lane == 0) tma_store_wait_read0();
      reinterpret_cast<float4*>(eps)[lane] = w4;
      reinterpret_cast<float4*>(eps + 128)[lane] = b4;
      __syncwarp();
      const bool lr = p.n_lr > 0;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32], z[32];
        tmem_ld32(tmem + b * BN + 32 * c + lane_off, r);
        if (lr) tmem_ld32(tmem + TM_LR + 32 * c + lane_off, z);
        tmem_wait_ld();
        uint32_t packed[16];
        float4 sw4, bs4;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          if ((j & 3) == 0) {
            sw4 = lds128(eps_sw + 4u * (32 * c + j));     // same address in every lane
            bs4 = lds128(eps_b + 4u * (32 * c + j));
          }
          const float w0 = (j & 2) ? sw4.z : sw4.x, w1 = (j & 2) ? sw4.w : sw4.y;
          float b0 = (j & 2) ? bs4.z : bs4.x, b1 = (j & 2) ? bs4.w : bs4.y;
          if (lr) {
            b0 = __fadd_rn(__uint_as_float(z[j]), b0);
            b1 = __fadd_rn(__uint_as_float(z[j + 1]), b1);
          }
          float2 v = make_float2(__fmaf_rn(__fmul_rn(sx, w0), __uint_as_float(r[j]), b0),
                                 __fmaf_rn(__fmul_rn(sx, w1), __uint_as_float(r[j + 1]), b1));
          if (gelu) v = make_float2(gelu_f(v.x), gelu_f(v.y));
          packed[j >> 1] = bf16x2_bits(v);
        }
        // row `lane` of box c / 2: 64 bytes at 16-byte chunk (4 (c & 1) + u) ^ (lane & 7)
        uint8_t* yb = ystage + (c >> 1) * L::Y_BOX + lane * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint4*>(yb + ((((c & 1) * 4 + u) ^ (lane & 7)) << 4)) =
              make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(tm_empty(b));
        if (lr) mbar_arrive(lrb_empty);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int box = 0; box < 2; ++box)
          tma_store_2d(&tm_y, n0 + 64 * box, m0 + 32 * q, smem_u32(ystage + box * L::Y_BOX));
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

cudaError_t launch_linear_nvfp4(const svdq_weights* w, int M, const uint8_t* xq,
                                const uint8_t* sfa, const float* s_x, const uint16_t* Z,
                                uint16_t* Y, int ldy, int epilogue, cudaStream_t st) {
  using L = F4Lay;
  static bool attr[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (!attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(linear_nvfp4_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    attr[dev] = true;
  }
  CUtensorMap ta, tb, ty, tz, tl;
  if (!make_map(&ta, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->K / 2, M, w->K / 2, 128, L::BM,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tb, w->d_wq4, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->K / 2, w->N, w->K / 2, 128, L::BN,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&ty, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->N, M, (uint64_t)ldy * 2, 64, 32,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  tz = ta;
  tl = ta;
  if (w->rank > 0 &&
      (!make_map(&tz, Z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->rank, M, (uint64_t)w->rank * 2, 8,
                 L::BM, CU_TENSOR_MAP_SWIZZLE_NONE) ||
       !make_map(&tl, w->d_L2T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->rank_pad32, w->N,
                 (uint64_t)w->rank_pad32 * 2, 8, L::BN, CU_TENSOR_MAP_SWIZZLE_NONE)))
    return cudaErrorInvalidValue;
  F4Args a{};
  a.s_x = s_x; a.s_w = w->d_sw4; a.bias = w->d_bias; a.sfa = sfa; a.sfb = w->d_sfb4;
  a.M = M; a.N = w->N; a.K = w->K; a.nkb = w->K / 64;
  a.n_lr = (w->rank + 15) / 16;
  a.epilogue = epilogue;
  a.tiles_n = (w->N + L::BN - 1) / L::BN;
  a.num_tiles = ((M + L::BM - 1) / L::BM) * a.tiles_n;
  a.err = w->d_err;
  const int grid = a.num_tiles < num_sms() ? a.num_tiles : num_sms();
  linear_nvfp4_kernel<<<grid, F4_THREADS, L::ALLOC, st>>>(ta, tb, ty, tz, tl, a);
  return cudaGetLastError();
}

}  // namespace svdq
