// W4A4 product with the 16-bit up-projection fused (SVDQuant review section
// 6.1, product side; eq. 7), warp-specialised for sm_100a.
//
// sm_100a tensor cores have no 4-bit integer kind, so the packed codes are
// streamed by TMA into shared memory and expanded there to one byte per code
// for tcgen05.mma.kind::f8f6f4 with E4M3 operands: a code q becomes the E4M3
// number q * 2^-9, i.e. the byte sign << 7 | |q| (|q| <= 7 are the format's
// subnormals m * 2^-9; |q| = 8 is its smallest normal 2^-6, bit pattern 0x08
// again).  Every product is then an integer times 2^-18 and every sum of a
// group of 64 is P_g 2^-18 with |P_g| <= 4096, so the fp32 TMEM accumulator
// holds each group's integer partial exactly and needs no conversion.  The
// weight codes are stored on the device as sign-magnitude nibbles (a layer
// with a code of -8, which only a subnormal scale can produce, keeps two's
// complement and the longer conversion).  The activation codes arrive as
// two's-complement nibbles (the public layout) and are expanded as u = q + 8
// (the nibble with its top bit flipped, whose byte is exactly the E4M3
// number u 2^-9: 0..7 subnormal, 8..15 the first binade), so that group's
// MMAs sum P_g + 8 S_g with S_g = sum_k q_w.  A third MMA per group (K = 32)
// adds the constant A slice (2^-6, 2^-3, 1, 0, ..) times the E4M3 digits
// (d0, d1, d2, 0, ..) of -S_g = d0 + 8 d1 + 64 d2 (from the pack), i.e.
// -8 S_g 2^-18, so the TMEM word is again exactly P_g 2^-18.  The device copy of the weight
// scales holds s_w 2^18 (exact), so the rescale is plain fp32 arithmetic, two
// operations per element and group: v = fl32(P_g s_w), acc = fl32(acc +
// v s_x).  The low-rank term Z L2 is one more tensor-core stage (kind::f16,
// bf16 operands, fp32 in TMEM) added unscaled; then the bias (and GELU) are
// applied and Y is written once, as bf16, by TMA.
//
// The same kernel can instead hand its output to the next layer (MODE 4,
// the cross-layer fusion): the epilogue quantises the bf16 tile with the
// next layer's smoothing factors into that layer's codes and scales, and
// one more tensor-core stage multiplies it with the next layer's L1 rows
// for a per-tile partial of that layer's down-projection.
//
// Persistent CTAs (one per SM, 128 x BN output tiles, static round-robin
// schedule); 16 warps:
//   warp 0      TMA producer: packed A (128 rows x 64 B) and B (BN x 64 B)
//               of two groups per stage, one 64-byte-swizzled box per
//               operand, into a 2-stage ring (narrow boxes would make the
//               copy engine's per-row rate the limit), and the bf16 Z / L2
//               slices of the low-rank stage (loaded straight into UMMA
//               layout);
//   warp 1      TMEM owner and MMA issuer (one thread);
//   warps 2-7   expanders: packed nibbles -> E4M3 bytes in the UMMA
//               K-major layout (2-stage ring);
//   warps 8-15  rescale + epilogue: warp w owns TMEM lanes 32 (w % 4).. and
//               BN/2 columns; double-buffered TMEM lets group g+1 run on
//               the tensor cores while group g is rescaled.
// The first two warpgroups hand registers to the last two (setmaxnreg).
// Every wait is bounded: an expired wait raises the handle's error word and
// the CTA drains and exits instead of hanging.
//
// Expanded operand layout (no swizzle): a 64-byte K row of a group is four
// 16-byte core-matrix rows; core matrix (row r/8, chunk c) is stored at
// (r/8)*512 + c*128, row r%8 at +16*(r%8).  Inside every 8 codes the
// expansion places the even-k codes before the odd-k codes; A and B use the
// same order, so each group's dot product is unchanged.  The low-rank
// slices use the other legal arrangement of the same core matrices, chunk c
// at c*rows*16 and row r at r*16, which a 16-byte-wide TMA box produces.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "gemm_common.cuh"
#include "ptx.cuh"
#include "quant_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 128;
constexpr int NP = 2;            // packed-code stages (two groups each)
constexpr int THREADS = 512;
constexpr int N_EXP = 192;       // expanders: warps 2-7
constexpr int RES_WARP0 = 8;     // rescale / epilogue: warps 8-15
constexpr int N_RES_WARPS = 8;
constexpr float P_SCALE = 262144.0f;           // 2^18: a group's TMEM word times this is P_g
// Register split after launch: the first two warpgroups (producer, MMA,
// expanders) give registers to the two rescale warpgroups.
// 256 * REG_LO + 256 * REG_HI
// must not exceed the launch allotment (THREADS x the kernel's register
// count); the launcher checks the compiled count before every launch.
constexpr int REG_LO = 56;
constexpr int REG_HI = 200;
constexpr int RCH = 2;           // 16-column TMEM chunks per rescale load batch
constexpr int REG_NEED = (256 * REG_LO + 256 * REG_HI + THREADS - 1) / THREADS;

struct LinArgs {
  const float* s_x;
  const float* s_w;
  const uint16_t* Z;
  const uint16_t* L2T;     // [N_pad][rank_pad32]
  const uint16_t* bias;
  int M, N, K, G;
  int rank, rank_pad32, n_lr;   // n_lr: 16-wide low-rank slices, ceil(rank / 16)
  int epilogue;
  int tiles_n, num_tiles, tile_m0, tile_n0;
  int* err;
  uint64_t limit_ns;       // bound on every wait (LIMIT_NS; shorter in the stall test)
  int stall;               // test hook: CTA 0's producer withholds its first stage
  int b_twos;              // 1: weight codes in two's complement (else sign-magnitude)
  int sx_tma;              // 1: s_x rows are 16-byte aligned (M % 4 == 0), copy by TMA
  int32_t* P;              // partial dump (MODE 1)
  int row0, nrows, col0, ncols;
  int splits;              // K splits per tile (1 except in MODE 3)
  float* part;             // MODE 3: fp32 partial tiles [tile][split][warp][32 x CW]
  int* cnt;                // MODE 3: arrivals per (tile, rescale warp), zero between uses
  // MODE 4: the next layer's activation side from this layer's output
  const float* inv_lambda2;  // [N]: the next layer's smoothing factors (its K = this N)
  uint8_t* xq2;              // [M][N / 2] packed codes
  float* s_x2;               // [N / 64][M] group scales
  float* zpart;              // [tiles_n][M][rank2] fp32 down-projection of each column tile
  int rank2, rank2_pad;      // the next layer's rank, and rounded up to 16
  int n_l1;                  // 128-column L1^T parts per tile (0 without a low-rank branch)
};

// One unit of work: output tile t, groups [g0, g1) of split sp.  The
// low-rank stage belongs to split 0.
struct WorkItem {
  int t, sp, g0, g1;
  bool lr;
};
__device__ __forceinline__ WorkItem work_item(const LinArgs& p, int wk) {
  WorkItem w;
  w.t = wk / p.splits;
  w.sp = wk - w.t * p.splits;
  w.g0 = (int)((long long)w.sp * p.G / p.splits);
  w.g1 = (int)((long long)(w.sp + 1) * p.G / p.splits);
  w.lr = w.sp == 0;
  return w;
}

template <int BN>
struct Lay {
  static constexpr int NB = 512 / BN;                    // TMEM accumulator buffers
  static constexpr int NE = BN == 256 ? 2 : 4;           // expanded-operand stages
  static constexpr int CW = BN / 2;                      // columns per rescale warp
  static constexpr int Y_BOX = 32 * 64 * 2;              // 32 rows x 64 bf16 (4 KB)
  static constexpr int Y_WARP = (CW / 64) * Y_BOX;
  // packed stage: 64-byte rows (two groups), 64-byte swizzle: chunk c of
  // row r at r * 64 + 16 (c ^ ((r >> 1) & 3)); chunk 2 gs + hf is half hf
  // of group gs of the stage
  static constexpr int PK_A = BM * 64, PK_B = BN * 64, PK_STAGE = PK_A + PK_B;
  // expanded stage: A and B of one group, then the correction slice of B: one
  // 16-byte row per column (digit bytes 0..3, the rest zero), read for both
  // K halves of the K = 32 MMA (leading offset 0)
  static constexpr int EX_A = BM * 64, EX_B = BN * 64, EX_X = BN * 16;
  static constexpr int EX_STAGE = EX_A + EX_B + EX_X;
  // the constant A slice of the correction MMA: 128 rows x 32 B (two 16-byte
  // chunks), bytes 0..2 of each row 2^-6, 2^-3, 1, the rest zero
  static constexpr int AX_BYTES = BM * 32;
  static constexpr int OFF_Y = 0;
  static constexpr int OFF_PK = OFF_Y + N_RES_WARPS * Y_WARP;
  static constexpr int OFF_EX = OFF_PK + NP * PK_STAGE;
  // low-rank stage: NLR slots of one 16-wide K slice each (2 chunks x rows x
  // 16 B of Z and of L2^T), so that slices load while earlier ones multiply
  // (four slots where shared memory allows: rank 64 in flight at once)
  static constexpr int NLR = BN == 256 ? 2 : 4;
  static constexpr int LR_SA = BM * 32, LR_SB = BN * 32, LR_SLOT = LR_SA + LR_SB;
  static constexpr int OFF_AX = OFF_EX + NE * EX_STAGE;
  static constexpr int OFF_LR = OFF_AX + AX_BYTES;
  // per-group scales: ring of 2 NP + NE + NB slots, each s_x[128], s_w[BN]
  // and the correction digits [BN] (one word per column), filled by the
  // producer warp together with the packed codes.  The
  // producer writes the slots of groups j, j + 1 (stage k) once the expanders
  // released stage k - NP, i.e. expanded every group up to j - 2 NP + 1;
  // through the MMA and TMEM barriers the rescale of group j + 1 - 2 NP - NE
  // - NB, the previous owner of the last slot written, has then finished.
  static constexpr int NS = 2 * NP + NE + NB;
  static constexpr int SC_SLOT = (BM + 2 * BN) * 4;
  static constexpr int OFF_SC = OFF_LR + NLR * LR_SLOT;
  static constexpr int OFF_BIAS = OFF_SC + NS * SC_SLOT;   // per warp CW floats
  // MODE 4: the next layer's smoothing factors of the warp's columns
  static constexpr int OFF_ILAM = OFF_BIAS + N_RES_WARPS * CW * 4;
  static constexpr int OFF_BAR = OFF_ILAM + N_RES_WARPS * CW * 4;
  // barriers: pk_full[NP], pk_empty[NP], ex_full[NE], ex_empty[NE], tm_full[NB],
  // tm_empty[NB], lr_full[NLR], lr_empty[NLR], xh_full, mma_drain
  static constexpr int N_BARS = 2 * NP + 2 * NE + 2 * NB + 2 * NLR + 2;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;              // slack for 1024-B alignment
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};


// The quantiser of MODE 4's epilogue runs in a runtime loop, one row and
// group per iteration, so that its code exists once: unrolled over the
// thread's eight rows and groups, that straight-line code, run once per
// tile, measured slower (instruction fetch).  The switch copies the values
// one iteration needs into a8, which keeps every source value at a static
// register index.
// a8[k] = src[i][8 j + k] for sel = 4 j + i: row i's pairs of 64-column group j.
template <typename T, int NP2>
__device__ __forceinline__ void row_group(const T (&src)[4][NP2], int sel, T (&a8)[8]) {
#define SVDQ_RG(S)                                                               \
  case S:                                                                        \
    if constexpr (8 * ((S) / 4) + 7 < NP2) {                                     \
      _Pragma("unroll") for (int k = 0; k < 8; ++k) a8[k] = src[(S) % 4][8 * ((S) / 4) + k]; \
    }                                                                            \
    break;
  switch (sel) {
    SVDQ_RG(0) SVDQ_RG(1) SVDQ_RG(2) SVDQ_RG(3) SVDQ_RG(4) SVDQ_RG(5) SVDQ_RG(6) SVDQ_RG(7)
    default: break;
  }
#undef SVDQ_RG
}

__device__ __forceinline__ void sts32u(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t lds32u(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// Codes -> E4M3 bytes, four at a time (one byte each of a 32-bit word).
// Two's complement: x holds four nibbles 0..15, y the same nibbles in the
// high half of each byte (bit 7 = the code's sign).  A negative code q = x - 16
// becomes (x ^ 0x8F) + 1 = 0x80 | (16 - x) = 0x80 | |q|, with no carry out of
// its byte (|q| <= 8); the sign masks come from one byte permute in
// sign-replicating mode.
__device__ __forceinline__ uint32_t e4m3_twos(uint32_t x, uint32_t y) {
  uint32_t m;
  asm("prmt.b32 %0, %1, 0, 0xBA98;" : "=r"(m) : "r"(y));
  return (x ^ (m & 0x8F8F8F8Fu)) + (m & 0x01010101u);
}
// The low (even-k) and high (odd-k) nibbles of four packed bytes.
template <bool TWOS>
__device__ __forceinline__ uint32_t e4m3_lo(uint32_t w) {
  if (TWOS) return e4m3_twos(w & 0x0F0F0F0Fu, w << 4);
  return (w & 0x07070707u) | ((w << 4) & 0x80808080u);     // sign-magnitude: s << 7 | m
}
template <bool TWOS>
__device__ __forceinline__ uint32_t e4m3_hi(uint32_t w) {
  if (TWOS) return e4m3_twos((w >> 4) & 0x0F0F0F0Fu, w);
  return ((w >> 4) & 0x07070707u) | (w & 0x80808080u);
}
// Activation codes as offset binary: the nibble with its top bit flipped is
// u = q + 8 in 0..15, and the byte u is exactly the E4M3 number u 2^-9.
__device__ __forceinline__ uint32_t e4m3_off_lo(uint32_t w) { return (w ^ 0x88888888u) & 0x0F0F0F0Fu; }
__device__ __forceinline__ uint32_t e4m3_off_hi(uint32_t w) { return ((w ^ 0x88888888u) >> 4) & 0x0F0F0F0Fu; }
__device__ __forceinline__ void expand_offset(uint32_t src, uint32_t d) {
  const uint4 p = lds128u(src);
  sts128(d, make_uint4(e4m3_off_lo(p.x), e4m3_off_hi(p.x), e4m3_off_lo(p.y), e4m3_off_hi(p.y)));
  sts128(d + 128, make_uint4(e4m3_off_lo(p.z), e4m3_off_hi(p.z), e4m3_off_lo(p.w), e4m3_off_hi(p.w)));
}

// 16 packed bytes (32 codes of one row: the first or second half of the
// group) -> two 16-byte core-matrix rows at d and d + 128.  Inside every 8
// codes the even-k codes come first.
template <bool TWOS>
__device__ __forceinline__ void expand_e4m3(uint32_t src, uint32_t d) {
  const uint4 p = lds128u(src);
  uint4 o0, o1;
  o0.x = e4m3_lo<TWOS>(p.x);
  o0.y = e4m3_hi<TWOS>(p.x);
  o0.z = e4m3_lo<TWOS>(p.y);
  o0.w = e4m3_hi<TWOS>(p.y);
  o1.x = e4m3_lo<TWOS>(p.z);
  o1.y = e4m3_hi<TWOS>(p.z);
  o1.z = e4m3_lo<TWOS>(p.w);
  o1.w = e4m3_hi<TWOS>(p.w);
  sts128(d, o0);
  sts128(d + 128, o1);
}

// The expanders' share of one group: NA rounds of 32 consecutive 16-byte
// units of A (activation codes) from round A0 and NB rounds of B (weight
// codes) from round B0 of that operand.  Unit j of an operand is half
// (j >> 3) & 1 of row 8 (j >> 4) + (j & 7), so each quarter-warp reads one
// half of eight consecutive rows (eight distinct 16-byte bank groups under
// the 64-byte swizzle) and writes 128 contiguous bytes.  Offsets are fixed
// per thread and computed once.
template <int BN, int NA, int NB>
struct ExpandPlan {
  static constexpr int CNT = NA + NB;
  uint32_t src[CNT], dst[CNT];
  __device__ __forceinline__ ExpandPlan(int a0, int b0, int lane) {
    using L = Lay<BN>;
#pragma unroll
    for (int k = 0; k < CNT; ++k) {
      const bool isa = k < NA;
      const int j = 32 * (isa ? a0 + k : b0 + k - NA) + lane;
      const int hf = (j >> 3) & 1, row = ((j >> 4) << 3) | (j & 7);
      // group 0 of the stage; group 1 is chunk + 2, i.e. the offset ^ 32
      src[k] = (isa ? 0 : L::PK_A) + row * 64 + ((hf ^ ((row >> 1) & 3)) << 4);
      dst[k] = (isa ? 0 : L::EX_A) + (row >> 3) * 512 + (row & 7) * 16 + hf * 256;
    }
  }
  // gsx = 32 * (group within the packed stage); activation codes become
  // offset binary, weight codes sign-magnitude (two's complement when BTWOS)
  template <bool BTWOS>
  __device__ __forceinline__ void run(uint32_t pa, uint32_t ea, uint32_t gsx) const {
#pragma unroll
    for (int k = 0; k < CNT; ++k) {
      if (k < NA) expand_offset(pa + (src[k] ^ gsx), ea + dst[k]);
      else if (BTWOS) expand_e4m3<true>(pa + (src[k] ^ gsx), ea + dst[k]);
      else expand_e4m3<false>(pa + (src[k] ^ gsx), ea + dst[k]);
    }
  }
};


// MODE 0: the layer (rescale, low-rank stage, epilogue, TMA store of Y).
// MODE 1: dump the int32 group partials of the tiles covering the requested
//         block instead of rescaling them (test hook).
// MODE 3: the layer with the K groups of each tile split over p.splits work
//         items; each writes its fp32 partial to p.part, and the last of a
//         tile's splits (per rescale warp, by an atomic count) sums them in
//         split order and runs the epilogue.
// MODE 4: the layer, followed in the epilogue by the next layer's activation
//         side instead of the store of Y: the bf16 output tile is smoothed
//         with the next layer's factors, quantised per token and group of 64
//         (a tile holds whole groups) into packed codes and scales, and
//         multiplied on the tensor cores, as bf16, with the matching rows of
//         the next layer's L1; each tile stores its fp32 partial
//         down-projection in p.zpart, summed in column-tile order by a
//         second kernel.
template <int BN, int MODE>
__global__ void __launch_bounds__(THREADS, 1)
linear_ws_kernel(const __grid_constant__ CUtensorMap tm_a,
                 const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_y,
                 const __grid_constant__ CUtensorMap tm_z,
                 const __grid_constant__ CUtensorMap tm_l2,
                 const __grid_constant__ CUtensorMap tm_sx,
                 const __grid_constant__ CUtensorMap tm_sw,
                 const __grid_constant__ CUtensorMap tm_l1,
                 const __grid_constant__ CUtensorMap tm_cs, const LinArgs p) {
  using L = Lay<BN>;
  constexpr bool LAYER = MODE != 1;
  constexpr bool SPLIT = MODE == 3;
  constexpr bool FUSE = MODE == 4;
  constexpr int CW = L::CW;
  constexpr int NE = L::NE;
  constexpr int NB = L::NB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::OFF_BAR;
  auto pk_full = [&](int s) { return bar0 + 8u * s; };
  auto pk_empty = [&](int s) { return bar0 + 8u * (NP + s); };
  auto ex_full = [&](int s) { return bar0 + 8u * (2 * NP + s); };
  auto ex_empty = [&](int s) { return bar0 + 8u * (2 * NP + NE + s); };
  auto tm_full = [&](int b) { return bar0 + 8u * (2 * NP + 2 * NE + b); };
  auto tm_empty = [&](int b) { return bar0 + 8u * (2 * NP + 2 * NE + NB + b); };
  constexpr int NLR = L::NLR;
  auto lr_full = [&](int s) { return bar0 + 8u * (2 * NP + 2 * NE + 2 * NB + s); };
  auto lr_empty = [&](int s) { return bar0 + 8u * (2 * NP + 2 * NE + 2 * NB + NLR + s); };
  const uint32_t xh_full = bar0 + 8u * (2 * NP + 2 * NE + 2 * NB + 2 * NLR);
  const uint32_t mma_drain = xh_full + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < NP; ++s) { mbar_init(pk_full(s), 1); mbar_init(pk_empty(s), N_EXP); }
    for (int s = 0; s < NE; ++s) { mbar_init(ex_full(s), N_EXP); mbar_init(ex_empty(s), 1); }
    for (int b = 0; b < NB; ++b) { mbar_init(tm_full(b), 1); mbar_init(tm_empty(b), N_RES_WARPS); }
    for (int s = 0; s < NLR; ++s) { mbar_init(lr_full(s), 1); mbar_init(lr_empty(s), 1); }
    mbar_init(xh_full, N_RES_WARPS);
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  // the correction MMA's constant A slice (core matrix (r / 8, c) at
  // (r / 8) 256 + c 128, row r % 8 at 16 (r % 8)) and the zero bytes of the
  // B slices; both are read by the tensor core (async proxy)
  for (int i = tid; i < L::AX_BYTES / 16; i += THREADS) {
    const bool first = ((i >> 3) & 1) == 0;         // chunk 0 of its core matrix
    sts128(sbase + L::OFF_AX + 16u * i, make_uint4(first ? 0x00382008u : 0u, 0u, 0u, 0u));
  }
  for (int se = 0; se < NE; ++se)
    for (int i = tid; i < L::EX_X / 16; i += THREADS)
      sts128(sbase + L::OFF_EX + se * L::EX_STAGE + L::EX_A + L::EX_B + 16u * i, make_uint4(0u, 0u, 0u, 0u));
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < RES_WARP0) {
    regs_dec<REG_LO>();
    if (warp == 0) {
      // ---------------------------------------------------- TMA producer
      uint32_t it = 0, ig = 0, il = 0;     // packed stages, groups, low-rank slices
      bool alive = true;
      for (int wk = blockIdx.x; wk < p.num_tiles * p.splits && alive; wk += gridDim.x) {
        const WorkItem wi = work_item(p, wk);
        const int t = wi.t;
        const int m0 = (p.tile_m0 + t / p.tiles_n) * BM;
        const int n0 = (p.tile_n0 + t % p.tiles_n) * BN;
        for (int g = wi.g0; g < wi.g1; g += 2, ++it) {
          const int ng = wi.g1 - g < 2 ? 1 : 2;     // groups in this stage
          const int s = it % NP;
          if (!wait_or_abort(pk_empty(s), ((it / NP) & 1) ^ 1, abort_flag, p.err, p.limit_ns)) { alive = false; break; }
          if (p.stall && it == 0 && blockIdx.x == 0) {
            // test hook: the first stage is never filled, so its consumers'
            // bounded waits run out (nothing is issued for it)
            ig += ng;
            __syncwarp();
            continue;
          }
          if (LAYER && !p.sx_tma) {
            // s_x rows not 16-byte aligned: 4-byte async copies by all lanes,
            // tracked by the stage's full barrier (raised before lane 0 arrives)
            for (int k = 0; k < ng; ++k) {
              const uint32_t slot = sbase + L::OFF_SC + ((ig + k) % L::NS) * L::SC_SLOT;
#pragma unroll 4
              for (int i = lane; i < BM; i += 32) {
                const int row = m0 + i;
                const bool in = row < p.M;
                cp_async4(slot + 4 * i, p.s_x + (in ? (size_t)(g + k) * p.M + row : 0), in ? 4u : 0u);
              }
            }
            cp_async_mbar_arrive(pk_full(s));
            __syncwarp();
          }
          if (lane == 0) {
            // scales (the layer only) and the correction digits (every mode)
            const uint32_t scale_bytes =
                ng * ((LAYER ? (p.sx_tma ? BM * 4 : 0) + BN * 4 : 0) + BN * 4);
            mbar_arrive_expect_tx(pk_full(s), L::PK_STAGE + scale_bytes);
            const uint32_t dst = sbase + L::OFF_PK + s * L::PK_STAGE;
            // one box per operand: packed bytes [32 g, 32 g + 64); a group
            // past the end of K reads as zeros and is not used
            tma_load_2d(dst, &tm_a, g * 32, m0, pk_full(s));
            tma_load_2d(dst + L::PK_A, &tm_b, g * 32, n0, pk_full(s));
            for (int k = 0; k < ng; ++k) {
              const uint32_t slot = sbase + L::OFF_SC + ((ig + k) % L::NS) * L::SC_SLOT;
              if (LAYER) {
                if (p.sx_tma) tma_load_2d(slot, &tm_sx, m0, g + k, pk_full(s));
                tma_load_2d(slot + 4 * BM, &tm_sw, n0, g + k, pk_full(s));
              }
              tma_load_2d(slot + 4 * (BM + BN), &tm_cs, n0, g + k, pk_full(s));
            }
          }
          ig += ng;
          __syncwarp();
        }
        if (!alive) break;
        if (lane == 0) {
          for (int j = 0; j < (wi.lr ? p.n_lr : 0); ++j, ++il) {
            const int ls = il % NLR;
            if (!wait_or_abort(lr_empty(ls), ((il / NLR) & 1) ^ 1, abort_flag, p.err, p.limit_ns)) { alive = false; break; }
            mbar_arrive_expect_tx(lr_full(ls), L::LR_SLOT);
            const uint32_t dst = sbase + L::OFF_LR + ls * L::LR_SLOT;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              tma_load_2d(dst + c * (BM * 16), &tm_z, 16 * j + 8 * c, m0, lr_full(ls));
              tma_load_2d(dst + L::LR_SA + c * (BN * 16), &tm_l2, 16 * j + 8 * c, n0, lr_full(ls));
            }
          }
          // MODE 4: the next layer's L1^T rows of this tile's columns, in
          // 128-column parts through the same slots (rank2_pad rows x 256 B
          // each, chunk c of 8 columns at c * rank2_pad * 16, row r at r * 16)
          for (int u = 0; FUSE && alive && u < p.n_l1; ++u, ++il) {
            const int ls = il % NLR;
            if (!wait_or_abort(lr_empty(ls), ((il / NLR) & 1) ^ 1, abort_flag, p.err, p.limit_ns)) { alive = false; break; }
            mbar_arrive_expect_tx(lr_full(ls), (uint32_t)p.rank2_pad * 256u);
            const uint32_t dst = sbase + L::OFF_LR + ls * L::LR_SLOT;
#pragma unroll 4
            for (int c = 0; c < 16; ++c)
              tma_load_2d(dst + c * (p.rank2_pad * 16), &tm_l1, n0 + 128 * u + 8 * c, 0, lr_full(ls));
          }
        }
        alive = __shfl_sync(0xFFFFFFFFu, alive ? 1 : 0, 0) != 0;
      }
      // every issued copy has landed before the CTA exits
      if (lane == 0) {
        for (uint32_t k = (it > NP ? it - NP : 0); k < it; ++k)
          if (!(p.stall && k == 0 && blockIdx.x == 0))     // the withheld stage issued nothing
            mbar_wait_bounded(pk_full(k % NP), (k / NP) & 1, p.limit_ns);
        for (uint32_t k = (il > NLR ? il - NLR : 0); k < il; ++k)
          mbar_wait_bounded(lr_full(k % NLR), (k / NLR) & 1, p.limit_ns);
      }
      cp_async_wait<0>();
      __syncwarp();
    } else if (warp == 1) {
      // ---------------------------------------------------- MMA issuer
      if (lane == 0) {
        const uint32_t id_f8 = idesc_e4m3(BM, BN), id_bf = idesc_bf16(BM, BN);
        const uint64_t ax_desc = sdesc_kmajor_noswizzle(sbase + L::OFF_AX, 128, 256);
        uint32_t ite = 0, tb = 0, il = 0, ixh = 0;
        for (int wk = blockIdx.x; wk < p.num_tiles * p.splits; wk += gridDim.x) {
          const WorkItem wi = work_item(p, wk);
          const bool lrs = wi.lr && p.n_lr > 0;
          for (int g = wi.g0; g < wi.g1 + (lrs ? 1 : 0); ++g) {
            const int b = tb % NB;
            if (!wait_or_abort(tm_empty(b), ((tb / NB) & 1) ^ 1, abort_flag, p.err, p.limit_ns)) goto mma_done;
            const uint32_t d = tmem + b * BN;
            if (g < wi.g1) {
              const int s = ite % NE;
              if (!wait_or_abort(ex_full(s), (ite / NE) & 1, abort_flag, p.err, p.limit_ns)) goto mma_done;
              tc_fence_after();
              const uint32_t ea = sbase + L::OFF_EX + s * L::EX_STAGE;
              const uint64_t ad = sdesc_kmajor_noswizzle(ea, 128, 512);
              const uint64_t bd = sdesc_kmajor_noswizzle(ea + L::EX_A, 128, 512);
              mma_f8f6f4(d, ad, bd, id_f8, 0u);          // D = (P_g + 8 S_g) 2^-18, K = 0..31
              mma_f8f6f4(d, ad + 16, bd + 16, id_f8, 1u);  // K = 32..63
              // - 8 S_g 2^-18: the constant slice times the digits
              mma_f8f6f4(d, ax_desc, sdesc_kmajor_noswizzle(ea + L::EX_A + L::EX_B, 0, 128), id_f8, 1u);
              mma_commit(ex_empty(s));
              ++ite;
            } else {
              for (int j = 0; j < p.n_lr; ++j, ++il) {
                const int ls = il % NLR;
                if (!wait_or_abort(lr_full(ls), (il / NLR) & 1, abort_flag, p.err, p.limit_ns)) goto mma_done;
                tc_fence_after();
                const uint32_t la = sbase + L::OFF_LR + ls * L::LR_SLOT;
                // chunk c of the slice at c * rows * 16 bytes, row r at r * 16
                const uint64_t ad = sdesc_kmajor_noswizzle(la, BM * 16, 128);
                const uint64_t bd = sdesc_kmajor_noswizzle(la + L::LR_SA, BN * 16, 128);
                mma_bf16(d, ad, bd, id_bf, j > 0 ? 1u : 0u);
                mma_commit(lr_empty(ls));
              }
            }
            mma_commit(tm_full(b));
            ++tb;
          }
          if (FUSE && p.n_l1 > 0) {
            // the next layer's down-projection of this tile: x~ (bf16, written
            // by the epilogue) times its L1 rows, into the next TMEM buffer
            const int b = tb % NB;
            if (!wait_or_abort(tm_empty(b), ((tb / NB) & 1) ^ 1, abort_flag, p.err, p.limit_ns)) goto mma_done;
            if (!wait_or_abort(xh_full, ixh & 1, abort_flag, p.err, p.limit_ns)) goto mma_done;
            tc_fence_after();
            const uint32_t d = tmem + b * BN;
            const uint32_t id_z = idesc_bf16(BM, p.rank2_pad);
            for (int u = 0; u < p.n_l1; ++u, ++il) {
              const int ls = il % NLR;
              if (!wait_or_abort(lr_full(ls), (il / NLR) & 1, abort_flag, p.err, p.limit_ns)) goto mma_done;
              tc_fence_after();
              const uint32_t la = sbase + L::OFF_LR + ls * L::LR_SLOT;
              for (int j = 0; j < 8; ++j) {
                // A: chunk kc of x~ at kc * BM * 16 bytes, row r at r * 16
                const uint64_t ad = sdesc_kmajor_noswizzle(
                    sbase + L::OFF_Y + (16 * u + 2 * j) * (BM * 16), BM * 16, 128);
                const uint64_t bd = sdesc_kmajor_noswizzle(la + 2 * j * (p.rank2_pad * 16),
                                                           p.rank2_pad * 16, 128);
                mma_bf16(d, ad, bd, id_z, (u > 0 || j > 0) ? 1u : 0u);
              }
              mma_commit(lr_empty(ls));
            }
            mma_commit(tm_full(b));
            ++tb;
            ++ixh;
          }
        }
      mma_done:
        // every MMA this thread issued has completed before TMEM is freed,
        // on the normal path and after an abort alike
        mma_commit(mma_drain);
        mbar_wait_bounded(mma_drain, 0, p.limit_ns);
      }
      __syncwarp();
    } else {
      // ---------------------------------------------------- expanders
      // warps 2, 3, 6, 7 also copy a quarter of each group's correction digits
      // (one word per column) from the scale slot into the B correction slice
      const int xq_i = (warp == 4 || warp == 5) ? -1 : (warp & 3) - 2 + 2 * ((warp >> 2) & 1);
      auto expand_loop = [&](const auto& plan, auto btwos) {
        constexpr bool BT = decltype(btwos)::value;
        uint32_t ist = 0, it = 0;            // packed stages, groups
        for (int wk = blockIdx.x; wk < p.num_tiles * p.splits; wk += gridDim.x) {
          const WorkItem wi = work_item(p, wk);
          for (int g = wi.g0; g < wi.g1; g += 2, ++ist) {
            const int ng = wi.g1 - g < 2 ? 1 : 2;
            const int sp = ist % NP;
            if (!wait_or_abort(pk_full(sp), (ist / NP) & 1, abort_flag, p.err, p.limit_ns)) return;
            for (int k = 0; k < ng; ++k, ++it) {
              const int se = it % NE;
              if (!wait_or_abort(ex_empty(se), ((it / NE) & 1) ^ 1, abort_flag, p.err, p.limit_ns)) return;
              plan.template run<BT>(sbase + L::OFF_PK + sp * L::PK_STAGE,
                                    sbase + L::OFF_EX + se * L::EX_STAGE, 32u * k);
              if (xq_i >= 0) {
                const uint32_t cs = sbase + L::OFF_SC + (it % L::NS) * L::SC_SLOT + 4 * (BM + BN);
                const uint32_t xs = sbase + L::OFF_EX + se * L::EX_STAGE + L::EX_A + L::EX_B;
#pragma unroll
                for (int r = xq_i * (BN / 4) + lane; r < (xq_i + 1) * (BN / 4); r += 32)
                  sts32u(xs + 16u * r, lds32u(cs + 4u * r));
              }
              fence_proxy_async_smem();
              mbar_arrive(ex_full(se));
            }
            mbar_arrive(pk_empty(sp));
          }
        }
      };
      auto expand_share = [&](const auto& plan) {
        if (p.b_twos) expand_loop(plan, std::true_type{});
        else expand_loop(plan, std::false_type{});
      };
      // Each SM sub-partition gets the same expansion cost: a round of A
      // (two's-complement conversion) costs about twice a round of B
      // (sign-magnitude).  Warps 4 and 5 sit alone on their sub-partitions
      // (beside the producer and the MMA issuer) and take two rounds of A and
      // a quarter of B each; warps 2, 6 and 3, 7 share theirs and take one
      // round of A and an eighth of B each.
      constexpr int AR = BM * 2 / 32, BR = BN * 2 / 32;
      static_assert(AR == 8 && BR % 8 == 0, "expander split");
      if (warp == 4 || warp == 5) {
        const int i = warp - 4;
        expand_share(ExpandPlan<BN, 2, BR / 4>(2 * i, (BR / 4) * i, lane));
      } else {
        const int slot_i = (warp & 3) - 2 + 2 * ((warp >> 2) & 1);   // warps 2,3,6,7 -> 0,1,2,3
        expand_share(ExpandPlan<BN, 1, BR / 8>(4 + slot_i, BR / 2 + (BR / 8) * slot_i, lane));
      }
    }
  } else {
    regs_inc<REG_HI>();
    // ------------------------------------------------------ rescale + epilogue
    // TMEM lanes 32q..32q+31 (the warp's quarter), columns h*CW..h*CW+CW-1.
    // Rescale layout (.16x256b loads): this thread owns rows r0 + 8i (i < 4)
    // of the quarter and, in each 16-column chunk c, the column pairs
    // 16c + 8b + 2pq (+1), b < 2.  acc[i][2c + b] holds that pair.
    const int rw = warp - RES_WARP0, q = warp & 3, h = rw >> 2;
    const int pq = lane & 3, r0 = lane >> 2;
    float* bb = reinterpret_cast<float*>(smem + L::OFF_BIAS) + rw * CW;
    uint8_t* ystage = smem + L::OFF_Y + rw * L::Y_WARP;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    uint32_t tb = 0, gs = 0;                   // TMEM use counter, group counter
    bool ok = true;
    for (int wk = blockIdx.x; wk < p.num_tiles * p.splits && ok; wk += gridDim.x) {
      const WorkItem wi = work_item(p, wk);
      const int t = wi.t;
      const int m0 = (p.tile_m0 + t / p.tiles_n) * BM;
      const int n0 = (p.tile_n0 + t % p.tiles_n) * BN;
      const int row = m0 + 32 * q + lane;
      const int ncol0 = n0 + h * CW;           // first column of this warp
      float2 acc[4][CW / 8];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < CW / 8; ++j) acc[i][j] = make_float2(0.0f, 0.0f);
      constexpr int PER = CW / 32;             // bias values loaded per lane
      float bias_n[PER];                       // prefetched for the epilogue
      float ilam_n[PER];                       // MODE 4: the next layer's smoothing factors
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int n = ncol0 + lane * PER + e;
        bias_n[e] = (LAYER && n < p.N) ? __uint_as_float((uint32_t)__ldg(p.bias + n) << 16) : 0.0f;
        ilam_n[e] = (FUSE && n < p.N) ? __ldg(p.inv_lambda2 + n) : 0.0f;
      }
      for (int g = wi.g0; g < wi.g1; ++g, ++tb, ++gs) {
        const uint32_t slot = sbase + L::OFF_SC + (gs % L::NS) * L::SC_SLOT;
        const int b = tb % NB;
        if (!wait_or_abort(tm_full(b), (tb / NB) & 1, abort_flag, p.err, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ta = tmem + b * BN + h * CW + lane_off;
        if (LAYER) {
          // 16-column chunks, double-buffered: the loads of chunk c+1 are in
          // flight while chunk c is rescaled (wait::ld waits for all).
          float2 sx2[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float v = lds32(slot + 4u * (32 * q + r0 + 8 * i));
            sx2[i] = make_float2(v, v);
          }
          const uint32_t swa = slot + 4u * (BM + h * CW) + 16u * pq;
          // batches of RCH 16-column chunks, double-buffered: the loads of
          // batch cb+1 are in flight while batch cb is rescaled (wait::ld
          // waits for all of them)
          uint32_t rb[2][16 * RCH];
          auto load_batch = [&](int cb, uint32_t* dst) {
#pragma unroll
            for (int u = 0; u < RCH; ++u) {
              tmem_ld16x256b_x2(ta + 16 * (cb * RCH + u), dst + 16 * u);
              tmem_ld16x256b_x2(ta + 16 * (cb * RCH + u) + (16u << 16), dst + 16 * u + 8);
            }
          };
          constexpr int NBATCH = CW / (16 * RCH);
          load_batch(0, rb[0]);
          tmem_wait_ld();
#pragma unroll
          for (int cb = 0; cb < NBATCH; ++cb) {
            if (cb + 1 < NBATCH) load_batch(cb + 1, rb[(cb + 1) & 1]);
#pragma unroll
            for (int u = 0; u < RCH; ++u) {
              const int c = cb * RCH + u;
              const uint32_t* r = rb[cb & 1] + 16 * u;
              const float4 s4 = lds128(swa + 64u * c);   // columns 2pq, 2pq+1, 8+2pq, 9+2pq
#pragma unroll
              for (int bb = 0; bb < 2; ++bb) {
                const float2 sw2 = bb ? make_float2(s4.z, s4.w) : make_float2(s4.x, s4.y);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  // register of row r0 + 8i: half (i >> 1), row (i & 1) of the 16-lane load
                  const uint32_t* wv = r + 8 * (i >> 1) + 4 * bb + 2 * (i & 1);
                  // the word is P_g 2^-18 and sw2 holds s_w 2^18: v = fl32(P_g s_w)
                  const float2 v = __fmul2_rn(make_float2(__uint_as_float(wv[0]), __uint_as_float(wv[1])),
                                              sw2);
                  acc[i][2 * c + bb] = __ffma2_rn(v, sx2[i], acc[i][2 * c + bb]);
                }
              }
            }
            if (cb + 1 < NBATCH) tmem_wait_ld();
          }
        } else {
#pragma unroll 1
          for (int c = 0; c < CW / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(ta + 16 * c, r);
            tmem_wait_ld();
            const int i = row - p.row0;
            if (i >= 0 && i < p.nrows) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int jj = ncol0 + 16 * c + j - p.col0;
                if (jj >= 0 && jj < p.ncols)
                  p.P[((size_t)g * p.nrows + i) * p.ncols + jj] =
                      __float2int_rn(__uint_as_float(r[j]) * P_SCALE);   // exact
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tm_empty(b));
      }
      if (!ok || !LAYER) continue;
      if (wi.lr && p.n_lr > 0) {
        const int b = tb % NB;
        if (!wait_or_abort(tm_full(b), (tb / NB) & 1, abort_flag, p.err, p.limit_ns)) { ok = false; break; }
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
          for (int bb = 0; bb < 2; ++bb)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t* wv = r + 8 * (i >> 1) + 4 * bb + 2 * (i & 1);
              acc[i][2 * c + bb] = __fadd2_rn(acc[i][2 * c + bb],
                                              make_float2(__uint_as_float(wv[0]), __uint_as_float(wv[1])));
            }
          if (c + 1 < CW / 16) tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tm_empty(b));
        ++tb;
      }
      if (SPLIT) {
        // write this split's partial (thread-private order, same for every
        // split), publish it, and let the last arriving split of this warp's
        // slice sum all of them in split order
        float2* mine = reinterpret_cast<float2*>(
            p.part + ((size_t)(t * p.splits + wi.sp) * N_RES_WARPS + rw) * (32 * CW));
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int k = 0; k < CW / 8; ++k) mine[(i * (CW / 8) + k) * 32 + lane] = acc[i][k];
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(p.cnt + t * N_RES_WARPS + rw, 1);
        old = __shfl_sync(0xFFFFFFFFu, old, 0);
        if (old != p.splits - 1) continue;
        __threadfence();
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int k = 0; k < CW / 8; ++k) acc[i][k] = make_float2(0.0f, 0.0f);
        for (int sp = 0; sp < p.splits; ++sp) {
          const float2* src = reinterpret_cast<const float2*>(
              p.part + ((size_t)(t * p.splits + sp) * N_RES_WARPS + rw) * (32 * CW));
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k = 0; k < CW / 8; ++k)
              acc[i][k] = __fadd2_rn(acc[i][k], __ldcg(src + (i * (CW / 8) + k) * 32 + lane));
        }
        __syncwarp();
        if (lane == 0) atomicExch(p.cnt + t * N_RES_WARPS + rw, 0);   // ready for the next call
      }
      if constexpr (FUSE) {
        // epilogue of MODE 4: h = bf16(epi(acc + bias)) exactly as the stored Y
        // would be, x~ = fl32(h inv_lambda2), the codes and scale of each of
        // the warp's 64-column groups per row, and bf16(x~) into the
        // down-projection's A operand (the Y staging area, unused here)
        float* lb = reinterpret_cast<float*>(smem + L::OFF_ILAM) + rw * CW;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          bb[lane * PER + e] = bias_n[e];
          lb[lane * PER + e] = ilam_n[e];
        }
        __syncwarp();
        const bool gelu = p.epilogue == SVDQ_EPI_GELU;
        const bool zlr = p.n_l1 > 0;
        const uint32_t xa = sbase + L::OFF_Y;
        // one row and 64-column group per iteration: h = bf16(epi(acc + b)),
        // x~ = fl32(h inv_lambda2), bf16(x~) into the down-projection's A
        // operand (chunk kc = column / 8 of the tile at kc * BM * 16 bytes,
        // row at 16 bytes each), then the group's codes and scale
#pragma unroll 1
        for (int ji = 0; ji < 4 * (CW / 64); ++ji) {
          const int j = ji >> 2;
          float2 a8[8];                          // acc[i][8 j + k], i = ji % 4
          row_group(acc, ji, a8);
          const int gcol = ncol0 + 64 * j;       // first column of the group
          const int rl = 32 * q + r0 + 8 * (ji & 3);   // row within the tile
          float v[16];                           // value 4 cc + 2 b2 + e: column 16 cc + 8 b2 + 2 pq + e
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
            for (int b2 = 0; b2 < 2; ++b2) {
              const int c = 4 * j + cc;
              const int col = 16 * c + 8 * b2 + 2 * pq;
              const float2 bv = *reinterpret_cast<const float2*>(bb + col);
              const float2 lv = *reinterpret_cast<const float2*>(lb + col);
              float2 y = __fadd2_rn(a8[2 * cc + b2], bv);
              if (gelu) y = make_float2(gelu_f(y.x), gelu_f(y.y));
              const uint32_t hb = bf16x2_bits(y);
              const float2 xh = __fmul2_rn(
                  make_float2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xFFFF0000u)), lv);
              v[4 * cc + 2 * b2] = xh.x;
              v[4 * cc + 2 * b2 + 1] = xh.y;
              if (zlr) {
                const uint32_t kc = (uint32_t)(h * CW + 16 * c + 8 * b2) >> 3;
                sts32u(xa + kc * (BM * 16) + rl * 16 + 4 * pq, bf16x2_bits(xh));
              }
            }
          }
          uint32_t u[2];
          const float sc = quant_group16(v, u);
          const uint32_t w0 = quad_transpose(u[0], pq), w1 = quad_transpose(u[1], pq);
          const int row = m0 + rl;
          if (row < p.M && gcol < p.N) {
            *reinterpret_cast<uint2*>(p.xq2 + (size_t)row * (p.N / 2) + gcol / 2 + 8 * pq) =
                make_uint2(w0, w1);
            if (pq == 0) p.s_x2[(size_t)(gcol / 64) * p.M + row] = sc;
          }
        }
        if (zlr) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(xh_full);
          // the tile's partial down-projection: 32x32b load, lane = row
          const int b = tb % NB;
          if (!wait_or_abort(tm_full(b), (tb / NB) & 1, abort_flag, p.err, p.limit_ns)) { ok = false; break; }
          tc_fence_after();
          if (16 * h < p.rank2_pad) {
            uint32_t r[16];
            tmem_ld16(tmem + b * BN + 16 * h + lane_off, r);
            tmem_wait_ld();
            const int row = m0 + 32 * q + lane;
            if (row < p.M) {
              // rank2 is a multiple of 8: whole 16-byte stores
              float4* zr = reinterpret_cast<float4*>(
                  p.zpart + ((size_t)(t % p.tiles_n) * p.M + row) * p.rank2 + 16 * h);
#pragma unroll
              for (int jj = 0; jj < 4; ++jj)
                if (16 * h + 4 * jj < p.rank2)
                  zr[jj] = make_float4(__uint_as_float(r[4 * jj]), __uint_as_float(r[4 * jj + 1]),
                                       __uint_as_float(r[4 * jj + 2]), __uint_as_float(r[4 * jj + 3]));
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tm_empty(b));
          ++tb;
        }
      } else {
      // epilogue: bias, GELU, bf16, swizzled staging, TMA store
#pragma unroll
      for (int e = 0; e < PER; ++e) bb[lane * PER + e] = bias_n[e];
      if (lane == 0) tma_store_wait_read0();
      __syncwarp();
      const float* bb_base = bb;
      const bool gelu = p.epilogue == SVDQ_EPI_GELU;
      // row r0 + 8i of the warp's 32, column pair 16c + 8b + 2pq: 4 bytes of the
      // 128-byte row of box c / 4, in 16-byte chunk (2c + b) & 7, swizzled by row
#pragma unroll
      for (int c = 0; c < CW / 16; ++c) {
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const int col = 16 * c + 8 * bb + 2 * pq;
          const float2 bv = *reinterpret_cast<const float2*>(bb_base + col);
          uint8_t* yb = ystage + (c >> 2) * L::Y_BOX + 4 * pq;
          const int ch = (2 * c + bb) & 7;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float2 v = __fadd2_rn(acc[i][2 * c + bb], bv);
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
          tma_store_2d(&tm_y, ncol0 + box * 64, m0 + 32 * q,
                       smem_u32(ystage + box * L::Y_BOX));
        tma_store_commit();
      }
      __syncwarp();
      }
    }
    if (LAYER && lane == 0) tma_store_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host side

struct LinMaps {
  CUtensorMap ta, tb, ty, tz, tl, tsx, tsw, tl1, tcs;
};

template <int BN, int MODE>
cudaError_t launch_ws(const LinMaps& m, LinArgs a, int tiles_m, cudaStream_t st) {
  using L = Lay<BN>;
  static bool attr[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (!attr[dev]) {
    cudaFuncAttributes fa;
    cudaError_t e0 = cudaFuncGetAttributes(&fa, linear_ws_kernel<BN, MODE>);
    if (e0 != cudaSuccess) return e0;
    if (fa.numRegs < REG_NEED) return cudaErrorInvalidConfiguration;  // split would not fit
    cudaError_t e = cudaFuncSetAttribute(linear_ws_kernel<BN, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    attr[dev] = true;
  }
  a.num_tiles = tiles_m * a.tiles_n;
  const int work = a.num_tiles * a.splits;
  const int grid = work < num_sms() ? work : num_sms();
  linear_ws_kernel<BN, MODE><<<grid, THREADS, L::ALLOC, st>>>(m.ta, m.tb, m.ty, m.tz, m.tl, m.tsx,
                                                              m.tsw, m.tl1, m.tcs, a);
  return cudaGetLastError();
}

// The correction digits [G][N_pad], one 32-bit word per column: a {BN x 1} box.
bool cs_map(const svdq_weights* w, int BN, LinMaps& m) {
  return make_map(&m.tcs, w->d_wcs, CU_TENSOR_MAP_DATA_TYPE_UINT32, w->N_pad, w->G,
                  (uint64_t)w->N_pad * 4, BN, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
}

int pick_bn(int N) {
  if (N <= 128) return 128;
  const int r = N % 256;
  return (r != 0 && r <= 128) ? 128 : 256;
}

// Tensor maps and kernel arguments shared by the layer launches.
bool build_linear(const svdq_weights* w, int M, const uint8_t* xq, const float* s_x,
                  const uint16_t* Z, uint16_t* Y, int ldy, int epilogue, int BN, LinMaps& m,
                  LinArgs& a) {
  if (!make_map(&m.ta, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->K / 2, M, w->K / 2, 64, BM,
                CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map(&m.tb, w->d_wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->K / 2, w->N, w->K / 2, 64, BN,
                CU_TENSOR_MAP_SWIZZLE_64B))
    return false;
  m.ty = m.ta;   // no Y in MODE 4
  if (Y && !make_map(&m.ty, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->N, M, (uint64_t)ldy * 2, 64, 32,
                     CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  m.tz = m.ta;
  m.tl1 = m.ta;
  m.tl = m.ta;
  m.tsx = m.ta;
  const bool sx_tma = (M % 4) == 0;
  if ((sx_tma && !make_map(&m.tsx, s_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, M, w->G,
                           (uint64_t)M * 4, BM, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) ||
      !make_map(&m.tsw, w->d_sw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w->N16, w->G,
                (uint64_t)w->N16 * 4, BN, 1, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !cs_map(w, BN, m))
    return false;
  if (w->rank > 0 &&
      (!make_map(&m.tz, Z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->rank, M, (uint64_t)w->rank * 2, 8,
                 BM, CU_TENSOR_MAP_SWIZZLE_NONE) ||
       !make_map(&m.tl, w->d_L2T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->rank_pad32, w->N,
                 (uint64_t)w->rank_pad32 * 2, 8, BN, CU_TENSOR_MAP_SWIZZLE_NONE)))
    return false;
  a = LinArgs{};
  a.s_x = s_x; a.s_w = w->d_sw; a.Z = Z; a.L2T = w->d_L2T; a.bias = w->d_bias;
  a.M = M; a.N = w->N; a.K = w->K; a.G = w->G;
  a.rank = w->rank; a.rank_pad32 = w->rank_pad32; a.n_lr = (w->rank + 15) / 16;
  a.epilogue = epilogue;
  a.tiles_n = (w->N + BN - 1) / BN;
  a.tile_m0 = 0; a.tile_n0 = 0;
  a.err = w->d_err;
  a.limit_ns = LIMIT_NS;
  a.stall = 0;
  a.b_twos = w->wq_twos ? 1 : 0;
  a.sx_tma = sx_tma ? 1 : 0;
  a.splits = 1;
  return true;
}

int num_tiles(const svdq_weights* w, int M) {
  const int BN = pick_bn(w->N);
  return ((M + BM - 1) / BM) * ((w->N + BN - 1) / BN);
}

size_t splitk_counter_bytes(const svdq_weights* w, int M) {
  return ((size_t)num_tiles(w, M) * N_RES_WARPS * sizeof(int) + 255) / 256 * 256;
}

}  // namespace

cudaError_t launch_linear(const svdq_weights* w, int M, const uint8_t* xq, const float* s_x,
                          const uint16_t* Z, uint16_t* Y, int ldy, int epilogue,
                          cudaStream_t st) {
  const int BN = pick_bn(w->N);
  LinMaps m;
  LinArgs a;
  if (!build_linear(w, M, xq, s_x, Z, Y, ldy, epilogue, BN, m, a)) return cudaErrorInvalidValue;
  const int tiles_m = (M + BM - 1) / BM;
  return BN == 256 ? launch_ws<256, 0>(m, a, tiles_m, st) : launch_ws<128, 0>(m, a, tiles_m, st);
}

cudaError_t launch_linear_stall(const svdq_weights* w, int M, const uint8_t* xq,
                                const float* s_x, const uint16_t* Z, uint16_t* Y, int ldy,
                                uint64_t limit_ns, cudaStream_t st) {
  const int BN = pick_bn(w->N);
  LinMaps m;
  LinArgs a;
  if (!build_linear(w, M, xq, s_x, Z, Y, ldy, SVDQ_EPI_NONE, BN, m, a)) return cudaErrorInvalidValue;
  a.limit_ns = limit_ns;
  a.stall = 1;
  const int tiles_m = (M + BM - 1) / BM;
  return BN == 256 ? launch_ws<256, 0>(m, a, tiles_m, st) : launch_ws<128, 0>(m, a, tiles_m, st);
}

int splitk_auto(const svdq_weights* w, int M) {
  const int tiles = num_tiles(w, M);
  if (2 * tiles > num_sms()) return 1;          // the tiles alone fill the GPU
  int s = num_sms() / (tiles > 0 ? tiles : 1);
  const int cap = w->G / 2 < SVDQ_MAX_SPLITS ? w->G / 2 : SVDQ_MAX_SPLITS;   // >= 2 groups each
  if (s > cap) s = cap;
  return s < 1 ? 1 : s;
}

size_t splitk_workspace(const svdq_weights* w, int M, int splits) {
  const int BN = pick_bn(w->N);
  return splitk_counter_bytes(w, M) + (size_t)num_tiles(w, M) * splits * BM * BN * sizeof(float);
}

cudaError_t launch_linear_splitk(const svdq_weights* w, int M, const uint8_t* xq,
                                 const float* s_x, const uint16_t* Z, uint16_t* Y, int ldy,
                                 int epilogue, int splits, void* workspace, cudaStream_t st) {
  if (splits == 1)      // nothing to split: the plain kernel, same result bits
    return launch_linear(w, M, xq, s_x, Z, Y, ldy, epilogue, st);
  const int BN = pick_bn(w->N);
  LinMaps m;
  LinArgs a;
  if (!build_linear(w, M, xq, s_x, Z, Y, ldy, epilogue, BN, m, a)) return cudaErrorInvalidValue;
  const size_t cb = splitk_counter_bytes(w, M);
  a.splits = splits;
  a.cnt = static_cast<int*>(workspace);
  a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + cb);
  // the arrival counts must start at zero (the kernel also leaves them at zero)
  cudaError_t e = cudaMemsetAsync(workspace, 0, cb, st);
  if (e != cudaSuccess) return e;
  const int tiles_m = (M + BM - 1) / BM;
  return BN == 256 ? launch_ws<256, 3>(m, a, tiles_m, st) : launch_ws<128, 3>(m, a, tiles_m, st);
}

cudaError_t launch_partials(const svdq_weights* w, int M, const uint8_t* xq, int row0,
                            int nrows, int col0, int ncols, int32_t* P, cudaStream_t st) {
  const int BN = pick_bn(w->N);
  LinMaps m;
  if (!make_map(&m.ta, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->K / 2, M, w->K / 2, 64, BM,
                CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map(&m.tb, w->d_wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->K / 2, w->N, w->K / 2, 64, BN,
                CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  m.ty = m.tz = m.tl = m.tsx = m.tsw = m.tl1 = m.ta;
  if (!cs_map(w, BN, m)) return cudaErrorInvalidValue;
  LinArgs a{};
  a.M = M; a.N = w->N; a.K = w->K; a.G = w->G;
  a.rank = 0; a.rank_pad32 = 0; a.n_lr = 0; a.epilogue = 0;
  a.splits = 1;
  a.err = w->d_err;
  a.limit_ns = LIMIT_NS;
  a.stall = 0;
  a.b_twos = w->wq_twos ? 1 : 0;
  a.P = P; a.row0 = row0; a.nrows = nrows; a.col0 = col0; a.ncols = ncols;
  const int tm0 = row0 / BM, tm1 = (row0 + nrows - 1) / BM;
  const int tn0 = col0 / BN, tn1 = (col0 + ncols - 1) / BN;
  a.tile_m0 = tm0; a.tile_n0 = tn0; a.tiles_n = tn1 - tn0 + 1;
  return BN == 256 ? launch_ws<256, 1>(m, a, tm1 - tm0 + 1, st)
                   : launch_ws<128, 1>(m, a, tm1 - tm0 + 1, st);
}

namespace {
// Z = bf16(sum over the column tiles t, in order, of part[t]) element by
// element: the next layer's Z of MODE 4.
__global__ void zpart_sum_kernel(const float* __restrict__ part, uint16_t* __restrict__ Z,
                                 long long n, int tiles) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int t = 0; t < tiles; ++t) s = __fadd_rn(s, __ldcs(part + (size_t)t * n + i));
    Z[i] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
  }
}
}  // namespace

size_t linear_next_workspace(const svdq_weights* w, const svdq_weights* w2, int M) {
  const int BN = pick_bn(w->N);
  return (size_t)((w->N + BN - 1) / BN) * M * w2->rank * sizeof(float);
}

cudaError_t launch_linear_next(const svdq_weights* w, const svdq_weights* w2, int M,
                               const uint8_t* xq, const float* s_x, const uint16_t* Z,
                               int epilogue, uint8_t* xq2, float* s_x2, uint16_t* Z2,
                               float* zpart, cudaStream_t st) {
  const int BN = pick_bn(w->N);
  LinMaps m;
  LinArgs a;
  if (!build_linear(w, M, xq, s_x, Z, nullptr, w->N, epilogue, BN, m, a)) return cudaErrorInvalidValue;
  a.inv_lambda2 = w2->d_inv_lambda;
  a.xq2 = xq2;
  a.s_x2 = s_x2;
  a.zpart = zpart;
  a.rank2 = w2->rank;
  a.rank2_pad = w2->rank_pad;
  a.n_l1 = w2->rank > 0 ? BN / 128 : 0;
  const long long nz = (long long)M * w2->rank;
  if (w2->rank > 0) {
    if (!make_map(&m.tl1, w2->d_L1T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w2->K, w2->rank_pad,
                  (uint64_t)w2->K * 2, 8, w2->rank_pad, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  const int tiles_m = (M + BM - 1) / BM;
  cudaError_t e = BN == 256 ? launch_ws<256, 4>(m, a, tiles_m, st) : launch_ws<128, 4>(m, a, tiles_m, st);
  if (e != cudaSuccess || nz == 0) return e;
  long long blocks = (nz + 255) / 256;
  if (blocks > 8LL * num_sms()) blocks = 8LL * num_sms();
  zpart_sum_kernel<<<(int)blocks, 256, 0, st>>>(zpart, Z2, nz, a.tiles_n);
  return cudaGetLastError();
}

}  // namespace svdq
