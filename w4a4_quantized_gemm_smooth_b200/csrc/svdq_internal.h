// Internal declarations shared by the host pack code and the device launchers.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "svdq.h"

struct svdq_weights {
  int K = 0, N = 0, G = 0;
  int rank = 0;        // total branch rank = svd_rank + lora_rank
  int svd_rank = 0, lora_rank = 0;
  int rank_pad = 0;    // rank rounded up to a multiple of 16 (zero rows)
  int rank_pad32 = 0;  // rank rounded up to a multiple of 32
  int N_pad = 0;       // N rounded up to a multiple of 256
  int N16 = 0;         // N rounded up to a multiple of 16 (row pitch of d_sw)
  int device = 0;
  int format = SVDQ_FORMAT_W4A4;   // residual / activation number format
  // device copies (owned)
  float* d_inv_lambda = nullptr;   // [K]
  // [N][K/2] packed residual codes, two per byte (even k low); each nibble is
  // sign << 3 | |q| (the GEMM's cheap E4M3 expansion), or the code in two's
  // complement when the layer holds a -8 (wq_twos)
  uint8_t* d_wq = nullptr;
  bool wq_twos = false;
  // [G][N16] weight scales times 2^18 (exact; the GEMM's group sums arrive as
  // P_g 2^-18), zero padded; inside each block of 16 columns, column
  // 8b + 2p + e is stored at 4p + 2b + e, so that the rescale thread that owns
  // the column pairs 2p, 2p+1 of both 8-column halves reads them as one float4
  float* d_sw = nullptr;
  // [G][N_pad] per group and column, the E4M3 bytes (0..2) of the balanced
  // base-8 digits d0 + 8 d1 + 64 d2 = -sum_k q_w over the group, zero padded.
  // The GEMM takes the activation codes as q + 8 (offset binary, its cheapest
  // expansion) and adds these digits times the constants 8, 64, 512 in one
  // more K = 32 MMA, which restores the exact group sum.
  uint32_t* d_wcs = nullptr;
  uint16_t* d_L1T = nullptr;       // [rank_pad][K] bf16, transposed L1
  uint16_t* d_L2 = nullptr;        // [rank_pad][N] bf16
  uint16_t* d_L2T = nullptr;       // [N_pad][rank_pad32] bf16, transposed L2
  uint16_t* d_bias = nullptr;      // [N] bf16
  int8_t* d_wq8 = nullptr;         // W8A8: [N][K] int8 residual codes
  float* d_sw8 = nullptr;          // W8A8: [N_pad] per-output-channel scales, zero padded
  uint8_t* d_wq4 = nullptr;        // NVFP4: [N][K/2] packed E2M1 codes
  uint8_t* d_sfb4 = nullptr;       // NVFP4: group scales in the tensor-core atom layout
                                   //   [N_pad/128][K/64][512 B] (svdq::nvfp4_sf_offset)
  float* d_sw4 = nullptr;          // NVFP4: [N_pad] row scales, zero padded
  int* d_err = nullptr;            // sticky device error word
  // host copies (export / save)
  std::vector<float> inv_lambda;
  std::vector<uint8_t> wq;
  std::vector<float> sw;
  std::vector<int8_t> wq8;         // W8A8 codes [N][K]
  std::vector<float> sw8;          // W8A8 scales [N]
  std::vector<uint8_t> wq4;        // NVFP4 codes [N][K/2]
  std::vector<uint8_t> sf4;        // NVFP4 E4M3 group scales [N][K/16]
  std::vector<float> sw4;          // NVFP4 row scales [N]
  std::vector<uint16_t> L1;        // [K][rank]
  std::vector<uint16_t> L2;        // [rank][N]
  std::vector<uint16_t> bias;      // [N]
  std::vector<double> sigma;       // [svd_rank + 1]
};

// The W4A4 GEMM multiplies E4M3 operands holding q 2^-9 and receives each
// group sum as P_g 2^-18; the device weight scales carry the factor 2^18.
// Scales at or above this bound would overflow (a residual group maximum
// above 7 * 2^110, about 9e33) and are rejected by the pack.
constexpr double SVDQ_SW_LIMIT = 1.2980742146337069e33;   // 2^110

// Device error word values.
enum { SVDQ_DEVERR_NONE = 0, SVDQ_DEVERR_TIMEOUT = 1 };

namespace svdq {

// NVFP4 group-scale atom layout shared by the pack, the activation pass and
// the GEMM: the scales of rows [128 a, 128 a + 128) and K block kb (64
// elements, four groups of 16) form a 512-byte atom; row r (within the
// block) sits at byte 16 (r % 32) + 4 (r / 32), group j (within the K
// block) at + j.  This is the layout tcgen05.cp 32x128b.warpx4 turns into
// the tensor-core scale-factor layout in TMEM.
inline size_t nvfp4_sf_offset(int row, int k16, int K) {
  const int a = row >> 7, r = row & 127, kb = k16 >> 2;
  return ((size_t)a * (K / 64) + kb) * 512 + 16 * (r & 31) + 4 * (r >> 5) + (k16 & 3);
}
inline size_t nvfp4_sf_bytes(int rows, int K) { return (size_t)((rows + 127) / 128) * (K / 64) * 512; }

// Upload the host copies of `w` to the current device (allocates).
svdq_status upload(svdq_weights* w, cudaStream_t stream);

// Kernel launchers (capi_device.cu validates, these only launch).
cudaError_t launch_act_quant(const svdq_weights* w, int M, const uint16_t* X,
                             int ldx, uint8_t* xq, float* s_x, uint16_t* Z,
                             cudaStream_t stream);
cudaError_t launch_linear(const svdq_weights* w, int M, const uint8_t* xq,
                          const float* s_x, const uint16_t* Z, uint16_t* Y,
                          int ldy, int epilogue, cudaStream_t stream);
// Argument checks of the svdq_linear entry points (SVDQ_OK or the error),
// and the split count a call resolves to (-1: invalid).
svdq_status check_linear(const svdq_weights* w, int M, const uint8_t* xq, const float* s_x,
                         const uint16_t* Z, const uint16_t* Y, int ldy, int epilogue);
int resolve_splits(const svdq_weights* w, int M, int splits);

// Split-K form of launch_linear (K groups of each tile spread over `splits`
// work items; workspace = zeroed counters then fp32 partials, sized by
// splitk_workspace).  splitk_auto picks a split count for M.
int splitk_auto(const svdq_weights* w, int M);
size_t splitk_workspace(const svdq_weights* w, int M, int splits);
cudaError_t launch_linear_splitk(const svdq_weights* w, int M, const uint8_t* xq,
                                 const float* s_x, const uint16_t* Z, uint16_t* Y, int ldy,
                                 int epilogue, int splits, void* workspace, cudaStream_t stream);
// W8A8 comparator: per-token int8 activation pass and the int8 product.
cudaError_t launch_act_quant_w8a8(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                                  int8_t* xq, float* s_x, uint16_t* Z, cudaStream_t stream);
cudaError_t launch_linear_w8a8(const svdq_weights* w, int M, const int8_t* xq, const float* s_x,
                               const uint16_t* Z, uint16_t* Y, int ldy, int epilogue,
                               cudaStream_t stream);
// NVFP4 variant: activation pass and block-scaled product.
cudaError_t launch_act_quant_nvfp4(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                                   uint8_t* xq, uint8_t* sfa, float* s_x, uint16_t* Z,
                                   cudaStream_t stream);
cudaError_t launch_linear_nvfp4(const svdq_weights* w, int M, const uint8_t* xq,
                                const uint8_t* sfa, const float* s_x, const uint16_t* Z,
                                uint16_t* Y, int ldy, int epilogue, cudaStream_t stream);
// launch_linear whose epilogue emits the next layer's activation side (codes,
// scales, and Z through per-column-tile fp32 partials in zpart, sized by
// linear_next_workspace) instead of Y.
size_t linear_next_workspace(const svdq_weights* w, const svdq_weights* w2, int M);
cudaError_t launch_linear_next(const svdq_weights* w, const svdq_weights* w2, int M,
                               const uint8_t* xq, const float* s_x, const uint16_t* Z,
                               int epilogue, uint8_t* xq2, float* s_x2, uint16_t* Z2,
                               float* zpart, cudaStream_t stream);
// Test hook: launch_linear whose waits are bounded by limit_ns and whose CTA
// 0 producer withholds its first stage (the consumers' waits run out).
cudaError_t launch_linear_stall(const svdq_weights* w, int M, const uint8_t* xq,
                                const float* s_x, const uint16_t* Z, uint16_t* Y, int ldy,
                                uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_partials(const svdq_weights* w, int M, const uint8_t* xq,
                            int row0, int nrows, int col0, int ncols,
                            int32_t* P, cudaStream_t stream);

// Host linear algebra for the pack (svd_host.cpp).
// Leading `nsv` singular triplets of the K x N row-major matrix A:
// sigma[0..nsv), L1 = U S as K x r row-major, L2 = V^T as r x N row-major,
// for r = min(nsv, r_out) columns/rows.  Returns 0 on success.
int top_singular(const double* A, int K, int N, int nsv, int r_out,
                 double* sigma, double* L1, double* L2);

}  // namespace svdq
