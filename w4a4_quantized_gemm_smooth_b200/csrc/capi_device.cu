// C ABI of the hot path: argument checks, then one kernel launch per call.
#include <cstdint>

#include "svdq_internal.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

svdq_status check_handle(const svdq_weights* w) {
  if (!w || !w->d_wq || !w->d_err) return SVDQ_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev != w->device) return SVDQ_ERR_INVALID_ARG;
  return SVDQ_OK;
}

// A handle of the W8A8 comparator, uploaded to the current device.
svdq_status check_handle_w8a8(const svdq_weights* w) {
  if (!w || w->format != SVDQ_FORMAT_W8A8 || !w->d_wq8 || !w->d_err) return SVDQ_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev != w->device) return SVDQ_ERR_INVALID_ARG;
  return SVDQ_OK;
}

// A handle of the NVFP4 variant, uploaded to the current device.
svdq_status check_handle_nvfp4(const svdq_weights* w) {
  if (!w || w->format != SVDQ_FORMAT_NVFP4 || !w->d_wq4 || !w->d_err) return SVDQ_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev != w->device) return SVDQ_ERR_INVALID_ARG;
  return SVDQ_OK;
}

svdq_status from_launch(cudaError_t e) { return e == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA; }

}  // namespace

namespace svdq {
// Validation shared by the svdq_linear entry points.
svdq_status check_linear(const svdq_weights* w, int M, const uint8_t* xq, const float* s_x,
                         const uint16_t* Z, const uint16_t* Y, int ldy, int epilogue) {
  svdq_status s = check_handle(w);
  if (s != SVDQ_OK) return s;
  if (M < 0 || ldy < w->N) return SVDQ_ERR_SHAPE;
  if (epilogue != SVDQ_EPI_NONE && epilogue != SVDQ_EPI_GELU) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!xq || !s_x || !Y || (w->rank > 0 && !Z)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(s_x) || !aligned16(Y) || (ldy % 8) != 0 ||
      (w->rank > 0 && !aligned16(Z)))
    return SVDQ_ERR_ALIGNMENT;
  return SVDQ_OK;
}

int resolve_splits(const svdq_weights* w, int M, int splits) {
  const int cap = w->G < SVDQ_MAX_SPLITS ? w->G : SVDQ_MAX_SPLITS;
  if (splits < 0 || splits > cap) return -1;
  return splits == 0 ? svdq::splitk_auto(w, M) : splits;
}
}  // namespace svdq
using svdq::check_linear;
using svdq::resolve_splits;

extern "C" {

svdq_status svdq_quantize_act(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                              uint8_t* xq, float* s_x, uint16_t* Z, cudaStream_t stream) {
  svdq_status s = check_handle(w);
  if (s != SVDQ_OK) return s;
  if (M < 0 || ldx < w->K) return SVDQ_ERR_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!X || !xq || !s_x || (w->rank > 0 && !Z)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(xq) || !aligned16(s_x) || (ldx % 8) != 0 ||
      (w->rank > 0 && !aligned16(Z)))
    return SVDQ_ERR_ALIGNMENT;
  return from_launch(svdq::launch_act_quant(w, M, X, ldx, xq, s_x, Z, stream));
}
svdq_status svdq_linear(const svdq_weights* w, int M, const uint8_t* xq, const float* s_x,
                        const uint16_t* Z, uint16_t* Y, int ldy, int epilogue,
                        cudaStream_t stream) {
  svdq_status s = check_linear(w, M, xq, s_x, Z, Y, ldy, epilogue);
  if (s != SVDQ_OK || M == 0) return s;
  return from_launch(svdq::launch_linear(w, M, xq, s_x, Z, Y, ldy, epilogue, stream));
}

// Device workspace of svdq_linear_host: X, codes, scales, Z and Y, each
// starting on a 256-byte boundary; Y rows padded to a multiple of 8.
struct HostLayerLayout {
  size_t x, xq, sx, z, y, total;
  int ldyd;
};
static HostLayerLayout host_layer_layout(const svdq_weights* w, int M) {
  auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
  const size_t m = (size_t)M, K = (size_t)w->K, N = (size_t)w->N, r = (size_t)w->rank;
  HostLayerLayout L;
  L.ldyd = (int)((N + 7) / 8 * 8);
  L.x = 0;
  L.xq = L.x + up(m * K * 2);
  L.sx = L.xq + up(m * K / 2);
  L.z = L.sx + up((K / 64) * m * 4);
  L.y = L.z + up(m * r * 2);
  L.total = L.y + up(m * (size_t)L.ldyd * 2);
  return L;
}

size_t svdq_linear_host_workspace(const svdq_weights* w, int M) {
  if (!w || M <= 0 || !w->d_wq) return 0;
  return host_layer_layout(w, M).total;
}

svdq_status svdq_linear_host(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                             uint16_t* Y, int ldy, int epilogue, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
  svdq_status s = check_handle(w);
  if (s != SVDQ_OK) return s;
  if (M < 0 || ldx < w->K || ldy < w->N) return SVDQ_ERR_SHAPE;
  if (epilogue != SVDQ_EPI_NONE && epilogue != SVDQ_EPI_GELU) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !Y || !workspace) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return SVDQ_ERR_ALIGNMENT;
  const HostLayerLayout L = host_layer_layout(w, M);
  if (workspace_bytes < L.total) return SVDQ_ERR_SHAPE;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint16_t* Xd = reinterpret_cast<uint16_t*>(base + L.x);
  uint8_t* xq = base + L.xq;
  float* sx = reinterpret_cast<float*>(base + L.sx);
  uint16_t* Zd = w->rank > 0 ? reinterpret_cast<uint16_t*>(base + L.z) : nullptr;
  uint16_t* Yd = reinterpret_cast<uint16_t*>(base + L.y);
  const size_t K = (size_t)w->K, N = (size_t)w->N;
  if (cudaMemcpy2DAsync(Xd, K * 2, X, (size_t)ldx * 2, K * 2, (size_t)M, cudaMemcpyHostToDevice,
                        stream) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  s = svdq_quantize_act(w, M, Xd, w->K, xq, sx, Zd, stream);
  if (s != SVDQ_OK) return s;
  s = svdq_linear(w, M, xq, sx, Zd, Yd, L.ldyd, epilogue, stream);
  if (s != SVDQ_OK) return s;
  if (cudaMemcpy2DAsync(Y, (size_t)ldy * 2, Yd, (size_t)L.ldyd * 2, N * 2, (size_t)M,
                        cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return SVDQ_OK;
}

size_t svdq_linear_quantize_next_workspace(const svdq_weights* w, const svdq_weights* w_next,
                                           int M) {
  if (!w || !w_next || M <= 0 || !w->d_wq || !w_next->d_wq || w_next->K != w->N) return 0;
  return svdq::linear_next_workspace(w, w_next, M);
}

svdq_status svdq_linear_quantize_next(const svdq_weights* w, const svdq_weights* w_next,
                                      int M, const uint8_t* xq, const float* s_x,
                                      const uint16_t* Z, int epilogue, uint8_t* xq_next,
                                      float* s_x_next, uint16_t* Z_next, void* workspace,
                                      size_t workspace_bytes, cudaStream_t stream) {
  svdq_status s = check_handle(w);
  if (s != SVDQ_OK) return s;
  s = check_handle(w_next);
  if (s != SVDQ_OK) return s;
  if (M < 0 || w_next->K != w->N || w_next->rank > 32) return SVDQ_ERR_SHAPE;
  if (epilogue != SVDQ_EPI_NONE && epilogue != SVDQ_EPI_GELU) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  const bool z2 = w_next->rank > 0;
  if (!xq || !s_x || (w->rank > 0 && !Z) || !xq_next || !s_x_next ||
      (z2 && (!Z_next || !workspace)))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(s_x) || (w->rank > 0 && !aligned16(Z)) ||
      !aligned16(xq_next) || !aligned16(s_x_next) ||
      (z2 && (!aligned16(Z_next) || !aligned16(workspace))))
    return SVDQ_ERR_ALIGNMENT;
  if (z2 && workspace_bytes < svdq::linear_next_workspace(w, w_next, M)) return SVDQ_ERR_SHAPE;
  return from_launch(svdq::launch_linear_next(w, w_next, M, xq, s_x, Z, epilogue, xq_next,
                                              s_x_next, Z_next, static_cast<float*>(workspace),
                                              stream));
}

size_t svdq_linear_splitk_workspace(const svdq_weights* w, int M, int splits) {
  if (!w || M <= 0 || !w->d_wq) return 0;
  const int sp = resolve_splits(w, M, splits);
  return sp < 1 ? 0 : svdq::splitk_workspace(w, M, sp);
}

svdq_status svdq_linear_splitk(const svdq_weights* w, int M, const uint8_t* xq,
                               const float* s_x, const uint16_t* Z, uint16_t* Y, int ldy,
                               int epilogue, int splits, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
  svdq_status s = check_linear(w, M, xq, s_x, Z, Y, ldy, epilogue);
  if (s != SVDQ_OK || M == 0) return s;
  const int sp = resolve_splits(w, M, splits);
  if (sp < 1 || !workspace) return SVDQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SVDQ_ERR_ALIGNMENT;
  if (workspace_bytes < svdq::splitk_workspace(w, M, sp)) return SVDQ_ERR_SHAPE;
  return from_launch(svdq::launch_linear_splitk(w, M, xq, s_x, Z, Y, ldy, epilogue, sp,
                                                workspace, stream));
}

svdq_status svdq_debug_partials(const svdq_weights* w, int M, const uint8_t* xq, int row0,
                                int nrows, int col0, int ncols, int32_t* P,
                                cudaStream_t stream) {
  svdq_status s = check_handle(w);
  if (s != SVDQ_OK) return s;
  if (M < 1 || nrows < 1 || ncols < 1 || row0 < 0 || col0 < 0 || row0 + nrows > M ||
      col0 + ncols > w->N)
    return SVDQ_ERR_SHAPE;
  if (!xq || !P) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(P)) return SVDQ_ERR_ALIGNMENT;
  return from_launch(svdq::launch_partials(w, M, xq, row0, nrows, col0, ncols, P, stream));
}

svdq_status svdq_debug_linear_stall(const svdq_weights* w, int M, const uint8_t* xq,
                                    const float* s_x, const uint16_t* Z, uint16_t* Y, int ldy,
                                    unsigned int limit_us, cudaStream_t stream) {
  svdq_status s = check_linear(w, M, xq, s_x, Z, Y, ldy, SVDQ_EPI_NONE);
  if (s != SVDQ_OK || M == 0) return s;
  if (limit_us < 1 || limit_us > 2000000u) return SVDQ_ERR_INVALID_ARG;
  return from_launch(svdq::launch_linear_stall(w, M, xq, s_x, Z, Y, ldy,
                                               (uint64_t)limit_us * 1000u, stream));
}

svdq_status svdq_quantize_act_w8a8(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                                   int8_t* xq, float* s_x, uint16_t* Z, cudaStream_t stream) {
  svdq_status s = check_handle_w8a8(w);
  if (s != SVDQ_OK) return s;
  if (M < 0 || ldx < w->K) return SVDQ_ERR_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!X || !xq || !s_x || (w->rank > 0 && !Z)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(xq) || !aligned16(s_x) || (ldx % 8) != 0 ||
      (w->rank > 0 && !aligned16(Z)))
    return SVDQ_ERR_ALIGNMENT;
  return from_launch(svdq::launch_act_quant_w8a8(w, M, X, ldx, xq, s_x, Z, stream));
}

svdq_status svdq_linear_w8a8(const svdq_weights* w, int M, const int8_t* xq, const float* s_x,
                             const uint16_t* Z, uint16_t* Y, int ldy, int epilogue,
                             cudaStream_t stream) {
  svdq_status s = check_handle_w8a8(w);
  if (s != SVDQ_OK) return s;
  if (M < 0 || ldy < w->N) return SVDQ_ERR_SHAPE;
  if (epilogue != SVDQ_EPI_NONE && epilogue != SVDQ_EPI_GELU) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!xq || !s_x || !Y || (w->rank > 0 && !Z)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(s_x) || !aligned16(Y) || (ldy % 8) != 0 ||
      (w->rank > 0 && !aligned16(Z)))
    return SVDQ_ERR_ALIGNMENT;
  return from_launch(svdq::launch_linear_w8a8(w, M, xq, s_x, Z, Y, ldy, epilogue, stream));
}

svdq_status svdq_quantize_act_nvfp4(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                                    uint8_t* xq, uint8_t* sfa, float* s_x, uint16_t* Z,
                                    cudaStream_t stream) {
  svdq_status s = check_handle_nvfp4(w);
  if (s != SVDQ_OK) return s;
  if (M < 0 || ldx < w->K) return SVDQ_ERR_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!X || !xq || !sfa || !s_x || (w->rank > 0 && !Z)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(xq) || !aligned16(sfa) || !aligned16(s_x) || (ldx % 8) != 0 ||
      (w->rank > 0 && !aligned16(Z)))
    return SVDQ_ERR_ALIGNMENT;
  return from_launch(svdq::launch_act_quant_nvfp4(w, M, X, ldx, xq, sfa, s_x, Z, stream));
}

svdq_status svdq_linear_nvfp4(const svdq_weights* w, int M, const uint8_t* xq, const uint8_t* sfa,
                              const float* s_x, const uint16_t* Z, uint16_t* Y, int ldy,
                              int epilogue, cudaStream_t stream) {
  svdq_status s = check_handle_nvfp4(w);
  if (s != SVDQ_OK) return s;
  if (M < 0 || ldy < w->N) return SVDQ_ERR_SHAPE;
  if (epilogue != SVDQ_EPI_NONE && epilogue != SVDQ_EPI_GELU) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!xq || !sfa || !s_x || !Y || (w->rank > 0 && !Z)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(sfa) || !aligned16(s_x) || !aligned16(Y) || (ldy % 8) != 0 ||
      (w->rank > 0 && !aligned16(Z)))
    return SVDQ_ERR_ALIGNMENT;
  return from_launch(svdq::launch_linear_nvfp4(w, M, xq, sfa, s_x, Z, Y, ldy, epilogue, stream));
}

}  // extern "C"
