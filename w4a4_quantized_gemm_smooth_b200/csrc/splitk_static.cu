// svdq_linear_splitk_noalloc: the split-K GEMM with its scratch (arrival
// counters and fp32 partial tiles) in a fixed device array of this library,
// so that a call allocates nothing.  The SVDQuant pages have no counterpart;
// this is an interface for allocation-free callers (e.g. inside a captured
// CUDA graph after the first call).
#include <mutex>

#include "svdq_internal.h"

namespace {

// Scratch for the split-K partial tiles: 16 MiB per device.  An explicit
// split count whose partial tiles need more is rejected; the automatic split
// is lowered until its tiles fit (e.g. M = 256, K = 4608, N = 1152 keeps its
// 8 ranges, 9.4 MB; M = 256, K = 15360, N = 3072 needs 18.9 MB at 6 ranges
// and runs at 5, 15.7 MB).
constexpr size_t kScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_splitk_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (the lookup may load the module onto the device, so the first call
// on a device must not be inside a stream capture).
svdq_status scratch_address(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return SVDQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[device]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_splitk_scratch);
    if (e != cudaSuccess || !p) return SVDQ_ERR_CUDA;
    g_scratch_addr[device] = p;
  }
  *out = g_scratch_addr[device];
  return SVDQ_OK;
}

}  // namespace

extern "C" {

svdq_status svdq_linear_splitk_noalloc(const svdq_weights* w, int M, const uint8_t* xq,
                                       const float* s_x, const uint16_t* Z, uint16_t* Y,
                                       int ldy, int epilogue, int splits,
                                       cudaStream_t stream) {
  svdq_status s = svdq::check_linear(w, M, xq, s_x, Z, Y, ldy, epilogue);
  if (s != SVDQ_OK || M == 0) return s;
  int sp = svdq::resolve_splits(w, M, splits);
  if (sp < 1) return SVDQ_ERR_INVALID_ARG;
  if (splits == 0)          // automatic: the largest split up to the choice that fits
    while (sp > 1 && svdq::splitk_workspace(w, M, sp) > kScratchBytes) --sp;
  if (sp > 1 && svdq::splitk_workspace(w, M, sp) > kScratchBytes) return SVDQ_ERR_SHAPE;
  void* scratch = nullptr;
  if ((s = scratch_address(w->device, &scratch)) != SVDQ_OK) return s;
  // launch_linear_splitk clears the arrival counters on `stream` first
  const cudaError_t e =
      svdq::launch_linear_splitk(w, M, xq, s_x, Z, Y, ldy, epilogue, sp, scratch, stream);
  return e == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

}  // extern "C"
