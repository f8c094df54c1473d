// patch_gemm_decode_noalloc: the decode GEMM for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain scratch memory: a plugin running inside
// a host framework that owns the device memory pool and hands the plugin
// only its input and output buffers, or a latency-critical loop in which a
// cudaMalloc (which may synchronise the whole device) is not acceptable.
// This entry point runs the CUDA-core split-K decode kernels (the path
// patch_gemm_ex takes with PATCH_PATH_DECODE_SIMT, not patch_gemm's default
// tensor-core decode kernel), with their fp32 partial sums in a fixed buffer
// compiled into the library (below) instead of a caller-provided workspace.
// That path sets no device status bits, so dev_status may be NULL.
//
// The buffer is a file-scope __device__ array: every GPU that loads the
// library holds PATCH_NOALLOC_SCRATCH_BYTES of it until the process exits.
// In host code its name only stands in for the symbol; the device address is
// looked up with cudaGetSymbolAddress once per device (with that device
// current) on the first call made there, and that address is what the
// kernels receive.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace patch {
namespace {

static __device__ __align__(256) uint8_t noalloc_scratch[PATCH_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of noalloc_scratch on `dev` (the current device); nullptr on failure.
void* scratch_address(int dev) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace
}  // namespace patch

using namespace patch;

extern "C" patch_status_t patch_gemm_decode_noalloc(const uint16_t* X, int64_t M, const patch_weight* W,
                                                   uint16_t* Y, int32_t* dev_status, void* stream) {
  (void)dev_status;  // nothing on this path's kernels reports through the status word
  if (M < 0 || M > PATCH_DECODE_MAX_M || !W) return PATCH_ERR_INVALID_ARG;
  if (!W->values || !W->desc || (W->n_sparse > 0 && !W->meta)) return PATCH_ERR_INVALID_ARG;
  if (W->N <= 0 || W->K <= 0 || W->N % kTile || W->K % kTile) return PATCH_ERR_SHAPE;
  const int64_t T = (W->N / kTile) * (W->K / kTile);
  if (W->n_sparse < 0 || W->n_sparse > T) return PATCH_ERR_INVALID_ARG;
  if (M == 0) return PATCH_OK;
  if (!X || !Y) return PATCH_ERR_INVALID_ARG;
  const auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (misaligned(X) || misaligned(Y) || misaligned(W->values) || misaligned(W->desc) ||
      (W->meta && misaligned(W->meta)))
    return PATCH_ERR_ALIGN;

  int dev = 0, major = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PATCH_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return PATCH_ERR_CUDA;
  if (major != 10) return PATCH_ERR_DEVICE;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return PATCH_ERR_CUDA;

#ifdef PATCH_DEBUG
  // debug build: the weight is checked on the device (needs the status word) before use
  if (!dev_status) return PATCH_ERR_INVALID_ARG;
  {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (launch_check_weight(*W, dev_status, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
      return PATCH_ERR_CUDA;
    int32_t bits = 0;
    if (cudaMemcpy(&bits, dev_status, sizeof bits, cudaMemcpyDeviceToHost) != cudaSuccess) return PATCH_ERR_CUDA;
    if (bits & PATCH_DEV_BOUNDS) return PATCH_ERR_BOUNDS;
  }
#endif
  // the built-in buffer must hold the split-K partials of this problem
  const DecodePlan plan = decode_plan(M, W->N, W->K, sms);
  if (plan.ws_bytes > PATCH_NOALLOC_SCRATCH_BYTES) return PATCH_ERR_WORKSPACE;
  void* scratch = scratch_address(dev);
  if (!scratch) return PATCH_ERR_CUDA;
  // Each partial-sum slot is written by exactly one CTA before the reduce
  // kernel reads it, so nothing left by an earlier call needs clearing.
  return launch_decode(X, M, *W, Y, scratch, sms, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PATCH_OK
             : PATCH_ERR_CUDA;
}
