// C ABI of libpatch: argument checks, path dispatch, status handling.
// Every entry point is declared and documented in include/patch.h.
#include <cuda_runtime.h>

#include <vector>

#include "common.cuh"
#include "kernels.cuh"

namespace patch {

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool shape_ok(int64_t N, int64_t K) {
  return N > 0 && K > 0 && N % kTile == 0 && K % kTile == 0 && N <= (int64_t(1) << 31) &&
         K <= (int64_t(1) << 31);
}

// SM count of the current device; PATCH_ERR_DEVICE unless it is compute capability 10.x
static patch_status_t device_sms(int* sms) {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PATCH_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return PATCH_ERR_CUDA;
  if (major != 10) return PATCH_ERR_DEVICE;
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return PATCH_ERR_CUDA;
  return PATCH_OK;
}

static patch_status_t check_weight(const patch_weight* W) {
  if (!W || !W->values || !W->desc) return PATCH_ERR_INVALID_ARG;
  if (!shape_ok(W->N, W->K)) return PATCH_ERR_SHAPE;
  const int64_t T = (W->N / kTile) * (W->K / kTile);
  if (W->n_sparse < 0 || W->n_sparse > T) return PATCH_ERR_INVALID_ARG;
  if (W->n_sparse > 0 && !W->meta) return PATCH_ERR_INVALID_ARG;
  if (!aligned16(W->values) || !aligned16(W->desc) || (W->meta && !aligned16(W->meta)))
    return PATCH_ERR_ALIGN;
  return PATCH_OK;
}

#ifdef PATCH_DEBUG
// Debug build: check a weight on the device before a GEMM indexes memory with
// it; synchronises the stream and refuses the call when the check fails.
static patch_status_t debug_check(const patch_weight* W, int32_t* status, void* stream) {
  if (!status) return PATCH_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (launch_check_weight(*W, status, s) != cudaSuccess) return PATCH_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PATCH_ERR_CUDA;
  int32_t bits = 0;
  if (cudaMemcpy(&bits, status, sizeof bits, cudaMemcpyDeviceToHost) != cudaSuccess) return PATCH_ERR_CUDA;
  return (bits & PATCH_DEV_BOUNDS) ? PATCH_ERR_BOUNDS : PATCH_OK;
}
#define PATCH_DEBUG_CHECK(W, status, stream)           \
  do {                                                 \
    patch_status_t dbg_ = debug_check(W, status, stream); \
    if (dbg_ != PATCH_OK) return dbg_;                 \
  } while (0)
#else
#define PATCH_DEBUG_CHECK(W, status, stream) \
  do {                                       \
  } while (0)
#endif

}  // namespace patch

using namespace patch;

extern "C" {

#ifdef PATCH_DEBUG
const char* patch_version(void) { return "patch-b200 0.2 (sm_100a, debug: weights checked before every GEMM)"; }
#else
const char* patch_version(void) { return "patch-b200 0.2 (sm_100a)"; }
#endif

const char* patch_strerror(patch_status_t s) {
  switch (s) {
    case PATCH_OK: return "ok";
    case PATCH_ERR_INVALID_ARG: return "invalid argument";
    case PATCH_ERR_SHAPE: return "N and K must be positive multiples of 128";
    case PATCH_ERR_ALIGN: return "pointer not 16-byte aligned";
    case PATCH_ERR_DEVICE: return "current device is not an sm_100 (B200-class) GPU";
    case PATCH_ERR_CUDA: return "CUDA call failed";
    case PATCH_ERR_BAD_PATTERN: return "pattern id > 5 inside a sparse tile";
    case PATCH_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case PATCH_ERR_WORKSPACE: return "workspace missing or too small";
    case PATCH_ERR_COUNT: return "bitmap's sparse-tile count differs from n_sparse";
    case PATCH_ERR_BOUNDS: return "packed weight breaks the format (descriptor table)";
  }
  return "unknown status";
}

patch_status_t patch_pack_sizes(int64_t N, int64_t K, int64_t n_sparse, size_t* values_bytes,
                                size_t* meta_bytes, size_t* desc_bytes) {
  if (!values_bytes || !meta_bytes || !desc_bytes) return PATCH_ERR_INVALID_ARG;
  if (!shape_ok(N, K)) return PATCH_ERR_SHAPE;
  const int64_t T = (N / kTile) * (K / kTile);
  if (n_sparse < 0 || n_sparse > T) return PATCH_ERR_INVALID_ARG;
  *values_bytes = size_t(T - n_sparse) * PATCH_DENSE_TILE_BYTES + size_t(n_sparse) * PATCH_SPARSE_TILE_BYTES;
  *meta_bytes = size_t(n_sparse) * PATCH_META_TILE_BYTES;
  *desc_bytes = size_t(T) * sizeof(patch_tile_desc);
  return PATCH_OK;
}

patch_status_t patch_hard_mask(const uint16_t* W, int64_t N, int64_t K, const float* tile_logits,
                               const float* pattern_logits, uint16_t* W_masked, uint8_t* bitmap,
                               uint8_t* pat_id, int32_t* dev_status, void* stream) {
  if (!tile_logits || !pattern_logits || !bitmap || !pat_id || !dev_status) return PATCH_ERR_INVALID_ARG;
  if (W_masked && !W) return PATCH_ERR_INVALID_ARG;
  if (!shape_ok(N, K)) return PATCH_ERR_SHAPE;
  if ((W && !aligned16(W)) || (W_masked && !aligned16(W_masked)) || !aligned16(pattern_logits) ||
      !aligned16(pat_id))
    return PATCH_ERR_ALIGN;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  if (launch_hard_mask(W, N, K, tile_logits, pattern_logits, W_masked, bitmap, pat_id, sms,
                       static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PATCH_ERR_CUDA;
  return PATCH_OK;
}

static bool mask_tile_ok(int64_t b) { return b == 4 || b == 8 || b == 16 || b == 32 || b == 64 || b == 128; }

patch_status_t patch_hard_mask_tiles(const uint16_t* W, int64_t N, int64_t K, int64_t mask_tile,
                                     const float* tile_logits, const float* pattern_logits, uint16_t* W_masked,
                                     uint8_t* bitmap, uint8_t* pat_id, int32_t* dev_status, void* stream) {
  if (!tile_logits || !pattern_logits || !bitmap || !pat_id || !dev_status) return PATCH_ERR_INVALID_ARG;
  if (W_masked && !W) return PATCH_ERR_INVALID_ARG;
  if (!mask_tile_ok(mask_tile)) return PATCH_ERR_INVALID_ARG;
  if (!shape_ok(N, K)) return PATCH_ERR_SHAPE;
  if ((W && !aligned16(W)) || (W_masked && !aligned16(W_masked)) || !aligned16(pattern_logits) ||
      !aligned16(pat_id) || reinterpret_cast<uintptr_t>(tile_logits) % 8)
    return PATCH_ERR_ALIGN;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  if (launch_hard_mask_tiles(W, N, K, mask_tile, tile_logits, pattern_logits, W_masked, bitmap, pat_id, sms,
                             static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PATCH_ERR_CUDA;
  return PATCH_OK;
}

patch_status_t patch_exec_tiles(const uint8_t* bitmap, int64_t N, int64_t K, int64_t mask_tile, uint8_t* exec,
                                int64_t* n_sparse, void* stream) {
  if (!bitmap || !exec || !n_sparse) return PATCH_ERR_INVALID_ARG;
  if (!mask_tile_ok(mask_tile)) return PATCH_ERR_INVALID_ARG;
  if (!shape_ok(N, K)) return PATCH_ERR_SHAPE;
  if (reinterpret_cast<uintptr_t>(n_sparse) % 8) return PATCH_ERR_ALIGN;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  if (launch_exec_tiles(bitmap, N, K, mask_tile, kTile, exec, n_sparse, sms, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return PATCH_ERR_CUDA;
  return PATCH_OK;
}

patch_status_t patch_pack(const uint16_t* W, int64_t N, int64_t K, const uint8_t* bitmap,
                          const uint8_t* pat_id, int64_t n_sparse, void* values, void* meta,
                          patch_tile_desc* desc, int32_t* dev_status, void* stream) {
  if (!W || !bitmap || !pat_id || !values || !desc || !dev_status) return PATCH_ERR_INVALID_ARG;
  if (!shape_ok(N, K)) return PATCH_ERR_SHAPE;
  const int64_t T = (N / kTile) * (K / kTile);
  if (n_sparse < 0 || n_sparse > T) return PATCH_ERR_INVALID_ARG;
  if (n_sparse > 0 && !meta) return PATCH_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(values) || !aligned16(desc) || (meta && !aligned16(meta)))
    return PATCH_ERR_ALIGN;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  if (launch_pack(W, N, K, bitmap, pat_id, nullptr, n_sparse, values, meta, desc, dev_status, sms,
                  static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PATCH_ERR_CUDA;
  return PATCH_OK;
}

patch_status_t patch_soft_mask(const uint16_t* W, int64_t N, int64_t K, const float* tile_logits,
                               const float* tile_noise, const float* pattern_logits, const float* pattern_noise,
                               float tau, uint16_t* W_soft, float* mask, void* stream) {
  if (!W || !tile_logits || !pattern_logits || !W_soft) return PATCH_ERR_INVALID_ARG;
  if (!(tau > 0.0f) || !(tau < 3.0e38f)) return PATCH_ERR_INVALID_ARG;  // positive and finite
  if (!shape_ok(N, K)) return PATCH_ERR_SHAPE;
  auto a8 = [](const void* q) { return reinterpret_cast<uintptr_t>(q) % 8 == 0; };
  if (!aligned16(W) || !aligned16(pattern_logits) || (pattern_noise && !aligned16(pattern_noise)) ||
      !aligned16(W_soft) || (mask && !aligned16(mask)) || !a8(tile_logits) || (tile_noise && !a8(tile_noise)))
    return PATCH_ERR_ALIGN;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  if (launch_soft_mask(W, N, K, tile_logits, tile_noise, pattern_logits, pattern_noise, tau, W_soft, mask, sms,
                       static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PATCH_ERR_CUDA;
  return PATCH_OK;
}

patch_status_t patch_tile_kinds(const float* tile_logits, int64_t N, int64_t K, uint8_t* bitmap,
                                int64_t* n_sparse, void* stream) {
  if (!tile_logits || !bitmap || !n_sparse) return PATCH_ERR_INVALID_ARG;
  if (!shape_ok(N, K)) return PATCH_ERR_SHAPE;
  if (reinterpret_cast<uintptr_t>(tile_logits) % 8 || reinterpret_cast<uintptr_t>(n_sparse) % 8)
    return PATCH_ERR_ALIGN;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  if (launch_tile_kinds(tile_logits, N, K, bitmap, n_sparse, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PATCH_ERR_CUDA;
  return PATCH_OK;
}

patch_status_t patch_pack_from_logits(const uint16_t* W, int64_t N, int64_t K, const uint8_t* bitmap,
                                      const float* pattern_logits, int64_t n_sparse, void* values, void* meta,
                                      patch_tile_desc* desc, int32_t* dev_status, void* stream) {
  if (!W || !bitmap || !pattern_logits || !values || !desc || !dev_status) return PATCH_ERR_INVALID_ARG;
  if (!shape_ok(N, K)) return PATCH_ERR_SHAPE;
  const int64_t T = (N / kTile) * (K / kTile);
  if (n_sparse < 0 || n_sparse > T) return PATCH_ERR_INVALID_ARG;
  if (n_sparse > 0 && !meta) return PATCH_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(pattern_logits) || !aligned16(values) || !aligned16(desc) ||
      (meta && !aligned16(meta)))
    return PATCH_ERR_ALIGN;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  if (launch_pack(W, N, K, bitmap, nullptr, pattern_logits, n_sparse, values, meta, desc, dev_status, sms,
                  static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PATCH_ERR_CUDA;
  return PATCH_OK;
}

patch_status_t patch_gemm_workspace_size(int64_t M, const patch_weight* W, size_t* bytes) {
  if (!bytes || !W || M < 0) return PATCH_ERR_INVALID_ARG;
  if (!shape_ok(W->N, W->K)) return PATCH_ERR_SHAPE;
  const int64_t T = (W->N / kTile) * (W->K / kTile);
  if (W->n_sparse < 0 || W->n_sparse > T) return PATCH_ERR_INVALID_ARG;
  *bytes = 0;
  if (M == 0) return PATCH_OK;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  // enough for every path M can take: the counter region, then that path's scratch
  const size_t pf = prefill_workspace_bytes(M, *W, sms);
  if (M > PATCH_DECODE_MAX_M) {
    *bytes = pf;
    return PATCH_OK;
  }
  const size_t tc = W->N / kTile <= kDecodeMaxTileRows ? decode_tc_workspace_bytes(M, *W, sms) : 0;
  const size_t simt = kDecodeCounterBytes + decode_plan(M, W->N, W->K, sms).ws_bytes;
  size_t b = tc > simt ? tc : simt;
  *bytes = b > pf ? b : pf;
  return PATCH_OK;
}

patch_status_t patch_gemm_ex(const uint16_t* X, int64_t M, const patch_weight* W, uint16_t* Y,
                             void* workspace, size_t workspace_bytes, int32_t* dev_status,
                             void* stream, int path, uint64_t wait_limit_us) {
  if (M < 0 || !dev_status) return PATCH_ERR_INVALID_ARG;
  const int inject = (path & PATCH_PATH_TEST_STALL) ? 1 : 0;
  path &= ~PATCH_PATH_TEST_STALL;
  if (inject && path != PATCH_PATH_PREFILL) return PATCH_ERR_INVALID_ARG;
  patch_status_t st = check_weight(W);
  if (st != PATCH_OK) return st;
  if (path == PATCH_PATH_AUTO)  // tensor-core decode up to kDecodeMaxTileRows tile rows, CUDA-core beyond
    path = M > PATCH_DECODE_MAX_M ? PATCH_PATH_PREFILL
                                  : (W->N / kTile <= kDecodeMaxTileRows ? PATCH_PATH_DECODE : PATCH_PATH_DECODE_SIMT);
  if (path != PATCH_PATH_DECODE && path != PATCH_PATH_PREFILL && path != PATCH_PATH_DECODE_SIMT)
    return PATCH_ERR_INVALID_ARG;
  if (path != PATCH_PATH_PREFILL && M > PATCH_DECODE_MAX_M) return PATCH_ERR_INVALID_ARG;
  if (path == PATCH_PATH_DECODE && W->N / kTile > kDecodeMaxTileRows) return PATCH_ERR_SHAPE;
  if (M == 0) return PATCH_OK;
  if (!X || !Y) return PATCH_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y)) return PATCH_ERR_ALIGN;
  if (M > (int64_t(1) << 30)) return PATCH_ERR_INVALID_ARG;
  int sms = 0;
  st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  PATCH_DEBUG_CHECK(W, dev_status, stream);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint64_t limit_ns = (wait_limit_us ? wait_limit_us : 2000000ull) * 1000ull;
  cudaError_t e;
  if (path == PATCH_PATH_DECODE) {
    const size_t need = decode_tc_workspace_bytes(M, *W, sms);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PATCH_ERR_WORKSPACE;
    e = launch_decode_tc(X, M, *W, Y, workspace, dev_status, sms, limit_ns, s);
  } else if (path == PATCH_PATH_DECODE_SIMT) {
    const DecodePlan p = decode_plan(M, W->N, W->K, sms);
    if (p.ws_bytes > 0 &&
        (!workspace || workspace_bytes < kDecodeCounterBytes + p.ws_bytes || !aligned16(workspace)))
      return PATCH_ERR_WORKSPACE;
    // its scratch follows the tensor-core kernel's counter region, which it leaves untouched
    void* scratch = p.ws_bytes > 0 ? static_cast<uint8_t*>(workspace) + kDecodeCounterBytes : nullptr;
    e = launch_decode(X, M, *W, Y, scratch, sms, s);
  } else {
    // the split-K mode uses the workspace only when it is there, aligned and big enough
    void* ws = workspace && aligned16(workspace) ? workspace : nullptr;
    e = launch_prefill(X, M, *W, Y, ws, ws ? workspace_bytes : 0, dev_status, sms, limit_ns, inject, s);
  }
  return e == cudaSuccess ? PATCH_OK : PATCH_ERR_CUDA;
}

patch_status_t patch_gemm(const uint16_t* X, int64_t M, const patch_weight* W, uint16_t* Y,
                          void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  return patch_gemm_ex(X, M, W, Y, workspace, workspace_bytes, dev_status, stream, PATCH_PATH_AUTO, 0);
}

// Checks of one chain call; M == 0 calls are valid and skipped.
static patch_status_t check_chain_call(const patch_chain_call& c) {
  if (c.M < 0 || c.M > PATCH_DECODE_MAX_M) return PATCH_ERR_INVALID_ARG;
  patch_status_t st = check_weight(&c.W);
  if (st != PATCH_OK) return st;
  if (c.W.N / kTile > kChainMaxTileRows) return PATCH_ERR_SHAPE;
  if (c.M == 0) return PATCH_OK;
  if (!c.X || !c.Y) return PATCH_ERR_INVALID_ARG;
  if (!aligned16(c.X) || !aligned16(c.Y)) return PATCH_ERR_ALIGN;
  return PATCH_OK;
}

// The calls that do work (M > 0), in order.
static patch_status_t chain_calls(const patch_chain_call* calls, int64_t n, std::vector<patch_chain_call>& out) {
  if (n < 0 || (n > 0 && !calls)) return PATCH_ERR_INVALID_ARG;
  out.clear();
  for (int64_t j = 0; j < n; ++j) {
    patch_status_t st = check_chain_call(calls[j]);
    if (st != PATCH_OK) return st;
    if (calls[j].M > 0) out.push_back(calls[j]);
  }
  return PATCH_OK;
}

patch_status_t patch_gemm_chain_workspace_size(const patch_chain_call* calls, int64_t n_calls, size_t* bytes) {
  if (!bytes) return PATCH_ERR_INVALID_ARG;
  std::vector<patch_chain_call> cs;
  patch_status_t st = chain_calls(calls, n_calls, cs);
  if (st != PATCH_OK) return st;
  *bytes = 0;
  if (cs.empty()) return PATCH_OK;
  int sms = 0;
  st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  *bytes = chain_workspace_bytes(cs.data(), int64_t(cs.size()), sms);
  return PATCH_OK;
}

patch_status_t patch_gemm_chain(const patch_chain_call* calls, int64_t n_calls, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, void* stream, uint64_t wait_limit_us) {
  if (!dev_status) return PATCH_ERR_INVALID_ARG;
  std::vector<patch_chain_call> cs;
  patch_status_t st = chain_calls(calls, n_calls, cs);
  if (st != PATCH_OK) return st;
  if (cs.empty()) return PATCH_OK;
  int sms = 0;
  st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  const int64_t n = int64_t(cs.size());
  if (!workspace || !aligned16(workspace) || workspace_bytes < chain_workspace_bytes(cs.data(), n, sms))
    return PATCH_ERR_WORKSPACE;
  for (int64_t j = 0; j < n; ++j) PATCH_DEBUG_CHECK(&cs[j].W, dev_status, stream);
  const uint64_t limit_ns = (wait_limit_us ? wait_limit_us : 2000000ull) * 1000ull;
  for (int64_t j0 = 0; j0 < n;) {
    const int64_t j1 = chain_launch_end(cs.data(), j0, n);
    if (launch_chain(cs.data(), j0, j1, workspace, dev_status, sms, limit_ns, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
      return PATCH_ERR_CUDA;
    j0 = j1;
  }
  return PATCH_OK;
}

patch_status_t patch_gemm_group(const patch_chain_call* calls, int64_t n_calls, int32_t* dev_status, void* stream,
                                uint64_t wait_limit_us) {
  if (!dev_status || n_calls < 0 || (n_calls > 0 && !calls)) return PATCH_ERR_INVALID_ARG;
  std::vector<PrefillGroupCall> cs;
  for (int64_t j = 0; j < n_calls; ++j) {
    const patch_chain_call& c = calls[j];
    if (c.M < 0 || c.M > (int64_t(1) << 30) || c.after_previous != 0) return PATCH_ERR_INVALID_ARG;
    patch_status_t st = check_weight(&c.W);
    if (st != PATCH_OK) return st;
    if (c.M == 0) continue;
    if (!c.X || !c.Y) return PATCH_ERR_INVALID_ARG;
    if (!aligned16(c.X) || !aligned16(c.Y)) return PATCH_ERR_ALIGN;
    cs.push_back(PrefillGroupCall{c.X, c.M, c.W, c.Y});
  }
  if (cs.empty()) return PATCH_OK;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  for (const PrefillGroupCall& c : cs) PATCH_DEBUG_CHECK(&c.W, dev_status, stream);
  const uint64_t limit_ns = (wait_limit_us ? wait_limit_us : 2000000ull) * 1000ull;
  const int n = int(cs.size());
  for (int j0 = 0; j0 < n; j0 += kPrefillGroupMax) {
    const int cnt = n - j0 < kPrefillGroupMax ? n - j0 : kPrefillGroupMax;
    if (launch_prefill_group(cs.data() + j0, cnt, dev_status, sms, limit_ns, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
      return PATCH_ERR_CUDA;
  }
  return PATCH_OK;
}

// decode scratch for the gated MLP: [decode GEMM workspace][G][U], 256-byte aligned parts
static size_t round256(size_t b) { return (b + 255) & ~size_t(255); }

patch_status_t patch_gemm_mlp_workspace_size(int64_t M, const patch_weight* W_gate, const patch_weight* W_up,
                                             size_t* bytes) {
  if (!bytes || !W_gate || !W_up) return PATCH_ERR_INVALID_ARG;
  if (W_gate->N != W_up->N || W_gate->K != W_up->K) return PATCH_ERR_SHAPE;
  size_t a = 0, b = 0;
  patch_status_t st = patch_gemm_workspace_size(M, W_gate, &a);
  if (st != PATCH_OK) return st;
  st = patch_gemm_workspace_size(M, W_up, &b);
  if (st != PATCH_OK) return st;
  *bytes = 0;
  if (M == 0 || M > PATCH_DECODE_MAX_M) return PATCH_OK;
  *bytes = round256(a > b ? a : b) + 2 * round256(size_t(M) * size_t(W_gate->N) * 2);
  return PATCH_OK;
}

patch_status_t patch_gemm_mlp(const uint16_t* X, int64_t M, const patch_weight* W_gate, const patch_weight* W_up,
                              uint16_t* H, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                              void* stream) {
  if (M < 0 || !dev_status || !W_gate || !W_up) return PATCH_ERR_INVALID_ARG;
  if (W_gate->N != W_up->N || W_gate->K != W_up->K) return PATCH_ERR_SHAPE;
  patch_status_t st = check_weight(W_gate);
  if (st != PATCH_OK) return st;
  st = check_weight(W_up);
  if (st != PATCH_OK) return st;
  if (M == 0) return PATCH_OK;
  if (!X || !H) return PATCH_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(H)) return PATCH_ERR_ALIGN;
  int sms = 0;
  st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  PATCH_DEBUG_CHECK(W_gate, dev_status, stream);
  PATCH_DEBUG_CHECK(W_up, dev_status, stream);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint64_t limit_ns = 2000000ull * 1000ull;
  if (M > PATCH_DECODE_MAX_M) {
    if (launch_prefill_mlp(X, M, *W_gate, *W_up, H, dev_status, sms, limit_ns, s) != cudaSuccess)
      return PATCH_ERR_CUDA;
    return PATCH_OK;
  }
  size_t need = 0;
  st = patch_gemm_mlp_workspace_size(M, W_gate, W_up, &need);
  if (st != PATCH_OK) return st;
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PATCH_ERR_WORKSPACE;
  size_t ws = 0;
  patch_gemm_workspace_size(M, W_gate, &ws);
  size_t wu = 0;
  patch_gemm_workspace_size(M, W_up, &wu);
  const size_t gemm_ws = round256(ws > wu ? ws : wu), yb = round256(size_t(M) * size_t(W_gate->N) * 2);
  uint16_t* G = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + gemm_ws);
  uint16_t* U = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + gemm_ws + yb);
  st = patch_gemm(X, M, W_gate, G, workspace, gemm_ws, dev_status, stream);
  if (st != PATCH_OK) return st;
  st = patch_gemm(X, M, W_up, U, workspace, gemm_ws, dev_status, stream);
  if (st != PATCH_OK) return st;
  if (launch_silu_mul(G, U, H, M * W_gate->N, sms, s) != cudaSuccess) return PATCH_ERR_CUDA;
  return PATCH_OK;
}

// Weight of tile row r under a shard balance: stored bytes (decode streams
// them) or the tensor cores' MMA work in units of a sparse tile's (prefill:
// a dense tile does 2, a sparse tile 1).
static int64_t row_weight(const uint8_t* bitmap, int64_t r, int64_t Tk, int64_t by) {
  int64_t w = by == PATCH_SHARD_BY_FLOPS ? 0 : 16 * Tk;
  for (int64_t k = 0; k < Tk; ++k) {
    const bool sparse = bitmap[r * Tk + k] != 0;
    if (by == PATCH_SHARD_BY_FLOPS)
      w += sparse ? 1 : 2;
    else
      w += sparse ? int64_t(PATCH_SPARSE_TILE_BYTES + PATCH_META_TILE_BYTES) : int64_t(PATCH_DENSE_TILE_BYTES);
  }
  return w;
}

patch_status_t patch_shard_rows_by(const uint8_t* bitmap, int64_t Tn, int64_t Tk, int64_t n_shards, int64_t by,
                                   int64_t* row_begin) {
  if (!bitmap || !row_begin || Tn < 1 || Tk < 1 || n_shards < 1 || n_shards > Tn) return PATCH_ERR_INVALID_ARG;
  if (by != PATCH_SHARD_BY_BYTES && by != PATCH_SHARD_BY_FLOPS) return PATCH_ERR_INVALID_ARG;
  int64_t total = 0;
  for (int64_t r = 0; r < Tn; ++r) total += row_weight(bitmap, r, Tk, by);
  row_begin[0] = 0;
  int64_t r = 0, before = 0;  // rows [0, r) weigh `before`
  for (int64_t i = 1; i < n_shards; ++i) {
    // first row whose prefix reaches i / n of the total (compared without rounding)
    while (r < Tn && before * n_shards < i * total) {
      before += row_weight(bitmap, r, Tk, by);
      ++r;
    }
    // strictly increasing, and leave at least one row for each later shard
    int64_t v = r;
    if (v <= row_begin[i - 1]) v = row_begin[i - 1] + 1;
    if (v > Tn - (n_shards - i)) v = Tn - (n_shards - i);
    row_begin[i] = v;
  }
  row_begin[n_shards] = Tn;
  return PATCH_OK;
}

patch_status_t patch_shard_rows(const uint8_t* bitmap, int64_t Tn, int64_t Tk, int64_t n_shards,
                                int64_t* row_begin) {
  return patch_shard_rows_by(bitmap, Tn, Tk, n_shards, PATCH_SHARD_BY_BYTES, row_begin);
}

patch_status_t patch_mma_probe_m(int m, int sparse, int64_t iters, int32_t* dev_status, void* stream) {
  if (iters < 1 || !dev_status || (m != 64 && m != 128)) return PATCH_ERR_INVALID_ARG;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  return launch_mma_probe(m, sparse ? 1 : 0, iters, sms, 2000000000ull, dev_status,
                          static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PATCH_OK
             : PATCH_ERR_CUDA;
}

patch_status_t patch_mma_probe(int sparse, int64_t iters, int32_t* dev_status, void* stream) {
  return patch_mma_probe_m(128, sparse, iters, dev_status, stream);
}

// ---- the 64 x 64 execution-tile format

static bool shape64_ok(int64_t N, int64_t K) {
  return N > 0 && K > 0 && N % 64 == 0 && K % 64 == 0 && N <= (int64_t(1) << 31) && K <= (int64_t(1) << 31);
}

static patch_status_t check_weight64(const patch_weight64* W) {
  if (!W || !W->values || !W->desc) return PATCH_ERR_INVALID_ARG;
  if (!shape64_ok(W->N, W->K)) return PATCH_ERR_SHAPE;
  const int64_t T = (W->N / 64) * (W->K / 64);
  if (W->n_sparse < 0 || W->n_sparse > T) return PATCH_ERR_INVALID_ARG;
  if (W->n_sparse > 0 && !W->meta) return PATCH_ERR_INVALID_ARG;
  if (!aligned16(W->values) || !aligned16(W->desc) || (W->meta && !aligned16(W->meta))) return PATCH_ERR_ALIGN;
  return PATCH_OK;
}

patch_status_t patch_pack64_sizes(int64_t N, int64_t K, int64_t n_sparse, size_t* values_bytes, size_t* meta_bytes,
                                  size_t* desc_bytes) {
  if (!values_bytes || !meta_bytes || !desc_bytes) return PATCH_ERR_INVALID_ARG;
  if (!shape64_ok(N, K)) return PATCH_ERR_SHAPE;
  const int64_t T = (N / 64) * (K / 64);
  if (n_sparse < 0 || n_sparse > T) return PATCH_ERR_INVALID_ARG;
  *values_bytes = size_t(T - n_sparse) * PATCH_DENSE_TILE64_BYTES + size_t(n_sparse) * PATCH_SPARSE_TILE64_BYTES;
  *meta_bytes = size_t(n_sparse) * PATCH_META_TILE64_BYTES;
  *desc_bytes = size_t(T) * sizeof(patch_tile_desc);
  return PATCH_OK;
}

patch_status_t patch_exec_tiles64(const uint8_t* bitmap, int64_t N, int64_t K, int64_t mask_tile, uint8_t* exec,
                                  int64_t* n_sparse, void* stream) {
  if (!bitmap || !exec || !n_sparse) return PATCH_ERR_INVALID_ARG;
  if (mask_tile != 4 && mask_tile != 8 && mask_tile != 16 && mask_tile != 32 && mask_tile != 64)
    return PATCH_ERR_INVALID_ARG;
  if (!shape64_ok(N, K)) return PATCH_ERR_SHAPE;
  if (reinterpret_cast<uintptr_t>(n_sparse) % 8) return PATCH_ERR_ALIGN;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  if (launch_exec_tiles(bitmap, N, K, mask_tile, 64, exec, n_sparse, sms, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return PATCH_ERR_CUDA;
  return PATCH_OK;
}

patch_status_t patch_pack64(const uint16_t* W, int64_t N, int64_t K, const uint8_t* bitmap, const uint8_t* pat_id,
                            int64_t n_sparse, void* values, void* meta, patch_tile_desc* desc, int32_t* dev_status,
                            void* stream) {
  if (!W || !bitmap || !pat_id || !values || !desc || !dev_status) return PATCH_ERR_INVALID_ARG;
  if (!shape64_ok(N, K)) return PATCH_ERR_SHAPE;
  const int64_t T = (N / 64) * (K / 64);
  if (n_sparse < 0 || n_sparse > T) return PATCH_ERR_INVALID_ARG;
  if (n_sparse > 0 && !meta) return PATCH_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(pat_id) || !aligned16(values) || !aligned16(desc) || (meta && !aligned16(meta)))
    return PATCH_ERR_ALIGN;
  int sms = 0;
  patch_status_t st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  if (launch_pack64(W, N, K, bitmap, pat_id, n_sparse, values, meta, desc, dev_status, sms,
                    static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PATCH_ERR_CUDA;
  return PATCH_OK;
}

patch_status_t patch_gemm64_workspace_size(int64_t M, const patch_weight64* W, size_t* bytes) {
  if (!bytes || M < 0) return PATCH_ERR_INVALID_ARG;
  patch_status_t st = check_weight64(W);
  if (st != PATCH_OK) return st;
  *bytes = 0;
  if (M == 0) return PATCH_OK;
  if (M > (int64_t(1) << 30)) return PATCH_ERR_INVALID_ARG;
  int sms = 0;
  st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  *bytes = gemm64_workspace_bytes(M, *W, sms);
  return PATCH_OK;
}

patch_status_t patch_gemm64(const uint16_t* X, int64_t M, const patch_weight64* W, uint16_t* Y, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, void* stream, uint64_t wait_limit_us) {
  if (M < 0 || !dev_status) return PATCH_ERR_INVALID_ARG;
  patch_status_t st = check_weight64(W);
  if (st != PATCH_OK) return st;
  if (M == 0) return PATCH_OK;
  if (!X || !Y) return PATCH_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y)) return PATCH_ERR_ALIGN;
  if (M > (int64_t(1) << 30)) return PATCH_ERR_INVALID_ARG;
  int sms = 0;
  st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  const size_t need = gemm64_workspace_bytes(M, *W, sms);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PATCH_ERR_WORKSPACE;
  const uint64_t limit_ns = (wait_limit_us ? wait_limit_us : 2000000ull) * 1000ull;
  return launch_gemm64(X, M, *W, Y, workspace, dev_status, sms, limit_ns, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? PATCH_OK
             : PATCH_ERR_CUDA;
}

patch_status_t patch_check_weight(const patch_weight* W, int32_t* dev_status, void* stream) {
  if (!dev_status) return PATCH_ERR_INVALID_ARG;
  patch_status_t st = check_weight(W);
  if (st != PATCH_OK) return st;
  int sms = 0;
  st = device_sms(&sms);
  if (st != PATCH_OK) return st;
  return launch_check_weight(*W, dev_status, static_cast<cudaStream_t>(stream)) == cudaSuccess ? PATCH_OK
                                                                                                : PATCH_ERR_CUDA;
}

patch_status_t patch_read_status(const int32_t* dev_status, void* stream, int32_t* host_bits) {
  if (!dev_status) return PATCH_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return PATCH_ERR_CUDA;
  int32_t bits = 0;
  if (cudaMemcpy(&bits, dev_status, sizeof bits, cudaMemcpyDeviceToHost) != cudaSuccess) return PATCH_ERR_CUDA;
  if (host_bits) *host_bits = bits;
  if (bits & PATCH_DEV_TIMEOUT) return PATCH_ERR_TIMEOUT;
  if (bits & PATCH_DEV_BOUNDS) return PATCH_ERR_BOUNDS;
  if (bits & PATCH_DEV_BAD_PATTERN) return PATCH_ERR_BAD_PATTERN;
  if (bits & PATCH_DEV_COUNT) return PATCH_ERR_COUNT;
  return PATCH_OK;
}

}  // extern "C"
