// patch_check_weight: device-side check of a packed weight's descriptor table
// against the packed format's rules, so that a weight from an untrusted
// source (a file, another process) can be refused before a GEMM indexes
// memory with it.  The debug build of the library runs it before every GEMM.
//
// Rules (the packed format of "PATCH: Learnable Tile-level Hybrid Sparsity for
// LLMs", section 2 "Core Mechanism": dense tiles stored whole, 2:4 tiles as
// their kept half plus 2-bit positions): tiles in row-major order; tile t's
// kind is 0 (dense) or 1 (sparse); a sparse tile's ordinal is the number of
// sparse tiles before it, a dense tile's is 0xFFFFFFFF; its values offset is
// the sum of the sizes of the tiles before it (32 KiB dense, 16 KiB sparse);
// the table holds exactly n_sparse sparse tiles.  Any violation ORs
// PATCH_DEV_BOUNDS into the status word.
#include "common.cuh"
#include "kernels.cuh"

namespace patch {

constexpr int kCheckThreads = 1024;

__global__ void __launch_bounds__(kCheckThreads) check_weight_kernel(const patch_tile_desc* __restrict__ desc,
                                                                      int64_t T, int64_t n_sparse,
                                                                      int32_t* status) {
  __shared__ int64_t scan_sparse[kCheckThreads], scan_bytes[kCheckThreads];
  const int i = threadIdx.x;
  const int64_t per = (T + kCheckThreads - 1) / kCheckThreads;
  const int64_t t0 = int64_t(i) * per, t1 = t0 + per < T ? t0 + per : T;
  // pass 1: this thread's sparse tiles and bytes
  int64_t ns = 0, bytes = 0;
  for (int64_t t = t0; t < t1; ++t) {
    const uint32_t kind = desc[t].kind;
    ns += kind == 1;
    bytes += kind == 1 ? PATCH_SPARSE_TILE_BYTES : PATCH_DENSE_TILE_BYTES;
  }
  scan_sparse[i] = ns;
  scan_bytes[i] = bytes;
  __syncthreads();
  // inclusive scan over the threads (Hillis-Steele)
  for (int off = 1; off < kCheckThreads; off <<= 1) {
    const int64_t a = i >= off ? scan_sparse[i - off] : 0, b = i >= off ? scan_bytes[i - off] : 0;
    __syncthreads();
    scan_sparse[i] += a;
    scan_bytes[i] += b;
    __syncthreads();
  }
  // pass 2: every tile against the prefix before it
  int64_t before_sparse = i ? scan_sparse[i - 1] : 0, before_bytes = i ? scan_bytes[i - 1] : 0;
  bool bad = false;
  for (int64_t t = t0; t < t1; ++t) {
    const patch_tile_desc d = desc[t];
    if (d.kind > 1) bad = true;
    if (d.kind == 1 ? d.sparse_ordinal != uint64_t(before_sparse) : d.sparse_ordinal != 0xFFFFFFFFu) bad = true;
    if (d.val_offset != uint64_t(before_bytes)) bad = true;
    before_sparse += d.kind == 1;
    before_bytes += d.kind == 1 ? PATCH_SPARSE_TILE_BYTES : PATCH_DENSE_TILE_BYTES;
  }
  if (i == kCheckThreads - 1 && scan_sparse[i] != n_sparse) bad = true;
  if (bad) set_status(status, PATCH_DEV_BOUNDS);
}

cudaError_t launch_check_weight(const patch_weight& W, int32_t* status, cudaStream_t stream) {
  const int64_t T = (W.N / kTile) * (W.K / kTile);
  check_weight_kernel<<<1, kCheckThreads, 0, stream>>>(W.desc, T, W.n_sparse, status);
  return cudaGetLastError();
}

}  // namespace patch
