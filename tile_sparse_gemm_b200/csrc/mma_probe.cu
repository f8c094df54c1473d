// patch_mma_probe: the tensor-core MMA issue rate of this GPU for the two
// instruction forms the hybrid GEMM uses, dense kind::f16 and 2:4-sparse
// kind::f16 (.sp), measured on shared-memory operands so that no memory
// traffic limits it.  It gives the mixed roofline of the prefill path its
// sparse half: the rate of sparse tiles relative to dense ones, which the
// datasheet puts at 2x ("Inference & Deployment": sparse tiles run on the 2:4
// sparse tensor cores).
//
// One CTA per SM; its shared memory holds pseudo-random bf16 operands (so the
// datapath toggles as it does on real weights) and valid metadata codes.  One
// thread issues `iters` rounds of four M = 128 (or M = 64: the first 64 rows
// of the panel, the shape of 64 x 64 execution tiles), N = 240 MMAs (the
// prefill kernel's token block) into two alternating TMEM accumulators: dense
// rounds cover K = 64 (four K = 16 MMAs over one panel), sparse rounds K = 128
// logical (four K = 32 .sp MMAs over a panel of kept values and its
// metadata), so a sparse round does twice a dense round's dense-equivalent
// work.  The caller times the launch; FLOPs = SMs x iters x 4 x 2 x M x 240 x
// (16 dense, 32 sparse).  Every metadata column an MMA may read holds valid
// codes for both shapes (four columns x 128 lanes are copied).
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace patch {
namespace probe {

using namespace tc;

constexpr int N = 240;                 // MMA N (tokens)
constexpr int THREADS = 128;
constexpr uint32_t TMEM_COLS = 512;    // accumulators at columns 0 and 256, metadata at column N
constexpr uint32_t ACC1 = 256, META_COL = N;

struct Shared {
  alignas(1024) uint8_t a[PATCH_PANEL_BYTES];  // 128 x 64 bf16, 128-byte swizzled rows
  alignas(1024) uint8_t b[2][N * 64 * 2];      // two 64-k panels of 256 x 64 bf16
  alignas(128) uint8_t e[PATCH_META_TILE_BYTES];
  uint64_t done;
  uint32_t tmem_base;
};
constexpr size_t SMEM_BYTES = sizeof(Shared) + 1024;

__device__ __forceinline__ uint32_t hash32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7FEB352Du;
  x ^= x >> 15;
  x *= 0x846CA68Bu;
  x ^= x >> 16;
  return x;
}

// a bf16 in [-1, 1) from a hash (sign, exponent 119..126, random mantissa)
__device__ __forceinline__ uint16_t rand_bf16(uint32_t h) {
  return uint16_t(((h >> 31) << 15) | ((119u + (h >> 28 & 7u)) << 7) | (h & 0x7Fu));
}

__global__ void __launch_bounds__(THREADS, 1) probe_kernel(int m, int sparse, int64_t iters, uint64_t limit_ns,
                                                           int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  Shared& s = *reinterpret_cast<Shared*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const uint32_t seed = blockIdx.x * 0x9E3779B9u;
  uint16_t* a16 = reinterpret_cast<uint16_t*>(s.a);
  for (int i = threadIdx.x; i < PATCH_PANEL_BYTES / 2; i += THREADS) a16[i] = rand_bf16(hash32(seed + i));
  uint16_t* b16 = reinterpret_cast<uint16_t*>(s.b);
  for (int i = threadIdx.x; i < 2 * N * 64; i += THREADS) b16[i] = rand_bf16(hash32(seed ^ 0x55555555u) + i * 7u);
  for (int i = threadIdx.x; i < PATCH_META_TILE_BYTES; i += THREADS) {
    // two valid 4-bit codes per byte (ids 0..5 -> codes 4 8 C 9 D E)
    const uint32_t h = hash32(seed + 0x1234567u + i);
    s.e[i] = uint8_t(pattern_code(h % 6u) | (pattern_code((h >> 8) % 6u) << 4));
  }
  if (threadIdx.x == 0) {
    mbar_init(&s.done, 1);
    fence_barrier_init();
  }
  fence_proxy_async_smem();  // the operands were written by the generic proxy, the MMA reads them asynchronously
  if (warp == 0) tmem_alloc(&s.tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  if (threadIdx.x == 0) {
    const uint32_t e_tmem = tmem + META_COL;  // 4 metadata columns after the first accumulator
    const uint64_t a0 = sw128_desc(smem_u32(s.a));
    const uint32_t id_d = idesc_bf16(m, N, false), id_s = idesc_bf16(m, N, true);
    if (sparse) tmem_cp_128x128b(e_tmem, meta_desc(smem_u32(s.e)));
    for (int64_t it = 0; it < iters; ++it) {
      const uint32_t acc = tmem + uint32_t(it & 1) * ACC1;
      if (sparse) {
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          const uint64_t b = sw128_desc(smem_u32(s.b[kb >> 1])) + ((kb & 1) * 64 >> 4);
          mma_sparse(acc, a0 + (kb * 32 >> 4), b, e_tmem + (kb & 2), id_s | (kb & 1), it > 1 || kb > 0);
        }
      } else {
        const uint64_t b0 = sw128_desc(smem_u32(s.b[0]));
#pragma unroll
        for (int k = 0; k < 4; ++k) mma_dense(acc, a0 + (k * 32 >> 4), b0 + (k * 32 >> 4), id_d, it > 1 || k > 0);
      }
    }
    tc_commit(&s.done);
    int abort_flag = 0;
    wait_bounded(&s.done, 0, &abort_flag, limit_ns, status, true);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace probe

cudaError_t launch_mma_probe(int m, int sparse, int64_t iters, int num_sms, uint64_t limit_ns, int32_t* status,
                             cudaStream_t stream) {
  using namespace probe;
  cudaError_t e = cudaFuncSetAttribute(probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  probe_kernel<<<num_sms, THREADS, SMEM_BYTES, stream>>>(m, sparse, iters, limit_ns, status);
  return cudaGetLastError();
}

}  // namespace patch
