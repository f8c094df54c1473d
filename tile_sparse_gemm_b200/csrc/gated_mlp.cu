// Elementwise half of the gated MLP for the decode path (M <= 16):
// H = silu(G) * U, with G = X W_gate^T and U = X W_up^T already computed by
// two decode GEMMs (bf16).  LLaMA's gated MLP multiplies the SiLU of the gate
// projection by the up projection; the prefill path does this inside the
// GEMM's epilogue instead.  HBM-bound: 4 B read and 2 B written per output.
#include "common.cuh"
#include "kernels.cuh"

namespace patch {

__global__ void __launch_bounds__(256) silu_mul_kernel(const uint4* __restrict__ G, const uint4* __restrict__ U,
                                                       uint4* __restrict__ H, int64_t n8) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // G and U come from the preceding GEMMs
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n8; i += int64_t(gridDim.x) * blockDim.x) {
    const uint4 g = G[i], u = U[i];
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w};
    uint32_t hw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float g0 = bf16_lo(gw[j]), g1 = bf16_hi(gw[j]);
      // silu with CUDA's fast exponential and division, as in the prefill epilogue
      const float h0 = __fdividef(g0, 1.0f + __expf(-g0)) * bf16_lo(uw[j]);
      const float h1 = __fdividef(g1, 1.0f + __expf(-g1)) * bf16_hi(uw[j]);
      hw[j] = uint32_t(f32_to_bf16_rne(h0)) | uint32_t(f32_to_bf16_rne(h1)) << 16;
    }
    H[i] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  }
}

cudaError_t launch_silu_mul(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t count, int num_sms,
                            cudaStream_t stream) {
  const int64_t n8 = count / 8;  // count is a multiple of 128 (N is)
  if (n8 == 0) return cudaSuccess;
  int64_t blocks = (n8 + 255) / 256;
  if (blocks > int64_t(num_sms) * 8) blocks = int64_t(num_sms) * 8;
  return launch_pdl(silu_mul_kernel, dim3(unsigned(blocks)), dim3(256), 0, stream, reinterpret_cast<const uint4*>(G),
                    reinterpret_cast<const uint4*>(U), reinterpret_cast<uint4*>(H), n8);
}

}  // namespace patch
