// Host-side launchers of libpatch's kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "patch.h"

namespace patch {

cudaError_t launch_hard_mask(const uint16_t* W, int64_t N, int64_t K, const float* tile_logits,
                             const float* pattern_logits, uint16_t* W_masked, uint8_t* bitmap,
                             uint8_t* pat_id, int num_sms, cudaStream_t stream);

// pattern ids from pat_id, or (pattern_logits != NULL) from the argmax of the pattern logits
cudaError_t launch_pack(const uint16_t* W, int64_t N, int64_t K, const uint8_t* bitmap,
                        const uint8_t* pat_id, const float* pattern_logits, int64_t n_sparse, void* values,
                        void* meta, patch_tile_desc* desc, int32_t* status, int num_sms, cudaStream_t stream);

cudaError_t launch_tile_kinds(const float* tile_logits, int64_t N, int64_t K, uint8_t* bitmap, int64_t* n_sparse,
                              cudaStream_t stream);

cudaError_t launch_soft_mask(const uint16_t* W, int64_t N, int64_t K, const float* tile_logits,
                             const float* tile_noise, const float* pattern_logits, const float* pattern_noise,
                             float tau, uint16_t* W_soft, float* mask, int num_sms, cudaStream_t stream);

// Decode split: L K-tiles per unit, S K-splits, units CTAs, smem bytes, fp32 workspace bytes.
struct DecodePlan {
  int L, S, units;
  size_t smem, ws_bytes;
};
DecodePlan decode_plan(int64_t M, int64_t N, int64_t K, int num_sms);

cudaError_t launch_decode(const uint16_t* X, int64_t M, const patch_weight& W, uint16_t* Y,
                          void* workspace, int num_sms, cudaStream_t stream);

// Prefill (any M): splits K across CTAs when the units would leave SMs idle and
// the workspace holds the partials (prefill_workspace_bytes; its counters use
// the decode paths' fixed counter region), else runs whole-K units.
cudaError_t launch_prefill(const uint16_t* X, int64_t M, const patch_weight& W, uint16_t* Y, void* workspace,
                           size_t workspace_bytes, int32_t* status, int num_sms, uint64_t limit_ns, int inject,
                           cudaStream_t stream);
size_t prefill_workspace_bytes(int64_t M, const patch_weight& W, int num_sms);

// Gated MLP first half, M > 16: H = silu(X W_gate^T) * (X W_up^T) in one prefill launch.
cudaError_t launch_prefill_mlp(const uint16_t* X, int64_t M, const patch_weight& W_gate, const patch_weight& W_up,
                               uint16_t* H, int32_t* status, int num_sms, uint64_t limit_ns, cudaStream_t stream);

// Independent prefill GEMMs Y_i = X_i W_i^T (M_i >= 1 each) in one launch of
// the prefill kernel; at most kPrefillGroupMax per launch.
constexpr int kPrefillGroupMax = 32;
struct PrefillGroupCall {
  const uint16_t* X;
  int64_t M;
  patch_weight W;
  uint16_t* Y;
};
cudaError_t launch_prefill_group(const PrefillGroupCall* calls, int n, int32_t* status, int num_sms,
                                 uint64_t limit_ns, cudaStream_t stream);

// H = silu(G) * U elementwise (bf16; count a multiple of 8).
cudaError_t launch_silu_mul(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t count, int num_sms,
                            cudaStream_t stream);

// Hard mask with b x b mask tiles (b = 4..128; 128 is launch_hard_mask).
cudaError_t launch_hard_mask_tiles(const uint16_t* W, int64_t N, int64_t K, int64_t mask_tile,
                                   const float* tile_logits, const float* pattern_logits, uint16_t* W_masked,
                                   uint8_t* bitmap, uint8_t* pat_id, int num_sms, cudaStream_t stream);
// exec_tile x exec_tile execution tiles (64 or 128) of a b x b mask bitmap, and their sparse count (device int64).
cudaError_t launch_exec_tiles(const uint8_t* bitmap, int64_t N, int64_t K, int64_t mask_tile, int64_t exec_tile,
                              uint8_t* exec, int64_t* n_sparse, int num_sms, cudaStream_t stream);

// The 64 x 64 execution-tile format: pack (scan + tiles) and GEMM.
cudaError_t launch_pack64(const uint16_t* W, int64_t N, int64_t K, const uint8_t* bitmap, const uint8_t* pat_id,
                          int64_t n_sparse, void* values, void* meta, patch_tile_desc* desc, int32_t* status,
                          int num_sms, cudaStream_t stream);
size_t gemm64_workspace_bytes(int64_t M, const patch_weight64& W, int num_sms);
cudaError_t launch_gemm64(const uint16_t* X, int64_t M, const patch_weight64& W, uint16_t* Y, void* workspace,
                          int32_t* status, int num_sms, uint64_t limit_ns, cudaStream_t stream);

// Workspace layout (patch_gemm_workspace_size covers every path): arrival
// counters sit in a fixed region at the start (the tensor-core decode kernel's,
// one u32 per tile-row quarter; the split-K prefill's, one per output block,
// row and lane quarter), which every call leaves zero, and each path's scratch
// (fp32 partial sums) follows it.  Since no call puts anything else in that
// region, one workspace serves every layer, token count and path in any order.
constexpr size_t kDecodeCounterBytes = 65536;
constexpr int64_t kDecodeMaxTileRows = int64_t(kDecodeCounterBytes / 16);  // tensor-core decode: N <= 524288

// Tensor-core decode (stream-K over panels, M <= 16, N / 128 <= kDecodeMaxTileRows).
size_t decode_tc_workspace_bytes(int64_t M, const patch_weight& W, int num_sms);
cudaError_t launch_decode_tc(const uint16_t* X, int64_t M, const patch_weight& W, uint16_t* Y, void* workspace,
                             int32_t* status, int num_sms, uint64_t limit_ns, cudaStream_t stream);

// Chained decode GEMMs (patch_gemm_chain).  chain_launch_end: end of the
// launch that starts at call j0 (calls fit PATCH_CHAIN_MAX_CALLS and the
// counter region); chain_workspace_bytes: workspace for all launches.
int64_t chain_launch_end(const patch_chain_call* calls, int64_t j0, int64_t n);
size_t chain_workspace_bytes(const patch_chain_call* calls, int64_t n, int num_sms);
cudaError_t launch_chain(const patch_chain_call* calls, int64_t j0, int64_t j1, void* workspace, int32_t* status,
                         int num_sms, uint64_t limit_ns, cudaStream_t stream);
constexpr int64_t kChainMaxTileRows = int64_t(kDecodeCounterBytes / 16) - 1;  // 4 counters per row + 2 words

// Device check of a packed weight's descriptor table (patch_check_weight).
cudaError_t launch_check_weight(const patch_weight& W, int32_t* status, cudaStream_t stream);

// Tensor-core MMA rate probe (patch_mma_probe, patch_mma_probe_m): MMA shape m = 64 or 128.
cudaError_t launch_mma_probe(int m, int sparse, int64_t iters, int num_sms, uint64_t limit_ns, int32_t* status,
                             cudaStream_t stream);

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream is finishing; it must call
// griddepcontrol.wait before touching anything that kernel may write.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// 2D bf16 tensor map with 128-byte swizzle (out-of-bounds reads fill zeros).
bool make_map_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                      uint32_t box_inner, uint32_t box_outer);
// The same with the 64-byte swizzle (box_inner <= 32 elements).
bool make_map_2d_bf16_sw64(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                           uint32_t box_inner, uint32_t box_outer);

}  // namespace patch
