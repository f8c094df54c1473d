// patch_hard_mask kernel: the inference-time (argmax) form of PATCH's hybrid
// mask.  "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", section 2
// "Methodology: PATCH", "Learnable Distributions": a 2-way tile logit chooses
// dense vs 2:4 sparse, a 6-way pattern logit per group of 4 chooses the kept
// pair inside sparse tiles.
//
// HBM-bound elementwise pass: per weight it reads 2 B of W and 6 B of pattern
// logits and writes 2 B of masked W plus 1/4 B of pattern id.  One thread
// handles 8 consecutive groups (32 weights) of one row: 4 x 16 B loads of W,
// 12 x 16 B loads of logits, 4 x 16 B stores, one 8 B store of ids.  The
// loads go through L1 (not the streaming hint): a warp's 16-byte pieces of
// 192-byte items use half of each 32-byte sector per instruction, and the
// next instruction finds the other half there.
#include "common.cuh"
#include "kernels.cuh"

namespace patch {

// Index of the first maximum (a later value wins only when strictly greater).
__device__ __forceinline__ uint32_t argmax6(const float* v) {
  uint32_t best = 0;
  float bv = v[0];
#pragma unroll
  for (uint32_t j = 1; j < 6; ++j) {
    if (v[j] > bv) {
      bv = v[j];
      best = j;
    }
  }
  return best;
}

__global__ void __launch_bounds__(256) hard_mask_kernel(
    const uint4* __restrict__ W, int64_t N, int64_t K, const float* __restrict__ tile_logits,
    const float4* __restrict__ pattern_logits, uint4* __restrict__ W_masked,
    uint8_t* __restrict__ bitmap, uint2* __restrict__ pat_id) {
  const int64_t items_per_row = K / 32;  // 8 groups per item
  const int64_t n_items = N * items_per_row;
  const int64_t Tk = K / kTile;
  for (int64_t it = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; it < n_items;
       it += int64_t(gridDim.x) * blockDim.x) {
    const int64_t n = it / items_per_row;
    const int64_t j = it - n * items_per_row;  // item within row: k = 32j .. 32j+31
    const int64_t tn = n / kTile, tk = (32 * j) / kTile;
    const float l0 = __ldg(tile_logits + 2 * (tn * Tk + tk));
    const float l1 = __ldg(tile_logits + 2 * (tn * Tk + tk) + 1);
    const bool sparse = l1 > l0;  // argmax of (dense, sparse), ties -> dense
    if (bitmap && n % kTile == 0 && (32 * j) % kTile == 0) bitmap[tn * Tk + tk] = sparse ? 1 : 0;

    // 8 groups x 6 logits = 48 floats = 12 float4, contiguous
    float lg[48];
    const float4* lp = pattern_logits + it * 12;
#pragma unroll
    for (int q = 0; q < 12; ++q) {
      float4 v = __ldg(lp + q);
      lg[4 * q] = v.x;
      lg[4 * q + 1] = v.y;
      lg[4 * q + 2] = v.z;
      lg[4 * q + 3] = v.w;
    }
    uint32_t ids[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) ids[g] = argmax6(lg + 6 * g);
    uint2 packed;
    packed.x = ids[0] | ids[1] << 8 | ids[2] << 16 | ids[3] << 24;
    packed.y = ids[4] | ids[5] << 8 | ids[6] << 16 | ids[7] << 24;
    __stcs(pat_id + it, packed);

    if (W_masked) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // 16 B = 8 weights = groups 2q, 2q+1
        uint4 w = __ldg(W + it * 4 + q);
        if (sparse) {
          const uint32_t c0 = pattern_code(ids[2 * q]), c1 = pattern_code(ids[2 * q + 1]);
          // keep-masks of the 4 bf16 lanes of each group (bit i set = keep position i)
          const uint32_t k0 = (1u << (c0 & 3)) | (1u << (c0 >> 2));
          const uint32_t k1 = (1u << (c1 & 3)) | (1u << (c1 >> 2));
          w.x &= ((k0 & 1) ? 0x0000FFFFu : 0u) | ((k0 & 2) ? 0xFFFF0000u : 0u);
          w.y &= ((k0 & 4) ? 0x0000FFFFu : 0u) | ((k0 & 8) ? 0xFFFF0000u : 0u);
          w.z &= ((k1 & 1) ? 0x0000FFFFu : 0u) | ((k1 & 2) ? 0xFFFF0000u : 0u);
          w.w &= ((k1 & 4) ? 0x0000FFFFu : 0u) | ((k1 & 8) ? 0xFFFF0000u : 0u);
        }
        __stcs(W_masked + it * 4 + q, w);
      }
    }
  }
}

cudaError_t launch_hard_mask(const uint16_t* W, int64_t N, int64_t K, const float* tile_logits,
                             const float* pattern_logits, uint16_t* W_masked, uint8_t* bitmap,
                             uint8_t* pat_id, int num_sms, cudaStream_t stream) {
  const int64_t n_items = N * (K / 32);
  const int threads = 256;
  int64_t blocks = (n_items + threads - 1) / threads;
  const int64_t cap = int64_t(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  hard_mask_kernel<<<int(blocks), threads, 0, stream>>>(
      reinterpret_cast<const uint4*>(W), N, K, tile_logits,
      reinterpret_cast<const float4*>(pattern_logits), reinterpret_cast<uint4*>(W_masked), bitmap,
      reinterpret_cast<uint2*>(pat_id));
  return cudaGetLastError();
}

// Mask tiles of b x b, b = 4..64 ("Ablation Studies", tile size: the learned
// tile may be as small as 4 x 4).  The same pass as hard_mask_kernel, but an
// item's 8 groups may lie in different mask tiles (b < 32), so the tile
// choice is taken per group; the tile logits ([N/b][K/b] pairs, 8 bytes a
// tile) are read through L1, where an item's neighbours find them.
__global__ void __launch_bounds__(256) hard_mask_tiles_kernel(
    const uint4* __restrict__ W, int64_t N, int64_t K, int lb, const float2* __restrict__ tile_logits,
    const float4* __restrict__ pattern_logits, uint4* __restrict__ W_masked, uint8_t* __restrict__ bitmap,
    uint2* __restrict__ pat_id) {
  const int64_t items_per_row = K / 32;
  const int64_t n_items = N * items_per_row;
  const int64_t b = int64_t(1) << lb, Tkb = K >> lb;
  for (int64_t it = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; it < n_items;
       it += int64_t(gridDim.x) * blockDim.x) {
    const int64_t n = it / items_per_row;
    const int64_t j = it - n * items_per_row;  // k = 32j .. 32j+31
    const int64_t tn = n >> lb;
    uint32_t sp = 0;  // bit g: group g lies in a sparse tile
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const int64_t k = 32 * j + 4 * g;
      const int64_t t = tn * Tkb + (k >> lb);
      const float2 l = __ldg(tile_logits + t);
      const bool sparse = l.y > l.x;  // argmax of (dense, sparse), ties -> dense
      sp |= uint32_t(sparse) << g;
      if (bitmap && (n & (b - 1)) == 0 && (k & (b - 1)) == 0) bitmap[t] = sparse ? 1 : 0;
    }
    float lg[48];
    const float4* lp = pattern_logits + it * 12;
#pragma unroll
    for (int q = 0; q < 12; ++q) {
      float4 v = __ldg(lp + q);
      lg[4 * q] = v.x;
      lg[4 * q + 1] = v.y;
      lg[4 * q + 2] = v.z;
      lg[4 * q + 3] = v.w;
    }
    uint32_t ids[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) ids[g] = argmax6(lg + 6 * g);
    uint2 packed;
    packed.x = ids[0] | ids[1] << 8 | ids[2] << 16 | ids[3] << 24;
    packed.y = ids[4] | ids[5] << 8 | ids[6] << 16 | ids[7] << 24;
    __stcs(pat_id + it, packed);

    if (W_masked) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // 16 B = 8 weights = groups 2q, 2q+1
        uint4 w = __ldg(W + it * 4 + q);
        const uint32_t c0 = pattern_code(ids[2 * q]), c1 = pattern_code(ids[2 * q + 1]);
        // keep-masks of the 4 bf16 lanes of each group (bit i set = keep position i)
        const uint32_t k0 = (sp >> (2 * q)) & 1 ? (1u << (c0 & 3)) | (1u << (c0 >> 2)) : 0xFu;
        const uint32_t k1 = (sp >> (2 * q + 1)) & 1 ? (1u << (c1 & 3)) | (1u << (c1 >> 2)) : 0xFu;
        w.x &= ((k0 & 1) ? 0x0000FFFFu : 0u) | ((k0 & 2) ? 0xFFFF0000u : 0u);
        w.y &= ((k0 & 4) ? 0x0000FFFFu : 0u) | ((k0 & 8) ? 0xFFFF0000u : 0u);
        w.z &= ((k1 & 1) ? 0x0000FFFFu : 0u) | ((k1 & 2) ? 0xFFFF0000u : 0u);
        w.w &= ((k1 & 4) ? 0x0000FFFFu : 0u) | ((k1 & 8) ? 0xFFFF0000u : 0u);
        __stcs(W_masked + it * 4 + q, w);
      }
    }
  }
}

cudaError_t launch_hard_mask_tiles(const uint16_t* W, int64_t N, int64_t K, int64_t mask_tile,
                                   const float* tile_logits, const float* pattern_logits, uint16_t* W_masked,
                                   uint8_t* bitmap, uint8_t* pat_id, int num_sms, cudaStream_t stream) {
  if (mask_tile == kTile)
    return launch_hard_mask(W, N, K, tile_logits, pattern_logits, W_masked, bitmap, pat_id, num_sms, stream);
  int lb = 0;
  while ((int64_t(1) << lb) < mask_tile) ++lb;
  const int64_t n_items = N * (K / 32);
  const int threads = 256;
  int64_t blocks = (n_items + threads - 1) / threads;
  const int64_t cap = int64_t(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  hard_mask_tiles_kernel<<<int(blocks), threads, 0, stream>>>(
      reinterpret_cast<const uint4*>(W), N, K, lb, reinterpret_cast<const float2*>(tile_logits),
      reinterpret_cast<const float4*>(pattern_logits), reinterpret_cast<uint4*>(W_masked), bitmap,
      reinterpret_cast<uint2*>(pat_id));
  return cudaGetLastError();
}

// Execution tiles of a b x b mask: the 128 x 128 tile (tn, tk) is sparse only
// when all r x r = (128/b)^2 mask tiles inside it are.  One warp per
// execution tile (its lanes read r consecutive bitmap bytes of one row at a
// time), one atomic increment of the device count per sparse tile; the count
// is zeroed on the stream before the launch.
__global__ void __launch_bounds__(256) exec_tiles_kernel(const uint8_t* __restrict__ bitmap, int64_t Tn,
                                                         int64_t Tk, int lr, uint8_t* __restrict__ exec,
                                                         unsigned long long* __restrict__ n_sparse) {
  const int lane = threadIdx.x & 31;
  const int64_t r = int64_t(1) << lr, Tkb = Tk << lr;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5; t < Tn * Tk; t += warps) {
    const int64_t tn = t / Tk, tk = t - tn * Tk;
    bool all = true;
    for (int64_t e = lane; e < r * r; e += 32)
      all = all && bitmap[((tn << lr) + (e >> lr)) * Tkb + (tk << lr) + (e & (r - 1))] != 0;
    all = __all_sync(0xFFFFFFFFu, all);
    if (lane == 0) {
      exec[t] = all ? 1 : 0;
      if (all) atomicAdd(n_sparse, 1ull);
    }
  }
}

cudaError_t launch_exec_tiles(const uint8_t* bitmap, int64_t N, int64_t K, int64_t mask_tile, int64_t exec_tile,
                              uint8_t* exec, int64_t* n_sparse, int num_sms, cudaStream_t stream) {
  int lr = 0;
  while ((exec_tile >> lr) > mask_tile) ++lr;
  const int64_t Tn = N / exec_tile, Tk = K / exec_tile;
  cudaError_t e = cudaMemsetAsync(n_sparse, 0, sizeof(int64_t), stream);
  if (e != cudaSuccess) return e;
  const int threads = 256;
  int64_t blocks = (Tn * Tk * 32 + threads - 1) / threads;
  const int64_t cap = int64_t(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  exec_tiles_kernel<<<int(blocks), threads, 0, stream>>>(bitmap, Tn, Tk, lr, exec,
                                                         reinterpret_cast<unsigned long long*>(n_sparse));
  return cudaGetLastError();
}

}  // namespace patch

namespace patch {

// Training-time (soft) hybrid mask: the Gumbel-Softmax relaxation of the two
// choices above ("Core Mechanism": the mask is a weighted combination of the
// dense option and the 2:4 option).  Per tile p = softmax((l + g) / tau) over
// (dense, sparse); per group q = softmax((l + g) / tau) over the 6 patterns;
// M = p_dense + p_sparse * sum_j q_j [position in pattern j]; W_soft = W * M.
// The Gumbel samples g are the caller's (NULL = none).  One thread per 8
// groups of one row, as in the hard mask; HBM-bound.
__global__ void __launch_bounds__(256) soft_mask_kernel(
    const uint4* __restrict__ W, int64_t N, int64_t K, const float2* __restrict__ tile_logits,
    const float2* __restrict__ tile_noise, const float4* __restrict__ pattern_logits,
    const float4* __restrict__ pattern_noise, float inv_tau, uint4* __restrict__ W_soft,
    float4* __restrict__ mask) {
  const int64_t items_per_row = K / 32;  // 8 groups per item
  const int64_t n_items = N * items_per_row;
  const int64_t Tk = K / kTile;
  for (int64_t it = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; it < n_items;
       it += int64_t(gridDim.x) * blockDim.x) {
    const int64_t n = it / items_per_row;
    const int64_t j = it - n * items_per_row;
    const int64_t t = (n / kTile) * Tk + (32 * j) / kTile;
    float2 tl = tile_logits[t];
    if (tile_noise) {
      const float2 g = tile_noise[t];
      tl.x += g.x;
      tl.y += g.y;
    }
    const float zd = tl.x * inv_tau, zs = tl.y * inv_tau, zm = fmaxf(zd, zs);
    const float ed = expf(zd - zm), es = expf(zs - zm);
    const float pd = ed / (ed + es), ps = es / (ed + es);

    float lg[48];
#pragma unroll
    for (int q = 0; q < 12; ++q) {
      float4 v = __ldg(pattern_logits + it * 12 + q);
      if (pattern_noise) {
        const float4 g = __ldg(pattern_noise + it * 12 + q);
        v.x += g.x;
        v.y += g.y;
        v.z += g.z;
        v.w += g.w;
      }
      lg[4 * q] = v.x;
      lg[4 * q + 1] = v.y;
      lg[4 * q + 2] = v.z;
      lg[4 * q + 3] = v.w;
    }
    float m[32];
#pragma unroll
    for (int gi = 0; gi < 8; ++gi) {
      const float* l = lg + 6 * gi;
      float zmax = l[0] * inv_tau;
#pragma unroll
      for (int c = 1; c < 6; ++c) zmax = fmaxf(zmax, l[c] * inv_tau);
      float e[6], sum = 0.0f;
#pragma unroll
      for (int c = 0; c < 6; ++c) {
        e[c] = expf(l[c] * inv_tau - zmax);
        sum += e[c];
      }
      // patterns 0:(0,1) 1:(0,2) 2:(0,3) 3:(1,2) 4:(1,3) 5:(2,3): each position lies in 3
      const float keep[4] = {e[0] + e[1] + e[2], e[0] + e[3] + e[4], e[1] + e[3] + e[5], e[2] + e[4] + e[5]};
#pragma unroll
      for (int i = 0; i < 4; ++i) m[4 * gi + i] = pd + ps * (keep[i] / sum);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // 16 B = 8 weights
      const uint4 w = __ldg(W + it * 4 + q);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
      uint32_t out[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float a = bf16_lo(ww[h]) * m[8 * q + 2 * h], b = bf16_hi(ww[h]) * m[8 * q + 2 * h + 1];
        out[h] = uint32_t(f32_to_bf16_rne(a)) | uint32_t(f32_to_bf16_rne(b)) << 16;
      }
      __stcs(W_soft + it * 4 + q, make_uint4(out[0], out[1], out[2], out[3]));
    }
    if (mask) {
#pragma unroll
      for (int q = 0; q < 8; ++q) __stcs(mask + it * 8 + q, make_float4(m[4 * q], m[4 * q + 1], m[4 * q + 2], m[4 * q + 3]));
    }
  }
}

cudaError_t launch_soft_mask(const uint16_t* W, int64_t N, int64_t K, const float* tile_logits,
                             const float* tile_noise, const float* pattern_logits, const float* pattern_noise,
                             float tau, uint16_t* W_soft, float* mask, int num_sms, cudaStream_t stream) {
  const int64_t n_items = N * (K / 32);
  int64_t blocks = (n_items + 255) / 256;
  if (blocks > int64_t(num_sms) * 8) blocks = int64_t(num_sms) * 8;
  soft_mask_kernel<<<int(blocks), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(W), N, K, reinterpret_cast<const float2*>(tile_logits),
      reinterpret_cast<const float2*>(tile_noise), reinterpret_cast<const float4*>(pattern_logits),
      reinterpret_cast<const float4*>(pattern_noise), 1.0f / tau, reinterpret_cast<uint4*>(W_soft),
      reinterpret_cast<float4*>(mask));
  return cudaGetLastError();
}

}  // namespace patch
