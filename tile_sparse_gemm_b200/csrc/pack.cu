// patch_pack kernels: build the mixed layout of dense tiles, compressed 2:4
// tiles (2 kept values per group of 4 plus a 4-bit position code) and the tile
// descriptor table.  "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs",
// section 2 "Methodology: PATCH", "Core Mechanism" (each 128 x 128 tile dense
// or 2:4 sparse) and "Inference & Deployment" (sparse tiles must feed the 2:4
// sparse tensor cores, dense tiles the dense ones).
//
// Launch 1 (one CTA): exclusive scan of the tile kinds in row-major tile
// order -> descriptors {kind, sparse ordinal, byte offset}.
// Launch 2 (one CTA per tile): dense tile -> 2 panels of 128 x 64 bf16;
// sparse tile -> 1 panel of kept values + 2048 B of metadata in the order the
// tensor-core sparse MMA reads it.  HBM-bound.  The pattern ids come either
// from pat_id or, fused with the hard mask, from the argmax of the pattern
// logits of sparse tiles only ("Learnable Distributions", item 2).
#include "common.cuh"
#include "kernels.cuh"

namespace patch {

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) pack_scan_kernel(
    const uint8_t* __restrict__ bitmap, int64_t T, int64_t n_sparse, uint64_t panel_bytes,
    patch_tile_desc* __restrict__ desc, int32_t* status) {
  __shared__ uint32_t warp_sums[kScanThreads / 32];
  __shared__ uint64_t carry_s;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int64_t base = 0; base < T; base += kScanThreads) {
    const int64_t t = base + threadIdx.x;
    const uint32_t kind = (t < T && bitmap[t] != 0) ? 1u : 0u;
    // inclusive warp scan
    uint32_t v = kind;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      uint32_t y = __shfl_up_sync(0xFFFFFFFFu, v, d);
      if (lane >= d) v += y;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
      uint32_t s = warp_sums[lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        uint32_t y = __shfl_up_sync(0xFFFFFFFFu, s, d);
        if (lane >= d) s += y;
      }
      warp_sums[lane] = s;  // inclusive prefix over warps
    }
    __syncthreads();
    const uint64_t carry = carry_s;
    const uint64_t before = carry + (warp > 0 ? warp_sums[warp - 1] : 0u) + v - kind;
    if (t < T) {
      patch_tile_desc d;
      d.kind = kind;
      d.sparse_ordinal = kind ? uint32_t(before) : 0xFFFFFFFFu;
      // dense tiles before t take 2 panels each, sparse ones 1
      d.val_offset = panel_bytes * (2ull * uint64_t(t) - before);
      desc[t] = d;
    }
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) carry_s = carry + warp_sums[31];
    __syncthreads();
  }
  if (threadIdx.x == 0 && carry_s != uint64_t(n_sparse)) set_status(status, PATCH_DEV_COUNT);
}

// Index of the first maximum of 6 logits (a later value wins only when
// strictly greater): the pattern decision of patch_hard_mask.
__device__ __forceinline__ uint32_t argmax6_first(const float* v) {
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

constexpr int kPackThreads = 256;                  // threads per tile-packing CTA
constexpr int kPackItems = 2048 / kPackThreads;     // 16-byte items per thread and tile (both kinds)

// FROM_LOGITS: a sparse tile's pattern ids are the argmax of its pattern
// logits (fused hard mask); otherwise they are read from pat_id.
template <bool FROM_LOGITS>
__global__ void __launch_bounds__(kPackThreads) pack_tiles_kernel(
    const uint16_t* __restrict__ W, int64_t K, const uint8_t* __restrict__ pat_id,
    const float4* __restrict__ pattern_logits, const patch_tile_desc* __restrict__ desc, int64_t T,
    int64_t n_sparse, uint64_t values_bytes, uint8_t* __restrict__ values, uint8_t* __restrict__ meta,
    int32_t* status) {
  __shared__ __align__(16) uint8_t meta_s[PATCH_META_TILE_BYTES];
  const int64_t Tk = K / kTile;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const patch_tile_desc d = desc[t];
    const int64_t tn = t / Tk, tk = t - tn * Tk;
    const uint64_t size = d.kind ? PATCH_SPARSE_TILE_BYTES : PATCH_DENSE_TILE_BYTES;
    // a bitmap whose count disagrees with n_sparse must not write past the blobs
    if (d.val_offset + size > values_bytes || (d.kind && int64_t(d.sparse_ordinal) >= n_sparse))
      continue;  // PATCH_DEV_COUNT is raised by the scan
    uint8_t* panel = values + d.val_offset;
    const uint16_t* wt = W + (tn * kTile) * K + tk * kTile;
    if (d.kind == 0) {
      // 2 panels x 128 rows x 8 chunks of 16 B: each thread issues its 8 loads
      // before its 8 stores, so 8 copies per thread are in flight, not one
      uint4 v[kPackItems];
#pragma unroll
      for (int j = 0; j < kPackItems; ++j) {
        const int c = threadIdx.x + j * kPackThreads, h = c >> 10, r = (c >> 3) & 127, q = c & 7;
        v[j] = __ldcs(reinterpret_cast<const uint4*>(wt + int64_t(r) * K + h * 64 + q * 8));
      }
#pragma unroll
      for (int j = 0; j < kPackItems; ++j) {
        const int c = threadIdx.x + j * kPackThreads, h = c >> 10, r = (c >> 3) & 127, q = c & 7;
        *reinterpret_cast<uint4*>(panel + h * PATCH_PANEL_BYTES + r * 128 + q * 16) = v[j];
      }
    } else {
      // 128 rows x 16 pairs of groups; each item reads 8 weights, writes 4
      // values + 1 byte.  Items go in batches (all loads, then the stores):
      // 4 per thread from pattern ids, 2 from logits (12 floats an item).
      constexpr int B = FROM_LOGITS ? 2 : 4;  // measured: logits batches of 1 / 2 / 4 give 0.66 / 0.68 / 0.68
#pragma unroll 1
      for (int j0 = 0; j0 < kPackItems; j0 += B) {
        uint4 w[B];
        uint32_t ids[B][2];
#pragma unroll
        for (int j = 0; j < B; ++j) {
          const int c = threadIdx.x + (j0 + j) * kPackThreads, r = c >> 4, p = c & 15;
          w[j] = __ldcs(reinterpret_cast<const uint4*>(wt + int64_t(r) * K + p * 8));
          // groups 2p, 2p+1 of row r of the tile
          const int64_t group = (tn * kTile + r) * (K / 4) + tk * 32 + 2 * p;
          if constexpr (FROM_LOGITS) {
            // 2 groups x 6 logits = 48 contiguous bytes, 16-byte aligned
            float lg[12];
#pragma unroll
            for (int q = 0; q < 3; ++q) {
              const float4 l = __ldg(pattern_logits + group * 6 / 4 + q);
              lg[4 * q] = l.x;
              lg[4 * q + 1] = l.y;
              lg[4 * q + 2] = l.z;
              lg[4 * q + 3] = l.w;
            }
            ids[j][0] = argmax6_first(lg);
            ids[j][1] = argmax6_first(lg + 6);
          } else {
            const uint16_t ids2 = *reinterpret_cast<const uint16_t*>(pat_id + group);
            ids[j][0] = ids2 & 0xFF;
            ids[j][1] = ids2 >> 8;
          }
        }
#pragma unroll
        for (int j = 0; j < B; ++j) {
          const int c = threadIdx.x + (j0 + j) * kPackThreads, r = c >> 4, p = c & 15;
          uint32_t id0 = ids[j][0], id1 = ids[j][1];
          if (!FROM_LOGITS && (id0 > 5 || id1 > 5)) {
            set_status(status, PATCH_DEV_BAD_PATTERN);
            if (id0 > 5) id0 = 0;
            if (id1 > 5) id1 = 0;
          }
          const uint32_t c0 = pattern_code(id0), c1 = pattern_code(id1);
          // the 4 bf16 of each group as one 64-bit word; position i is bits 16i..16i+15
          const uint64_t g0 = uint64_t(w[j].y) << 32 | w[j].x, g1 = uint64_t(w[j].w) << 32 | w[j].z;
          uint2 out;
          out.x = uint32_t((g0 >> (16 * (c0 & 3))) & 0xFFFFu) | uint32_t((g0 >> (16 * (c0 >> 2))) & 0xFFFFu) << 16;
          out.y = uint32_t((g1 >> (16 * (c1 & 3))) & 0xFFFFu) | uint32_t((g1 >> (16 * (c1 >> 2))) & 0xFFFFu) << 16;
          *reinterpret_cast<uint2*>(panel + r * 128 + p * 8) = out;
          meta_s[meta_byte_index(r, 2 * p)] = uint8_t(c0 | (c1 << 4));
        }
      }
      __syncthreads();
      uint8_t* mt = meta + uint64_t(d.sparse_ordinal) * PATCH_META_TILE_BYTES;
      for (int c = threadIdx.x; c < PATCH_META_TILE_BYTES / 16; c += blockDim.x)
        reinterpret_cast<uint4*>(mt)[c] = reinterpret_cast<const uint4*>(meta_s)[c];
      __syncthreads();
    }
  }
}

cudaError_t launch_pack(const uint16_t* W, int64_t N, int64_t K, const uint8_t* bitmap,
                        const uint8_t* pat_id, const float* pattern_logits, int64_t n_sparse, void* values,
                        void* meta, patch_tile_desc* desc, int32_t* status, int num_sms, cudaStream_t stream) {
  const int64_t T = (N / kTile) * (K / kTile);
  const uint64_t values_bytes =
      uint64_t(T - n_sparse) * PATCH_DENSE_TILE_BYTES + uint64_t(n_sparse) * PATCH_SPARSE_TILE_BYTES;
  pack_scan_kernel<<<1, kScanThreads, 0, stream>>>(bitmap, T, n_sparse, PATCH_PANEL_BYTES, desc, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int64_t blocks = T < int64_t(num_sms) * 16 ? T : int64_t(num_sms) * 16;
  if (pattern_logits)
    pack_tiles_kernel<true><<<int(blocks), kPackThreads, 0, stream>>>(
        W, K, nullptr, reinterpret_cast<const float4*>(pattern_logits), desc, T, n_sparse, values_bytes,
        static_cast<uint8_t*>(values), static_cast<uint8_t*>(meta), status);
  else
    pack_tiles_kernel<false><<<int(blocks), kPackThreads, 0, stream>>>(W, K, pat_id, nullptr, desc, T, n_sparse,
                                                              values_bytes, static_cast<uint8_t*>(values),
                                                              static_cast<uint8_t*>(meta), status);
  return cudaGetLastError();
}

// The 64 x 64 execution-tile format: 64 rows x 32 bf16 panels (64-byte rows),
// a dense tile = 2 panels (k 0..31, 32..63), a sparse tile = 1 panel of kept
// values plus 512 B of metadata stored 8 bytes per tensor-memory lane of the
// M = 64 sparse MMA.  One CTA of 128 threads per tile; 4 items of 16 bytes
// per thread (all loads, then all stores).
constexpr int kPack64Threads = 128;
constexpr int kPack64Items = 512 / kPack64Threads;

__global__ void __launch_bounds__(kPack64Threads) pack64_tiles_kernel(
    const uint16_t* __restrict__ W, int64_t K, const uint8_t* __restrict__ pat_id,
    const patch_tile_desc* __restrict__ desc, int64_t T, int64_t n_sparse, uint64_t values_bytes,
    uint8_t* __restrict__ values, uint8_t* __restrict__ meta, int32_t* status) {
  __shared__ __align__(16) uint8_t meta_s[PATCH_META_TILE64_BYTES];
  const int64_t Tk = K / 64;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const patch_tile_desc d = desc[t];
    const int64_t tn = t / Tk, tk = t - tn * Tk;
    const uint64_t size = d.kind ? PATCH_SPARSE_TILE64_BYTES : PATCH_DENSE_TILE64_BYTES;
    if (d.val_offset + size > values_bytes || (d.kind && int64_t(d.sparse_ordinal) >= n_sparse))
      continue;  // PATCH_DEV_COUNT is raised by the scan
    uint8_t* panel = values + d.val_offset;
    const uint16_t* wt = W + (tn * 64) * K + tk * 64;
    uint4 v[kPack64Items];
    if (d.kind == 0) {
      // 64 rows x 8 chunks of 8 values: chunk q of row r goes to panel q/4, byte 16*(q%4) of row r
#pragma unroll
      for (int j = 0; j < kPack64Items; ++j) {
        const int c = threadIdx.x + j * kPack64Threads, r = c >> 3, q = c & 7;
        v[j] = __ldcs(reinterpret_cast<const uint4*>(wt + int64_t(r) * K + q * 8));
      }
#pragma unroll
      for (int j = 0; j < kPack64Items; ++j) {
        const int c = threadIdx.x + j * kPack64Threads, r = c >> 3, q = c & 7;
        *reinterpret_cast<uint4*>(panel + (q >> 2) * PATCH_PANEL64_BYTES + r * 64 + (q & 3) * 16) = v[j];
      }
    } else {
      // 64 rows x 8 pairs of groups; item (r, p) reads groups 2p, 2p+1 of row r
      uint32_t ids[kPack64Items][2];
#pragma unroll
      for (int j = 0; j < kPack64Items; ++j) {
        const int c = threadIdx.x + j * kPack64Threads, r = c >> 3, p = c & 7;
        v[j] = __ldcs(reinterpret_cast<const uint4*>(wt + int64_t(r) * K + p * 8));
        const uint16_t ids2 =
            *reinterpret_cast<const uint16_t*>(pat_id + (tn * 64 + r) * (K / 4) + tk * 16 + 2 * p);
        ids[j][0] = ids2 & 0xFF;
        ids[j][1] = ids2 >> 8;
      }
#pragma unroll
      for (int j = 0; j < kPack64Items; ++j) {
        const int c = threadIdx.x + j * kPack64Threads, r = c >> 3, p = c & 7;
        uint32_t id0 = ids[j][0], id1 = ids[j][1];
        if (id0 > 5 || id1 > 5) {
          set_status(status, PATCH_DEV_BAD_PATTERN);
          if (id0 > 5) id0 = 0;
          if (id1 > 5) id1 = 0;
        }
        const uint32_t c0 = pattern_code(id0), c1 = pattern_code(id1);
        const uint64_t g0 = uint64_t(v[j].y) << 32 | v[j].x, g1 = uint64_t(v[j].w) << 32 | v[j].z;
        uint2 out;
        out.x = uint32_t((g0 >> (16 * (c0 & 3))) & 0xFFFFu) | uint32_t((g0 >> (16 * (c0 >> 2))) & 0xFFFFu) << 16;
        out.y = uint32_t((g1 >> (16 * (c1 & 3))) & 0xFFFFu) | uint32_t((g1 >> (16 * (c1 >> 2))) & 0xFFFFu) << 16;
        *reinterpret_cast<uint2*>(panel + r * 64 + p * 8) = out;
        meta_s[meta64_byte_index(r, 2 * p)] = uint8_t(c0 | (c1 << 4));
      }
      __syncthreads();
      uint8_t* mt = meta + uint64_t(d.sparse_ordinal) * PATCH_META_TILE64_BYTES;
      for (int c = threadIdx.x; c < PATCH_META_TILE64_BYTES / 16; c += blockDim.x)
        reinterpret_cast<uint4*>(mt)[c] = reinterpret_cast<const uint4*>(meta_s)[c];
      __syncthreads();
    }
  }
}

cudaError_t launch_pack64(const uint16_t* W, int64_t N, int64_t K, const uint8_t* bitmap, const uint8_t* pat_id,
                          int64_t n_sparse, void* values, void* meta, patch_tile_desc* desc, int32_t* status,
                          int num_sms, cudaStream_t stream) {
  const int64_t T = (N / 64) * (K / 64);
  const uint64_t values_bytes =
      uint64_t(T - n_sparse) * PATCH_DENSE_TILE64_BYTES + uint64_t(n_sparse) * PATCH_SPARSE_TILE64_BYTES;
  pack_scan_kernel<<<1, kScanThreads, 0, stream>>>(bitmap, T, n_sparse, PATCH_PANEL64_BYTES, desc, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t blocks = T < int64_t(num_sms) * 16 ? T : int64_t(num_sms) * 16;
  pack64_tiles_kernel<<<int(blocks), kPack64Threads, 0, stream>>>(W, K, pat_id, desc, T, n_sparse, values_bytes,
                                                                   static_cast<uint8_t*>(values),
                                                                   static_cast<uint8_t*>(meta), status);
  return cudaGetLastError();
}

// Tile kinds from the tile logits (argmax of 2, ties -> dense) and their count:
// one thread per tile over a grid of 256-thread blocks, the count summed per
// warp (shuffle), per block (shared memory) and then once per block into the
// device count, which is zeroed on the stream before the launch.
__global__ void __launch_bounds__(256) tile_kinds_kernel(const float2* __restrict__ tile_logits, int64_t T,
                                                         uint8_t* __restrict__ bitmap,
                                                         unsigned long long* __restrict__ n_sparse) {
  __shared__ unsigned int block_total;
  if (threadIdx.x == 0) block_total = 0;
  __syncthreads();
  const int64_t t = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  unsigned int sparse = 0;
  if (t < T) {
    const float2 l = __ldg(tile_logits + t);
    sparse = l.y > l.x ? 1u : 0u;
    bitmap[t] = uint8_t(sparse);
  }
  const unsigned int warp_total = __reduce_add_sync(0xFFFFFFFFu, sparse);
  if ((threadIdx.x & 31) == 0) atomicAdd(&block_total, warp_total);
  __syncthreads();
  if (threadIdx.x == 0 && block_total) atomicAdd(n_sparse, static_cast<unsigned long long>(block_total));
}

cudaError_t launch_tile_kinds(const float* tile_logits, int64_t N, int64_t K, uint8_t* bitmap, int64_t* n_sparse,
                              cudaStream_t stream) {
  const int64_t T = (N / kTile) * (K / kTile);
  cudaError_t e = cudaMemsetAsync(n_sparse, 0, sizeof(int64_t), stream);
  if (e != cudaSuccess) return e;
  tile_kinds_kernel<<<int((T + 255) / 256), 256, 0, stream>>>(reinterpret_cast<const float2*>(tile_logits), T,
                                                              bitmap, reinterpret_cast<unsigned long long*>(n_sparse));
  return cudaGetLastError();
}

}  // namespace patch
