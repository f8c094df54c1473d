// Decode path of patch_gemm (M <= 16 tokens): split-K GEMV on CUDA cores
// that streams exactly the stored bytes of the packed weight once.
//
// Layer: Y[m][n] = sum_k X[m][k] * W_eff[n][k], W_eff the hybrid tile-sparse
// weight of "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs" (section 2
// "Methodology: PATCH", "Core Mechanism"): dense 128 x 128 tiles are read as
// 2 panels of 128 x 64 bf16, sparse tiles as 1 panel of kept values plus
// their 4-bit position codes ("Inference & Deployment": sparse tiles carry
// only the 2 kept values per group of 4).
//
// Work unit = (slab of 16*R rows inside one 128-row tile row, range of L
// K-tiles).  A CTA of 256 threads = 16 row slots x 16 k-lanes; thread
// (slot, kl) owns rows slot + 16 i (i < R) and the 8 logical k = 8 kl .. 8 kl+7
// of every tile in its range.  Per tile it loads R x 16 B (dense) or
// R x (8 B values + 1 B codes) (sparse), expands sparse groups to 8 fp32
// weights with zeros at pruned positions, and accumulates R x MT fp32 dot
// products against X staged in shared memory (one 16 B smem read per token,
// reused by R rows).  The 16 k-lanes of a row reduce by shuffles at the end;
// with several K splits the fp32 partials go to workspace [S][M][N] and a
// second kernel sums them in split order (deterministic) and rounds to bf16.
#include "common.cuh"
#include "kernels.cuh"

namespace patch {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeR = 4;  // rows per thread -> 64-row slabs

struct TileRaw {
  uint4 v;        // dense: 8 bf16; sparse: 4 kept bf16 in v.x, v.y
  uint32_t code;  // sparse: codes of groups 2kl (low nibble) and 2kl+1 (high nibble)
};

template <int R>
__device__ __forceinline__ void load_tile(TileRaw (&raw)[R], const patch_tile_desc& d,
                                          const uint8_t* __restrict__ values,
                                          const uint8_t* __restrict__ meta, int row0, int kl) {
  const uint8_t* base = values + d.val_offset;
  if (d.kind == 0) {
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int r = row0 + 16 * i;
      raw[i].v = __ldcs(reinterpret_cast<const uint4*>(base + (kl >> 3) * PATCH_PANEL_BYTES + r * 128 +
                                                       (kl & 7) * 16));
      raw[i].code = 0;
    }
  } else {
    const uint8_t* mt = meta + uint64_t(d.sparse_ordinal) * PATCH_META_TILE_BYTES;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int r = row0 + 16 * i;
      const uint2 v = __ldcs(reinterpret_cast<const uint2*>(base + r * 128 + kl * 8));
      raw[i].v = make_uint4(v.x, v.y, 0u, 0u);
      raw[i].code = __ldg(mt + meta_byte_index(r, 2 * kl));
    }
  }
}

// 4 weights of one group from its 2 kept values (a, b) and code (i0 | i1 << 2)
__device__ __forceinline__ void expand_group(uint32_t kept2, uint32_t code, float* w4) {
  const float a = bf16_lo(kept2), b = bf16_hi(kept2);
  const uint32_t i0 = code & 3, i1 = (code >> 2) & 3;
#pragma unroll
  for (uint32_t p = 0; p < 4; ++p) w4[p] = (p == i0) ? a : ((p == i1) ? b : 0.0f);
}

template <int MT, int R>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_gemm_kernel(
    const uint16_t* __restrict__ X, int64_t N, int64_t K, const uint8_t* __restrict__ values,
    const uint8_t* __restrict__ meta, const patch_tile_desc* __restrict__ desc, int L, int S,
    uint16_t* __restrict__ Y, float* __restrict__ ws) {
  extern __shared__ __align__(16) uint16_t xs[];  // [MT][L*128]
  const int64_t Tk = K / kTile;
  const int slabs_per_row = kTile / (16 * R);
  const int unit = blockIdx.x;
  const int split = unit % S;
  const int slab = unit / S;
  const int64_t tn = slab / slabs_per_row;
  const int row_base = (slab % slabs_per_row) * 16 * R;
  const int kt0 = split * L;
  const int kt1 = (kt0 + L < Tk) ? kt0 + L : int(Tk);
  const int nkt = kt1 - kt0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int kl = lane & 15;
  const int row0 = row_base + warp * 2 + (lane >> 4);  // tile row of i = 0

  // stage X[0..MT)[kt0*128 .. kt1*128) in shared memory, 16 B per thread-step
  const int kspan = nkt * kTile;
  const int chunks = MT * (kspan / 8);
  for (int c = threadIdx.x; c < chunks; c += kDecodeThreads) {
    const int m = c / (kspan / 8), q = c - m * (kspan / 8);
    *reinterpret_cast<uint4*>(xs + m * (L * kTile) + q * 8) =
        __ldg(reinterpret_cast<const uint4*>(X + int64_t(m) * K + int64_t(kt0) * kTile + q * 8));
  }
  __syncthreads();

  float acc[R][MT];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[i][m] = 0.0f;

  TileRaw raw[R];
  patch_tile_desc d = desc[tn * Tk + kt0];
  load_tile<R>(raw, d, values, meta, row0, kl);
  for (int lt = 0; lt < nkt; ++lt) {
    // expand the current tile to fp32 weights
    float wf[R][8];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      if (d.kind == 0) {
        const uint32_t u[4] = {raw[i].v.x, raw[i].v.y, raw[i].v.z, raw[i].v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          wf[i][2 * q] = bf16_lo(u[q]);
          wf[i][2 * q + 1] = bf16_hi(u[q]);
        }
      } else {
        expand_group(raw[i].v.x, raw[i].code & 0xF, &wf[i][0]);
        expand_group(raw[i].v.y, raw[i].code >> 4, &wf[i][4]);
      }
    }
    // issue the next tile's loads before the FMAs
    if (lt + 1 < nkt) {
      d = desc[tn * Tk + kt0 + lt + 1];
      load_tile<R>(raw, d, values, meta, row0, kl);
    }
    const uint16_t* xrow = xs + lt * kTile + kl * 8;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const uint4 xv = *reinterpret_cast<const uint4*>(xrow + m * (L * kTile));
      const float x[8] = {bf16_lo(xv.x), bf16_hi(xv.x), bf16_lo(xv.y), bf16_hi(xv.y),
                          bf16_lo(xv.z), bf16_hi(xv.z), bf16_lo(xv.w), bf16_hi(xv.w)};
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][m] = fmaf(wf[i][j], x[j], acc[i][m]);
    }
  }

  // reduce across the 16 k-lanes of each row (xor stays inside the half warp)
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float v = acc[i][m];
      v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
      v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
      v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
      v += __shfl_xor_sync(0xFFFFFFFFu, v, 8);
      acc[i][m] = v;
    }
  // k-lane kl writes token m == kl (and m == kl + 16, unused for MT <= 16)
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int64_t n = tn * kTile + row0 + 16 * i;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (kl == m) {
        if (S == 1)
          Y[int64_t(m) * N + n] = f32_to_bf16_rne(acc[i][m]);
        else
          ws[(int64_t(split) * MT + m) * N + n] = acc[i][m];
      }
    }
  }
}

__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float4* __restrict__ ws,
                                                            int64_t MN4, int S,
                                                            uint2* __restrict__ Y) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < MN4;
       i += int64_t(gridDim.x) * blockDim.x) {
    float4 s = __ldcs(ws + i);
    for (int p = 1; p < S; ++p) {
      const float4 v = __ldcs(ws + int64_t(p) * MN4 + i);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    uint2 o;
    o.x = uint32_t(f32_to_bf16_rne(s.x)) | uint32_t(f32_to_bf16_rne(s.y)) << 16;
    o.y = uint32_t(f32_to_bf16_rne(s.z)) | uint32_t(f32_to_bf16_rne(s.w)) << 16;
    Y[i] = o;
  }
}

DecodePlan decode_plan(int64_t M, int64_t N, int64_t K, int num_sms) {
  DecodePlan p;
  const int64_t Tk = K / kTile;
  const int64_t slabs = N / (16 * kDecodeR);
  const int64_t target = int64_t(num_sms) * 4;
  int64_t S = (target + slabs - 1) / slabs;
  if (S < 1) S = 1;
  int64_t L = (Tk + S - 1) / S;
  const int64_t Lmax = (48 * 1024) / (M * kTile * 2);  // X chunk <= 48 KB of smem
  if (L > Lmax) L = Lmax;
  if (L < 1) L = 1;
  S = (Tk + L - 1) / L;
  p.L = int(L);
  p.S = int(S);
  p.units = int(slabs * S);
  p.smem = size_t(M) * size_t(L) * kTile * 2;
  p.ws_bytes = S > 1 ? size_t(S) * size_t(M) * size_t(N) * 4 : 0;
  return p;
}

template <int MT>
static cudaError_t launch_decode_mt(const uint16_t* X, const patch_weight& W, uint16_t* Y,
                                    float* ws, const DecodePlan& p, cudaStream_t stream) {
  auto kern = decode_gemm_kernel<MT, kDecodeR>;
  if (p.smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(p.smem));
    if (e != cudaSuccess) return e;
  }
  kern<<<p.units, kDecodeThreads, p.smem, stream>>>(
      X, W.N, W.K, static_cast<const uint8_t*>(W.values), static_cast<const uint8_t*>(W.meta), W.desc,
      p.L, p.S, Y, ws);
  return cudaGetLastError();
}

cudaError_t launch_decode(const uint16_t* X, int64_t M, const patch_weight& W, uint16_t* Y,
                          void* workspace, int num_sms, cudaStream_t stream) {
  const DecodePlan p = decode_plan(M, W.N, W.K, num_sms);
  float* ws = static_cast<float*>(workspace);
  cudaError_t e;
  switch (M) {
#define PATCH_DECODE_CASE(mt) \
  case mt: e = launch_decode_mt<mt>(X, W, Y, ws, p, stream); break;
    PATCH_DECODE_CASE(1) PATCH_DECODE_CASE(2) PATCH_DECODE_CASE(3) PATCH_DECODE_CASE(4)
    PATCH_DECODE_CASE(5) PATCH_DECODE_CASE(6) PATCH_DECODE_CASE(7) PATCH_DECODE_CASE(8)
    PATCH_DECODE_CASE(9) PATCH_DECODE_CASE(10) PATCH_DECODE_CASE(11) PATCH_DECODE_CASE(12)
    PATCH_DECODE_CASE(13) PATCH_DECODE_CASE(14) PATCH_DECODE_CASE(15) PATCH_DECODE_CASE(16)
#undef PATCH_DECODE_CASE
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess || p.S == 1) return e;
  const int64_t MN4 = M * W.N / 4;  // N % 128 == 0
  int64_t blocks = (MN4 + 255) / 256;
  if (blocks > int64_t(num_sms) * 8) blocks = int64_t(num_sms) * 8;
  splitk_reduce_kernel<<<int(blocks), 256, 0, stream>>>(reinterpret_cast<const float4*>(ws), MN4, p.S,
                                                        reinterpret_cast<uint2*>(Y));
  return cudaGetLastError();
}

}  // namespace patch
