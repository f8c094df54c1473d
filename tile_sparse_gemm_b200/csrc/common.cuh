// Shared device helpers of libpatch (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "patch.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libpatch is written for sm_100a (B200) only"
#endif

namespace patch {

constexpr int kTile = PATCH_TILE;

// bf16 bit pattern <-> fp32 (exact widening; RNE narrowing)
__device__ __forceinline__ float bf16_lo(uint32_t two) { return __uint_as_float(two << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t two) { return __uint_as_float(two & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  // cvt.rn.bf16.f32 rounds to nearest even and keeps NaN a NaN
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
  return r;
}

__device__ __forceinline__ void set_status(int32_t* status, int32_t bits) {
  if (status) atomicOr(status, bits);
}

// Byte of a sparse tile's 2048-byte metadata block holding group g (0..31) of
// tile row r (0..127); the code sits in the low nibble for even g.
__host__ __device__ __forceinline__ uint32_t meta_byte_index(uint32_t r, uint32_t g) {
  return ((g >> 1) & 1u) | (((r >> 3) & 1u) << 1) | ((g >> 3) << 2) | ((r & 7u) << 4) |
         (((g >> 2) & 1u) << 7) | ((r >> 4) << 8);
}

// Byte of a 64 x 64 sparse tile's 512-byte metadata block holding group g
// (0..15) of tile row r (0..63): 8 bytes per tensor-memory lane of the M = 64
// sparse MMA (lane 32*(r>>4) + (r&7) + 8*((g>>2)&1)), column g>>3 in bytes 4*(g>>3)..
__host__ __device__ __forceinline__ uint32_t meta64_byte_index(uint32_t r, uint32_t g) {
  return ((g >> 1) & 1u) | (((r >> 3) & 1u) << 1) | ((g >> 3) << 2) | ((r & 7u) << 3) | (((g >> 2) & 1u) << 6) |
         ((r >> 4) << 7);
}

// kept pair (i0, i1) of pattern id p, packed as i0 | i1 << 2 (the metadata code)
__host__ __device__ __forceinline__ uint32_t pattern_code(uint32_t p) {
  // ids 0..5 -> codes 0x4 0x8 0xC 0x9 0xD 0xE, nibble p of this constant
  return (0xED9C84u >> (4 * p)) & 0xFu;  // only valid for p <= 5
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

}  // namespace patch
