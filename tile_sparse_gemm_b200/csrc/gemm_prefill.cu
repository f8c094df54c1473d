// Prefill path of patch_gemm (M > 16): a persistent, warp-specialised
// TMA + tcgen05 kernel for sm_100a in which dense tiles run on the dense
// tensor-core MMA and 2:4 sparse tiles on the structured-sparse MMA, both
// accumulating into one fp32 tile in tensor memory.
//
// "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", section 2
// "Methodology: PATCH", "Inference & Deployment": hybrid execution over
// 128 x 128 tiles; dense tiles use dense tensor-core kernels, sparse tiles the
// 2:4 sparse tensor cores.
//
// The sparse operand of the tensor-core MMA is A (the M side), so the kernel
// computes Y^T = W_eff * X^T: the MMA's M = 128 rows of W (one tile row), its
// N = BT tokens, K streams over the tiles of the row.
//
// CTA = 6 warps, one CTA per SM, static round-robin over output tiles
// (tile row tn, token block tb):
//   warp 0  producer: per K-tile reads the descriptor; TMA-loads a dense tile's
//           2 panels (or a sparse tile's 1 value panel + its 2 KB of metadata
//           by bulk copy) into the A ring and the 2 matching 64-k panels of X
//           into the B ring.
//   warp 1  MMA issuer (one thread) and TMEM owner: dense panel -> 4 x
//           tcgen05.mma kind::f16 (K = 16); sparse tile -> tcgen05.cp of the
//           metadata into TMEM, then 4 x tcgen05.mma.sp kind::f16 (K = 32
//           logical); tcgen05.commit releases ring slots and, per output tile,
//           signals the epilogue.
//   warps 2-5 epilogue: tcgen05.ld of the 128 x BT fp32 accumulator, one
//           round to bf16 (nearest even), stores to Y[m][n]; two TMEM
//           accumulators let it drain one output tile while the MMAs of the
//           next one run.
// Every mbarrier wait is bounded in time; when one runs out the kernel sets
// PATCH_DEV_TIMEOUT, the other roles stop at their next wait, the producer
// waits for its copies in flight, the MMA thread for its MMAs, and TMEM is
// freed before the CTA exits.  No cluster multicast is used anywhere.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace patch {
namespace prefill {

using namespace tc;

constexpr int BM = 128;                  // W rows per output tile (MMA M)
constexpr int BT = 240;                  // tokens per output tile (MMA N; 2 x 240 + metadata fit TMEM)
constexpr int NA = 5;                    // A ring: W panels of 128 x 64 bf16
constexpr int NB = 4;                    // B ring: X panels of BT x 64 bf16
constexpr int NE = 4;                    // metadata ring
constexpr int A_BYTES = PATCH_PANEL_BYTES;
constexpr int B_BYTES = BT * 64 * 2;
constexpr int E_BYTES = PATCH_META_TILE_BYTES;
constexpr int THREADS = 192;
constexpr int MAXTK = 256;               // descriptors of one tile row staged in shared memory
constexpr int NACC = 2;                  // accumulators: the epilogue of one tile overlaps the next
constexpr uint32_t TMEM_COLS = 512;      // accumulators at columns 0 and 256, metadata slots at BT..
constexpr uint32_t ACC_STRIDE = 256;
constexpr uint32_t META_COL0 = BT;
static_assert(META_COL0 + 4 * 4 <= ACC_STRIDE && ACC_STRIDE + BT <= TMEM_COLS, "TMEM layout");

constexpr uint32_t IDESC_DENSE = tc::idesc_bf16(BM, BT, false);
constexpr uint32_t IDESC_SPARSE = tc::idesc_bf16(BM, BT, true);

struct Shared {
  alignas(1024) uint8_t a[NA][A_BYTES];
  alignas(1024) uint8_t b[NB][B_BYTES];
  alignas(128) uint8_t e[NE][E_BYTES];
  uint64_t a_full[NA], a_empty[NA], b_full[NB], b_empty[NB], e_full[NE], e_empty[NE];
  uint64_t acc_full[NACC], acc_empty[NACC], drain;
  uint64_t pdesc_full[2];             // descriptor rows, bulk-copied by the producer
  alignas(16) patch_tile_desc pdesc[2][MAXTK];
  uint32_t a_kind[NA];                // tile kind of the panel in each A slot (producer -> MMA)
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t SMEM_BYTES = sizeof(Shared) + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// ---------------------------------------------------------------- roles

struct Args {
  const uint8_t* meta;
  const patch_tile_desc* desc;
  uint16_t* Y;
  int M, N, Tk, n_items;
  uint64_t limit_ns;
  int32_t* status;
  int inject;  // 1: producer stops after the first K-tile (exercises the timeout path)
};

// Descriptor of tile (tn, kt): from the staged row when it fits, else from global memory.
__device__ __forceinline__ patch_tile_desc row_desc(const Shared& s, const Args& p, bool staged, int buf, int tn,
                                                    int kt) {
  return staged ? s.pdesc[buf][kt] : p.desc[int64_t(tn) * p.Tk + kt];
}

__device__ void producer(Shared& s, const CUtensorMap* tmap_x, const CUtensorMap* tmap_w, const Args& p) {
  const int Tn = p.N / BM;
  const bool staged = p.Tk <= MAXTK;
  uint32_t a_i = 0, b_i = 0, e_i = 0, d_i = 0;  // loads issued per ring / descriptor rows staged
  bool ok = true, waited = false;
  // stage the first item's descriptor row
  if (staged && int(blockIdx.x) < p.n_items) {
    const int tn0 = int(blockIdx.x) % Tn;
    mbar_expect_tx(&s.pdesc_full[0], uint32_t(p.Tk * sizeof(patch_tile_desc)));
    bulk_load(s.pdesc[0], p.desc + int64_t(tn0) * p.Tk, uint32_t(p.Tk * sizeof(patch_tile_desc)), &s.pdesc_full[0]);
    ++d_i;
  }
  int it = 0;
  for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++it) {
    const int tn = item % Tn, tb = item / Tn;
    const int buf = it & 1;
    if (staged) {
      if (!(ok = wait_bounded(&s.pdesc_full[buf], (it >> 1) & 1, &s.abort_flag, p.limit_ns, p.status, false)))
        break;
      // prefetch the next item's row into the other buffer (its previous row is done)
      const int next = item + gridDim.x;
      if (next < p.n_items) {
        mbar_expect_tx(&s.pdesc_full[buf ^ 1], uint32_t(p.Tk * sizeof(patch_tile_desc)));
        bulk_load(s.pdesc[buf ^ 1], p.desc + int64_t(next % Tn) * p.Tk, uint32_t(p.Tk * sizeof(patch_tile_desc)),
                  &s.pdesc_full[buf ^ 1]);
        ++d_i;
      }
    }
    // CTAs that share an X block (same tb) or a W tile row (same tn) start
    // their K loop at different tiles, so they do not all hit the same L2 lines
    // at the same moment; the sum order is the only thing that changes
    const int rot = (tn + 7 * tb) % p.Tk;
    for (int j = 0; ok && j < p.Tk; ++j) {
      const int kt = (j + rot) % p.Tk;
      if (p.inject && (item != int(blockIdx.x) || j > 0)) {
        ok = false;
        break;
      }
      const patch_tile_desc d = row_desc(s, p, staged, buf, tn, kt);
      const int panel = int(d.val_offset / A_BYTES);
      if (d.kind) {
        const uint32_t es = e_i % NE;
        if (!(ok = wait_bounded(&s.e_empty[es], ((e_i / NE) & 1) ^ 1, &s.abort_flag, p.limit_ns, p.status, false))) break;
        mbar_expect_tx(&s.e_full[es], E_BYTES);
        bulk_load(s.e[es], p.meta + uint64_t(d.sparse_ordinal) * E_BYTES, E_BYTES, &s.e_full[es]);
        ++e_i;
      }
      const int n_a = d.kind ? 1 : 2;
      for (int h = 0; h < n_a; ++h) {
        const uint32_t as = a_i % NA;
        if (!(ok = wait_bounded(&s.a_empty[as], ((a_i / NA) & 1) ^ 1, &s.abort_flag, p.limit_ns, p.status, false)))
          break;
        s.a_kind[as] = d.kind;  // published to the MMA thread by the barrier's release
        mbar_expect_tx(&s.a_full[as], A_BYTES);
        tma_load_2d(s.a[as], tmap_w, &s.a_full[as], 0, (panel + h) * 128);
        ++a_i;
      }
      if (!ok) break;
      // X may be the previous kernel's output: wait for it before the first X load
      if (!waited) {
        pdl_wait_previous();
        waited = true;
      }
      for (int h = 0; h < 2; ++h) {
        const uint32_t bs = b_i % NB;
        if (!(ok = wait_bounded(&s.b_empty[bs], ((b_i / NB) & 1) ^ 1, &s.abort_flag, p.limit_ns, p.status, false)))
          break;
        mbar_expect_tx(&s.b_full[bs], B_BYTES);
        tma_load_2d(s.b[bs], tmap_x, &s.b_full[bs], kt * kTile + 64 * h, tb * BT);
        ++b_i;
      }
    }
  }
  // every copy issued must have landed before the CTA may exit
  for (uint32_t i = (a_i > NA ? a_i - NA : 0); i < a_i; ++i)
    wait_bounded(&s.a_full[i % NA], (i / NA) & 1, &s.abort_flag, p.limit_ns, p.status, true);
  for (uint32_t i = (b_i > NB ? b_i - NB : 0); i < b_i; ++i)
    wait_bounded(&s.b_full[i % NB], (i / NB) & 1, &s.abort_flag, p.limit_ns, p.status, true);
  for (uint32_t i = (e_i > NE ? e_i - NE : 0); i < e_i; ++i)
    wait_bounded(&s.e_full[i % NE], (i / NE) & 1, &s.abort_flag, p.limit_ns, p.status, true);
  for (uint32_t i = (d_i > 2 ? d_i - 2 : 0); i < d_i; ++i)
    wait_bounded(&s.pdesc_full[i & 1], (i >> 1) & 1, &s.abort_flag, p.limit_ns, p.status, true);
}

__device__ void mma_issuer(Shared& s, uint32_t tmem, const Args& p) {
  uint32_t a_i = 0, b_i = 0, e_i = 0;
  bool ok = true;
  int it = 0;
  for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++it) {
    const int buf = it % NACC;
    if (!(ok = wait_bounded(&s.acc_empty[buf], ((it / NACC) & 1) ^ 1, &s.abort_flag, p.limit_ns, p.status, false)))
      break;
    tc_fence_after();
    const uint32_t acc = tmem + ACC_STRIDE * buf;
    uint32_t accumulate = 0;
    for (int kt = 0; ok && kt < p.Tk; ++kt) {
      // the tile's kind arrives with its first A panel
      uint32_t as = a_i % NA;
      if (!(ok = wait_bounded(&s.a_full[as], (a_i / NA) & 1, &s.abort_flag, p.limit_ns, p.status, false))) break;
      const uint32_t kind = *reinterpret_cast<volatile uint32_t*>(&s.a_kind[as]);
      if (kind) {
        const uint32_t es = e_i % NE;
        if (!(ok = wait_bounded(&s.e_full[es], (e_i / NE) & 1, &s.abort_flag, p.limit_ns, p.status, false))) break;
        tc_fence_after();
        const uint32_t e_tmem = tmem + META_COL0 + 4 * es;
        tmem_cp_128x128b(e_tmem, meta_desc(smem_u32(s.e[es])));
        const uint64_t a0 = sw128_desc(smem_u32(s.a[as]));
        for (int h = 0; h < 2; ++h) {
          const uint32_t bs = b_i % NB;
          if (!(ok = wait_bounded(&s.b_full[bs], (b_i / NB) & 1, &s.abort_flag, p.limit_ns, p.status, false))) break;
          tc_fence_after();
          const uint64_t b0 = sw128_desc(smem_u32(s.b[bs]));
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint32_t kb = 2 * h + j;  // 32-k block of the tile: 16 kept values = 32 B of A
            mma_sparse(acc, a0 + (kb * 32 >> 4), b0 + (j * 64 >> 4), e_tmem + (kb & 2u),
                       IDESC_SPARSE | (kb & 1u), accumulate);
            accumulate = 1;
          }
          tc_commit(&s.b_empty[bs]);
          ++b_i;
        }
        if (!ok) break;
        tc_commit(&s.a_empty[as]);
        ++a_i;
        tc_commit(&s.e_empty[es]);
        ++e_i;
      } else {
        for (int h = 0; h < 2; ++h) {
          as = a_i % NA;
          const uint32_t bs = b_i % NB;
          if (h == 1 &&
              !(ok = wait_bounded(&s.a_full[as], (a_i / NA) & 1, &s.abort_flag, p.limit_ns, p.status, false)))
            break;
          if (!(ok = wait_bounded(&s.b_full[bs], (b_i / NB) & 1, &s.abort_flag, p.limit_ns, p.status, false))) break;
          tc_fence_after();
          const uint64_t a0 = sw128_desc(smem_u32(s.a[as]));
          const uint64_t b0 = sw128_desc(smem_u32(s.b[bs]));
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // K = 16 per MMA = 32 B along the swizzled row
            mma_dense(acc, a0 + (j * 32 >> 4), b0 + (j * 32 >> 4), IDESC_DENSE, accumulate);
            accumulate = 1;
          }
          tc_commit(&s.a_empty[as]);
          ++a_i;
          tc_commit(&s.b_empty[bs]);
          ++b_i;
        }
      }
    }
    if (ok) tc_commit(&s.acc_full[buf]);
  }
  // all MMAs and copies issued must be complete before TMEM is freed
  tc_commit(&s.drain);
  wait_bounded(&s.drain, 0, &s.abort_flag, p.limit_ns, p.status, true);
}

__device__ void epilogue(Shared& s, uint32_t tmem, const Args& p) {
  const int Tn = p.N / BM;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;  // the TMEM lane quarter this warp may access
  int it = 0;
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++it) {
    const int tn = item % Tn, tb = item / Tn;
    const int buf = it % NACC;
    if (!wait_bounded(&s.acc_full[buf], (it / NACC) & 1, &s.abort_flag, p.limit_ns, p.status, false)) break;
    tc_fence_after();
    const int64_t n = int64_t(tn) * BM + 32 * q + lane;
    const int m0 = tb * BT;
    const uint32_t acc = tmem + (uint32_t(32 * q) << 16) + ACC_STRIDE * buf;
    for (int c = 0; c < BT / 16; ++c) {
      if (m0 + 16 * c >= p.M) break;  // warp-uniform
      uint32_t v[16];
      tmem_ld_16cols(acc + uint32_t(16 * c), v);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int m = m0 + 16 * c + j;
        if (m < p.M) p.Y[int64_t(m) * p.N + n] = f32_to_bf16_rne(__uint_as_float(v[j]));
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.acc_empty[buf]);
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                   const Args p) {
  extern __shared__ uint8_t smem_raw[];
  Shared& s = *reinterpret_cast<Shared*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();  // the next kernel may run its prologue as our CTAs finish

  if (threadIdx.x == 0) {
    for (int i = 0; i < NA; ++i) {
      mbar_init(&s.a_full[i], 1);
      mbar_init(&s.a_empty[i], 1);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(&s.b_full[i], 1);
      mbar_init(&s.b_empty[i], 1);
    }
    for (int i = 0; i < NE; ++i) {
      mbar_init(&s.e_full[i], 1);
      mbar_init(&s.e_empty[i], 1);
    }
    for (int i = 0; i < NACC; ++i) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 4);
    }
    mbar_init(&s.drain, 1);
    mbar_init(&s.pdesc_full[0], 1);
    mbar_init(&s.pdesc_full[1], 1);
    s.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s.tmem_base)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    if (lane == 0) producer(s, &tmap_x, &tmap_w, p);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_issuer(s, tmem, p);
    __syncwarp();
  } else {
    epilogue(s, tmem, p);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                 : "memory");
  }
}

}  // namespace prefill

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D bf16 tensor map, 128-byte swizzle, out-of-bounds reads fill zeros.
bool make_map_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                        uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_prefill(const uint16_t* X, int64_t M, const patch_weight& W, uint16_t* Y,
                           int32_t* status, int num_sms, uint64_t limit_ns, int inject,
                           cudaStream_t stream) {
  using namespace prefill;
  const int64_t Tn = W.N / BM, Tk = W.K / kTile, T = Tn * Tk;
  const uint64_t n_panels = uint64_t(2 * (T - W.n_sparse) + W.n_sparse);
  CUtensorMap tmap_x, tmap_w;
  if (!make_map_2d_bf16(&tmap_x, X, uint64_t(W.K), uint64_t(M), uint64_t(W.K) * 2, 64, BT)) return cudaErrorUnknown;
  if (!make_map_2d_bf16(&tmap_w, W.values, 64, n_panels * 128, 128, 64, 128)) return cudaErrorUnknown;
  Args p;
  p.meta = static_cast<const uint8_t*>(W.meta);
  p.desc = W.desc;
  p.Y = Y;
  p.M = int(M);
  p.N = int(W.N);
  p.Tk = int(Tk);
  p.n_items = int(Tn * ((M + BT - 1) / BT));
  p.limit_ns = limit_ns;
  p.status = status;
  p.inject = inject;
  const int grid = p.n_items < num_sms ? p.n_items : num_sms;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  return launch_pdl(prefill_kernel, dim3(unsigned(grid)), dim3(THREADS), SMEM_BYTES, stream, tmap_x, tmap_w, p);
}

}  // namespace patch
