// Prefill path of patch_gemm (M > 16): a persistent, warp-specialised
// TMA + tcgen05 kernel for sm_100a in which dense tiles run on the dense
// tensor-core MMA and 2:4 sparse tiles on the structured-sparse MMA, both
// accumulating into fp32 tiles in tensor memory.
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
// Work unit = two tile rows (2 x 128 output features, rows rp and rp + Tn/2)
// x BT tokens.  Both rows
// multiply the same X panels, so one 30 KiB X panel in shared memory feeds
// two MMA chains; each row keeps its own kind per K-tile (dense or sparse),
// so the two rows of a unit never need to agree.  Per byte brought in from L2
// this does 1.5x (dense) to 1.6x (sparse) the tensor-core work of a one-row
// tile, which is what bounds a 128-row tile on this GPU.
//
// CTA = 16 warps, one CTA per SM, static round-robin over units
// (row pair rp, token block tb):
//   warps 0, 2  W producers of rows 0 and 1: per K-tile the row's descriptor
//           (staged in shared memory); a sparse tile's 2 KiB of metadata by
//           bulk copy; the W panels (2 per dense tile, 1 per sparse tile) by
//           TMA into the row's A ring.
//   warps 1, 3  MMA issuers of rows 0 and 1 (one thread each; warp 1 owns
//           TMEM): dense panel -> 4 x tcgen05.mma kind::f16 (K = 16); sparse
//           tile -> tcgen05.cp of the metadata into TMEM, then 4 x
//           tcgen05.mma.sp kind::f16 (K = 32 logical); tcgen05.commit
//           releases ring slots and, per unit, signals the row's epilogue.
//           One issuing thread for both rows cannot keep the tensor core
//           busy: every wait, commit and MMA issue is a long-latency
//           instruction in one serial chain.
//   warp 4  X producer: TMA-loads the 2 matching 64-k panels of X per K-tile
//           into the B ring shared by both rows.
//   warps 8-15 epilogue: warps 8-11 drain row 0's accumulator, 12-15 row 1's
//           (each warp its TMEM lane quarter): tcgen05.ld, one round to bf16
//           (nearest even), stores to Y[m][n].
// Tensor memory: row 0's accumulator at columns 0..BT-1, row 1's at 256..,
// metadata slots of 4 columns after each.  The two accumulators use all of
// it, so a unit's epilogue does not overlap the next unit's MMAs; the
// producer keeps loading meanwhile, so the rings are full when they restart.
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

constexpr int BM = 128;                  // W rows per tile row (MMA M)
constexpr int ROWS = 2;                  // tile rows per unit, sharing the X panels
constexpr int BT = 240;                  // most tokens per unit (MMA N); each launch picks bt <= BT
constexpr int NA = 3;                    // A ring per row: W panels of 128 x 64 bf16
constexpr int NB = 3;                    // B ring: X panels of BT x 64 bf16
constexpr int NE = 2;                    // metadata ring per row
constexpr int A_BYTES = PATCH_PANEL_BYTES;
constexpr int B_BYTES = BT * 64 * 2;
constexpr int E_BYTES = PATCH_META_TILE_BYTES;
constexpr int EPI_WARP0 = 8;             // warps 8-11 drain row 0, 12-15 row 1
constexpr int YT = 16;                   // tokens per chunk of the split-K epilogue
constexpr int YC = 32;                   // tokens per chunk of the whole-K epilogue (one 32-column TMEM load)
constexpr int THREADS = 32 * (EPI_WARP0 + 4 * ROWS);
constexpr int MAXTK = 128;               // descriptors of one tile row staged in shared memory (K <= 16384)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_STRIDE = 256;     // row r's accumulator at column 256 r
constexpr uint32_t META_COL0 = BT;       // row r's metadata slot e at column 256 r + BT + 4 e
static_assert(META_COL0 + 4 * NE <= ACC_STRIDE && ACC_STRIDE + BT <= TMEM_COLS, "TMEM layout");
static_assert(B_BYTES % 1024 == 0, "X panels keep the 1024-byte alignment of the 128-byte swizzle");


struct Shared {
  alignas(1024) uint8_t a[ROWS][NA][A_BYTES];
  alignas(1024) uint8_t b[NB][B_BYTES];
  alignas(128) uint8_t e[ROWS][NE][E_BYTES];
  uint64_t a_full[ROWS][NA], a_empty[ROWS][NA], e_full[ROWS][NE], e_empty[ROWS][NE];
  uint64_t b_full[NB], b_empty[NB];   // b_empty: one arrival per row's MMA thread
  uint64_t acc_full[ROWS], acc_empty[ROWS], drain[ROWS];
  uint64_t pdesc_full[ROWS][2];       // descriptor rows, bulk-copied by each row's producer
  alignas(16) patch_tile_desc pdesc[ROWS][2][MAXTK];
  uint32_t a_kind[ROWS][NA];          // tile kind of the panel in each A slot (producer -> MMA)
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t SMEM_BYTES = sizeof(Shared) + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct Args {
  const uint8_t* meta[ROWS];          // row r of a unit reads weight r (the same weight unless mlp)
  const patch_tile_desc* desc[ROWS];
  int mlp;                            // 1: row 0 = gate, row 1 = up tile row rp; Y = silu(gate) * up
  uint16_t* Y;
  int M, N, Tn, Tk, n_pairs, n_tb, n_items;  // units: see unit_of()
  int ks;                      // K parts per output block (split K; 1 = whole K per unit)
  float* part;                 // ks > 1: fp32 partials [block][ks][ROWS][bt][128]
  uint32_t* counters;          // ks > 1: arrivals [block][ROWS][4] (zero between calls)
  int bt;                      // tokens per unit: a multiple of 16, at most BT
  uint32_t idesc_dense, idesc_sparse;
  uint64_t limit_ns;
  int32_t* status;
  int inject;  // 1: row 0's producer stops after the first K-tile (exercises the timeout path)
};

// Row pair rp holds tile rows rp and rp + n_pairs (n_pairs = ceil(Tn / 2);
// the last pair of an odd Tn has one row).  A unit costs the sum of its two
// rows' MMA time, so pairing each row with the one half the layer away keeps
// unit costs even when sparse tiles come in bands of tile rows (a band of half
// the rows puts exactly one row of every pair inside it), where neighbouring
// rows would pair dense with dense and sparse with sparse and a one-wave grid
// would wait for the dense pairs.  A gated-MLP unit is gate and up tile row rp.
__device__ __forceinline__ int rows_of(const Args& p, int rp) {
  return p.mlp ? ROWS : (rp + p.n_pairs < p.Tn ? ROWS : 1);
}
// the tile row of its weight that row r of unit row pair rp reads
__device__ __forceinline__ int tile_row(const Args& p, int rp, int r) { return p.mlp ? rp : rp + r * p.n_pairs; }

// Units run row pair by row pair (all token blocks of a pair are consecutive
// items), so the CTAs of one wave read a few row pairs' W, which stays in L2
// while every token block uses it, instead of every wave reading all of W.
// Units that share an X block (same tb) or W rows (same rp) start their K loop
// at different tiles, so they do not all hit the same L2 lines at the same
// moment; only the order of the fp32 sum changes.
__device__ __forceinline__ int k_rotation(int rp, int tb, int Tk) { return (rp + 7 * tb) % Tk; }

// Work unit `item`: output block blk = (row pair rp, token block tb) and its K
// part kp, which covers K-tiles [k0, k0 + len).  With ks = 1 a unit is a whole
// output block (item = blk).  The K loop starts at a rotated tile of the part.
struct Unit {
  int blk, kp, rp, tb, k0, len, rot;
};
__device__ __forceinline__ Unit unit_of(const Args& p, int item) {
  Unit u;
  u.blk = item / p.ks;
  u.kp = item - u.blk * p.ks;
  u.rp = u.blk / p.n_tb;
  u.tb = u.blk - u.rp * p.n_tb;
  u.k0 = int(int64_t(u.kp) * p.Tk / p.ks);
  u.len = int(int64_t(u.kp + 1) * p.Tk / p.ks) - u.k0;
  u.rot = k_rotation(u.rp, u.tb, u.len);
  return u;
}

// ---------------------------------------------------------------- roles

// W producer of row r: the row's descriptors, metadata and W panels.  It never
// touches X, so it may run ahead of the previous kernel in the stream (W, the
// metadata and the descriptors are inputs that no kernel triggering an early
// launch writes).
__device__ void producer_w(Shared& s, const CUtensorMap* tmap_w, const Args& p, int r) {
  const patch_tile_desc* desc = r ? p.desc[1] : p.desc[0];
  const uint8_t* meta = r ? p.meta[1] : p.meta[0];
  const bool staged = p.Tk <= MAXTK;
  const uint32_t row_bytes = uint32_t(p.Tk * sizeof(patch_tile_desc));
  uint32_t a_i = 0, e_i = 0, d_i = 0;  // loads issued per ring / descriptor rows staged
  bool ok = true;
  // stage (or, for a pair without row r, complete with no bytes) the descriptor row of an item
  auto stage_row = [&](int item, int buf) {
    const int rp = unit_of(p, item).rp;
    const bool has = r < rows_of(p, rp);
    mbar_expect_tx(&s.pdesc_full[r][buf], has ? row_bytes : 0u);
    if (has) bulk_load(s.pdesc[r][buf], desc + int64_t(tile_row(p, rp, r)) * p.Tk, row_bytes, &s.pdesc_full[r][buf]);
    ++d_i;
  };
  if (staged && int(blockIdx.x) < p.n_items) stage_row(blockIdx.x, 0);
  int it = 0;
  for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++it) {
    const Unit u = unit_of(p, item);
    const int rp = u.rp, tn = tile_row(p, rp, r);
    const int buf = it & 1;
    if (staged) {
      if (!(ok = wait_bounded(&s.pdesc_full[r][buf], (it >> 1) & 1, &s.abort_flag, p.limit_ns, p.status, false)))
        break;
      // prefetch the next unit's row into the other buffer (its previous row is done)
      if (item + int(gridDim.x) < p.n_items) stage_row(item + gridDim.x, buf ^ 1);
    }
    if (r >= rows_of(p, rp)) continue;
    int kt = u.k0 + u.rot;
    for (int j = 0; ok && j < u.len; ++j, kt = (kt + 1 == u.k0 + u.len ? u.k0 : kt + 1)) {
      if (p.inject && r == 0 && (item != int(blockIdx.x) || j > 0)) {
        ok = false;
        break;
      }
      const patch_tile_desc d = staged ? s.pdesc[r][buf][kt] : desc[int64_t(tn) * p.Tk + kt];
      if (d.kind) {
        const uint32_t es = e_i % NE;
        if (!(ok = wait_bounded(&s.e_empty[r][es], ((e_i / NE) & 1) ^ 1, &s.abort_flag, p.limit_ns, p.status, false)))
          break;
        mbar_expect_tx(&s.e_full[r][es], E_BYTES);
        bulk_load(s.e[r][es], meta + uint64_t(d.sparse_ordinal) * E_BYTES, E_BYTES, &s.e_full[r][es]);
        ++e_i;
      }
      // a dense tile's 2 panels (one per 64-k half), a sparse tile's one
      const int panel = int(d.val_offset / A_BYTES);
      for (int h = 0; h < (d.kind ? 1 : 2); ++h) {
        const uint32_t as = a_i % NA;
        if (!(ok = wait_bounded(&s.a_empty[r][as], ((a_i / NA) & 1) ^ 1, &s.abort_flag, p.limit_ns, p.status, false)))
          break;
        s.a_kind[r][as] = d.kind;  // published to the MMA thread by the barrier's release
        mbar_expect_tx(&s.a_full[r][as], A_BYTES);
        tma_load_2d(s.a[r][as], tmap_w, &s.a_full[r][as], 0, (panel + h) * 128);
        ++a_i;
      }
    }
  }
  // every copy issued must have landed before the CTA may exit
  for (uint32_t i = (a_i > NA ? a_i - NA : 0); i < a_i; ++i)
    wait_bounded(&s.a_full[r][i % NA], (i / NA) & 1, &s.abort_flag, p.limit_ns, p.status, true);
  for (uint32_t i = (e_i > NE ? e_i - NE : 0); i < e_i; ++i)
    wait_bounded(&s.e_full[r][i % NE], (i / NE) & 1, &s.abort_flag, p.limit_ns, p.status, true);
  for (uint32_t i = (d_i > 2 ? d_i - 2 : 0); i < d_i; ++i)
    wait_bounded(&s.pdesc_full[r][i & 1], (i >> 1) & 1, &s.abort_flag, p.limit_ns, p.status, true);
}

// X producer: the two 64-k panels of X per K-tile, in the same rotated K order.
__device__ void producer_x(Shared& s, const CUtensorMap* tmap_x, const Args& p) {
  uint32_t b_i = 0;
  bool ok = true;
  // X may be the previous kernel's output: wait for it before the first X load
  pdl_wait_previous();
  for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
    const Unit u = unit_of(p, item);
    const int tb = u.tb;
    int kt = u.k0 + u.rot;
    for (int j = 0; ok && j < u.len; ++j, kt = (kt + 1 == u.k0 + u.len ? u.k0 : kt + 1)) {
      for (int h = 0; ok && h < 2; ++h) {
        const uint32_t bs = b_i % NB;
        if (!(ok = wait_bounded(&s.b_empty[bs], ((b_i / NB) & 1) ^ 1, &s.abort_flag, p.limit_ns, p.status, false)))
          break;
        mbar_expect_tx(&s.b_full[bs], uint32_t(p.bt) * 128u);
        tma_load_2d(s.b[bs], tmap_x, &s.b_full[bs], kt * kTile + 64 * h, tb * p.bt);
        ++b_i;
      }
    }
  }
  for (uint32_t i = (b_i > NB ? b_i - NB : 0); i < b_i; ++i)
    wait_bounded(&s.b_full[i % NB], (i / NB) & 1, &s.abort_flag, p.limit_ns, p.status, true);
}

// MMA issuer of row r (one thread): each row has its own issuing thread, so
// the two chains' barrier waits, commits and bookkeeping overlap and the
// tensor core, shared by both, stays fed.  Both consume the same X slots; a
// slot is free once both rows' MMAs on it are complete (two commits).
__device__ void mma_issuer(Shared& s, uint32_t tmem, const Args& p, int r) {
  const uint32_t acc = tmem + ACC_STRIDE * r;
  uint32_t a_i = 0, b_i = 0, e_i = 0;
  bool ok = true;
  int it = 0;
  for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++it) {
    const Unit u = unit_of(p, item);
    const bool active = r < rows_of(p, u.rp);
    if (!(ok = wait_bounded(&s.acc_empty[r], (it & 1) ^ 1, &s.abort_flag, p.limit_ns, p.status, false))) break;
    tc_fence_after();
    uint32_t accumulate = 0;
    for (int kt = 0; ok && kt < u.len; ++kt) {
      uint32_t kind = 0, as = 0, es = 0;
      for (int h = 0; h < 2; ++h) {
        // the tile's kind arrives with its first panel; a sparse tile's one
        // panel serves both halves and its metadata goes to TMEM first
        if (active && (h == 0 || !kind)) {
          as = a_i % NA;
          if (!(ok = wait_bounded(&s.a_full[r][as], (a_i / NA) & 1, &s.abort_flag, p.limit_ns, p.status, false)))
            break;
          ++a_i;
          if (h == 0) kind = *reinterpret_cast<volatile uint32_t*>(&s.a_kind[r][as]);
          if (h == 0 && kind) {
            es = e_i % NE;
            if (!(ok = wait_bounded(&s.e_full[r][es], (e_i / NE) & 1, &s.abort_flag, p.limit_ns, p.status, false)))
              break;
            ++e_i;
            tc_fence_after();
            tmem_cp_128x128b(acc + META_COL0 + 4 * es, meta_desc(smem_u32(s.e[r][es])));
          }
        }
        const uint32_t bs = b_i % NB;
        if (!(ok = wait_bounded(&s.b_full[bs], (b_i / NB) & 1, &s.abort_flag, p.limit_ns, p.status, false))) break;
        ++b_i;
        if (!active) {  // the pair's missing row only paces the X ring
          mbar_arrive(&s.b_empty[bs]);
          continue;
        }
        tc_fence_after();
        const uint64_t a0 = sw128_desc(smem_u32(s.a[r][as]));
        const uint64_t b0 = sw128_desc(smem_u32(s.b[bs]));
        if (kind) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint32_t kb = 2 * h + j;  // 32-k block of the tile: 16 kept values = 32 B of A
            mma_sparse(acc, a0 + (kb * 32 >> 4), b0 + (j * 64 >> 4), acc + META_COL0 + 4 * es + (kb & 2u),
                       p.idesc_sparse | (kb & 1u), accumulate);
            accumulate = 1;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // K = 16 per MMA = 32 B along the swizzled row
            mma_dense(acc, a0 + (j * 32 >> 4), b0 + (j * 32 >> 4), p.idesc_dense, accumulate);
            accumulate = 1;
          }
        }
        tc_commit(&s.b_empty[bs]);
        if (!kind) {
          tc_commit(&s.a_empty[r][as]);
        } else if (h == 1) {
          tc_commit(&s.a_empty[r][as]);
          tc_commit(&s.e_empty[r][es]);
        }
      }
    }
    if (ok) {
      if (active)
        tc_commit(&s.acc_full[r]);
      else
        mbar_arrive(&s.acc_full[r]);
    }
  }
  // all MMAs and copies issued must be complete before TMEM is freed
  tc_commit(&s.drain[r]);
  wait_bounded(&s.drain[r], 0, &s.abort_flag, p.limit_ns, p.status, true);
}

// Epilogue warp groups (4 warps each, one per TMEM lane quarter): per chunk
// of YC tokens, each warp loads its 32 features x YC tokens from TMEM (one
// load), rounds to bf16 and stores them to Y from registers: per token, the
// warp's 32 features are 64 contiguous bytes.  No shared-memory staging, so
// no barrier or wait on an earlier store per chunk.  Group g drains row g of
// the pair; for the gated MLP both groups read both rows (gate and up of the
// same 128 features) and take every other chunk: Y = silu(gate) * up.
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* a, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(a), "r"(v) : "memory");
  return old;
}

// Split K (ks > 1): the unit's fp32 accumulator of row g goes to its slot of
// the workspace, token-major ([bt][128]: a warp's 32 rows of one token are
// 128 contiguous bytes, for its stores and for the reduction's loads), the
// accumulator is released, and the last of the block's ks units to arrive
// (counted per row and TMEM lane quarter, acquire-release) adds the ks
// partials in K-part order (deterministic), stores Y and resets the counter.
__device__ void epilogue_split(Shared& s, uint32_t tmem, const Args& p, const Unit& u, int g, int q, int lane) {
  const bool has = g < rows_of(p, u.rp);
  const int row = 32 * q + lane;
  const int64_t n = int64_t(tile_row(p, u.rp, g)) * BM + row;
  const int m0 = u.tb * p.bt;
  const int valid = p.M - m0 < p.bt ? p.M - m0 : p.bt;  // tokens of this block inside X
  const int64_t slot_floats = int64_t(BM) * p.bt;        // one row g of one unit
  const int64_t blk_base = int64_t(u.blk) * p.ks * ROWS;
  if (has) {
    float* mine = p.part + ((blk_base + int64_t(u.kp) * ROWS + g) * slot_floats) + row;
    const uint32_t lanes = tmem + (uint32_t(32 * q) << 16) + ACC_STRIDE * g;
    for (int c = 0; c * YT < valid; ++c) {
      uint32_t v[YT];
      tmem_ld_16cols(lanes + uint32_t(YT * c), v);
#pragma unroll
      for (int j = 0; j < YT; ++j) __stcg(mine + int64_t(YT * c + j) * BM, __uint_as_float(v[j]));
    }
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&s.acc_empty[g]);
  if (!has) return;
  // the warp's partial stores are ordered before lane 0's release-acquire increment
  uint32_t* counter = p.counters + (int64_t(u.blk) * ROWS + g) * 4 + q;
  uint32_t old = 0;
  if (lane == 0) old = atom_add_acq_rel_gpu(counter, 1u);
  old = __shfl_sync(0xFFFFFFFFu, old, 0);
  if (old != uint32_t(p.ks - 1)) return;
  __syncwarp();  // orders lane 0's acquire before every lane's loads
  for (int c = 0; c * YT < valid; ++c) {
    float sum[YT];
#pragma unroll
    for (int j = 0; j < YT; ++j) sum[j] = 0.0f;
    for (int kp = 0; kp < p.ks; ++kp) {
      const float* src = p.part + ((blk_base + int64_t(kp) * ROWS + g) * slot_floats) + int64_t(YT * c) * BM + row;
      float part[YT];
#pragma unroll
      for (int j = 0; j < YT; ++j) part[j] = __ldcg(src + int64_t(j) * BM);
#pragma unroll
      for (int j = 0; j < YT; ++j) sum[j] += part[j];
    }
#pragma unroll
    for (int j = 0; j < YT; ++j)
      if (YT * c + j < valid) p.Y[int64_t(m0 + YT * c + j) * p.N + n] = f32_to_bf16_rne(sum[j]);
  }
  if (lane == 0) *counter = 0;  // ready for the next call
}

__device__ void epilogue(Shared& s, uint32_t tmem, const Args& p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;                  // the TMEM lane quarter this warp may access
  const int g = (warp - EPI_WARP0) >> 2;   // warp group
  const uint32_t bar_id = 1 + g;           // named barrier of the group's 128 threads
  int it = 0;
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++it) {
    const Unit u = unit_of(p, item);
    const int rp = u.rp, tb = u.tb;
    // the four warps of a group take the same decision, so none is left at a barrier
    bool ok = wait_bounded(&s.acc_full[g], it & 1, &s.abort_flag, p.limit_ns, p.status, false);
    if (p.mlp) ok = ok && wait_bounded(&s.acc_full[g ^ 1], it & 1, &s.abort_flag, p.limit_ns, p.status, false);
    if (!named_bar_and(bar_id, 128, ok)) break;
    tc_fence_after();
    if (p.ks > 1) {  // split K (never with the gated MLP)
      epilogue_split(s, tmem, p, u, g, q, lane);
      continue;
    }
    if (p.mlp || g < rows_of(p, rp)) {
      const int n0 = tile_row(p, rp, g) * BM, m0 = tb * p.bt;
      const int valid = p.M - m0 < p.bt ? p.M - m0 : p.bt;  // tokens of this unit inside X
      const uint32_t lanes = tmem + (uint32_t(32 * q) << 16);
      const int c0 = p.mlp ? g : 0, dc = p.mlp ? 2 : 1;
      // this thread's feature; a warp's 32 stores of one token fill 64 contiguous bytes of Y
      uint16_t* yp = p.Y + int64_t(m0) * p.N + n0 + 32 * q + lane;
      for (int c = c0; c * YC < valid; c += dc) {
        uint32_t v[YC];
        if (p.mlp) {
#pragma unroll
          for (int hh = 0; hh < YC / 16; ++hh) {  // in 16-column halves (registers)
            uint32_t gt[16], u[16];
            tmem_ld_16cols(lanes + uint32_t(YC * c + 16 * hh), gt);               // gate
            tmem_ld_16cols(lanes + ACC_STRIDE + uint32_t(YC * c + 16 * hh), u);   // up
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              // silu(gate) = gate / (1 + e^-gate), with CUDA's fast exponential and
              // division (relative error ~1e-6, far below the bf16 rounding of H);
              // a huge denominator gives -0 for a very negative gate
              const float gate = __uint_as_float(gt[j]);
              v[16 * hh + j] = __float_as_uint(__fdividef(gate, 1.0f + __expf(-gate)) * __uint_as_float(u[j]));
            }
          }
        } else {
          tmem_ld_32cols(lanes + ACC_STRIDE * g + uint32_t(YC * c), v);
        }
        uint16_t* yr = yp + int64_t(YC * c) * p.N;
        const int nj = valid - YC * c < YC ? valid - YC * c : YC;
#pragma unroll
        for (int j = 0; j < YC; ++j, yr += p.N)
          if (j < nj) *yr = f32_to_bf16_rne(__uint_as_float(v[j]));
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&s.acc_empty[g]);
      if (p.mlp) mbar_arrive(&s.acc_empty[g ^ 1]);
    }
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w0,
                   const __grid_constant__ CUtensorMap tmap_w1,
                   const Args p) {
  extern __shared__ uint8_t smem_raw[];
  Shared& s = *reinterpret_cast<Shared*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();  // the next kernel may run its prologue as our CTAs finish

  if (threadIdx.x == 0) {
    for (int r = 0; r < ROWS; ++r) {
      for (int i = 0; i < NA; ++i) {
        mbar_init(&s.a_full[r][i], 1);
        mbar_init(&s.a_empty[r][i], 1);
      }
      for (int i = 0; i < NE; ++i) {
        mbar_init(&s.e_full[r][i], 1);
        mbar_init(&s.e_empty[r][i], 1);
      }
      mbar_init(&s.acc_full[r], 1);
      mbar_init(&s.acc_empty[r], p.mlp ? 8 : 4);  // the gated MLP's groups both read both rows
      mbar_init(&s.drain[r], 1);
      mbar_init(&s.pdesc_full[r][0], 1);
      mbar_init(&s.pdesc_full[r][1], 1);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(&s.b_full[i], 1);
      mbar_init(&s.b_empty[i], ROWS);
    }
    s.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensormap(&tmap_x);
    prefetch_tensormap(&tmap_w0);
    prefetch_tensormap(&tmap_w1);
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

  // warps 0/2: W producers of rows 0/1; 1/3: MMA issuers of rows 0/1; 4: X producer
  if (warp < 4) {
    if (lane == 0) {
      if (warp & 1)
        mma_issuer(s, tmem, p, warp >> 1);
      else
        producer_w(s, (warp >> 1) ? &tmap_w1 : &tmap_w0, p, warp >> 1);
    }
    __syncwarp();
  } else if (warp == 4) {
    if (lane == 0) producer_x(s, &tmap_x, p);
    __syncwarp();
  } else if (warp >= EPI_WARP0) {
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

// As make_map_2d_bf16 with the 64-byte swizzle (box_inner * 2 <= 64).
bool make_map_2d_bf16_sw64(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                           uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// Tokens per unit: the multiple of 16 in [64, BT] that minimises the time of
// the slowest CTA, modelled as (units per CTA, rounded up) x (unit time).  A
// unit's K-tile costs the larger of its tensor-core cycles (8 bt: 2 rows x
// 128 K at 8192 FLOP per cycle) and the cycles to bring its 64 KiB of W plus
// 256 bt bytes of X from L2 at about 64 B per cycle; a unit adds ~4000 cycles
// of pipeline fill and epilogue.  Ties go to the larger bt.
// Launch plan: tokens per unit (bt) and K parts per output block (ks).  Cost
// model in SM cycles: waves x per-unit time, a unit's K-tile costing the larger
// of its MMAs (8 bt) and its weight feed (1024 + 4 bt), plus a fixed 4000; a
// split unit also stores its fp32 partial and one of the ks reads all of them
// back (32 bt cycles per partial, and 8000 for the hand-over), constants fitted
// to LLaMA-2-7B q, gate and down timings at M = 17 ... 512.  K is split only
// to fill one wave of otherwise idle SMs, with at least 4 K-tiles per part.
struct PrefillPlan {
  int bt, ks;
  int64_t n_pairs, n_tb;
  size_t part_bytes;  // split-K partials (0 when ks == 1)
};

static PrefillPlan prefill_plan(int64_t M, int64_t n_pairs, int64_t Tk, int num_sms, bool allow_split) {
  using prefill::BT;
  PrefillPlan best{BT, 1, n_pairs, 0, 0};
  int64_t best_cost = -1;
  for (int bt = BT; bt >= 64; bt -= 16) {
    const int64_t units = n_pairs * ((M + bt - 1) / bt);
    const int64_t mma = 8 * bt, feed = 1024 + 4 * bt, per_tile = mma > feed ? mma : feed;
    for (int ks = 1; ks <= (allow_split ? 4 : 1); ++ks) {
      if (ks > 1 && (units * ks > num_sms || Tk / ks < 4)) break;
      const int64_t waves = (units * ks + num_sms - 1) / num_sms;
      const int64_t cost = waves * ((Tk + ks - 1) / ks * per_tile + 4000 + (ks > 1 ? (ks + 1) * 32 * bt + 8000 : 0));
      if (best_cost < 0 || cost < best_cost) {
        best_cost = cost;
        best.bt = bt;
        best.ks = ks;
      }
    }
  }
  best.n_tb = (M + best.bt - 1) / best.bt;
  best.part_bytes = best.ks > 1 ? size_t(n_pairs * best.n_tb * best.ks) * prefill::ROWS * prefill::BM * best.bt * 4 : 0;
  return best;
}

size_t prefill_workspace_bytes(int64_t M, const patch_weight& W, int num_sms) {
  const PrefillPlan pl = prefill_plan(M, (W.N / prefill::BM + prefill::ROWS - 1) / prefill::ROWS, W.K / kTile,
                                      num_sms, true);
  return pl.ks > 1 ? kDecodeCounterBytes + pl.part_bytes : 0;
}

// Shared by the plain GEMM (w1 == w0, units of two consecutive tile rows) and
// the gated MLP (w0 = gate, w1 = up, units of one tile row of each).
static cudaError_t launch_prefill_impl(const uint16_t* X, int64_t M, const patch_weight& W0, const patch_weight& W1,
                                       bool mlp, uint16_t* Y, void* workspace, size_t workspace_bytes,
                                       int32_t* status, int num_sms, uint64_t limit_ns, int inject,
                                       cudaStream_t stream) {
  using namespace prefill;
  const int64_t Tn = W0.N / BM, Tk = W0.K / kTile;
  const int64_t n_pairs = mlp ? Tn : (Tn + ROWS - 1) / ROWS;
  // split K only when the caller's workspace holds the partials (and never for the gated MLP)
  PrefillPlan plan = prefill_plan(M, n_pairs, Tk, num_sms, !mlp);
  if (plan.ks > 1 && (!workspace || workspace_bytes < kDecodeCounterBytes + plan.part_bytes))
    plan = prefill_plan(M, n_pairs, Tk, num_sms, false);
  const int bt = plan.bt;
  CUtensorMap tmap_x, tmap_w0, tmap_w1;
  if (!make_map_2d_bf16(&tmap_x, X, uint64_t(W0.K), uint64_t(M), uint64_t(W0.K) * 2, 64, uint32_t(bt)))
    return cudaErrorUnknown;
  const patch_weight* Ws[2] = {&W0, &W1};
  CUtensorMap* maps[2] = {&tmap_w0, &tmap_w1};
  for (int r = 0; r < 2; ++r) {
    const int64_t T = (Ws[r]->N / BM) * Tk;
    const uint64_t n_panels = uint64_t(2 * (T - Ws[r]->n_sparse) + Ws[r]->n_sparse);
    if (!make_map_2d_bf16(maps[r], Ws[r]->values, 64, n_panels * 128, 128, 64, 128)) return cudaErrorUnknown;
  }
  Args p;
  for (int r = 0; r < ROWS; ++r) {
    p.meta[r] = static_cast<const uint8_t*>(Ws[r]->meta);
    p.desc[r] = Ws[r]->desc;
  }
  p.mlp = mlp ? 1 : 0;
  p.Y = Y;
  p.M = int(M);
  p.N = int(Tn * BM);
  p.Tn = int(Tn);
  p.Tk = int(Tk);
  p.n_pairs = int(n_pairs);
  p.n_tb = int(plan.n_tb);
  p.ks = plan.ks;
  p.n_items = int(n_pairs) * p.n_tb * p.ks;
  p.bt = bt;
  p.counters = static_cast<uint32_t*>(workspace);  // the fixed counter region at the start (used when ks > 1)
  p.part = plan.ks > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kDecodeCounterBytes) : nullptr;
  p.idesc_dense = tc::idesc_bf16(BM, bt, false);
  p.idesc_sparse = tc::idesc_bf16(BM, bt, true);
  p.limit_ns = limit_ns;
  p.status = status;
  p.inject = inject;
  const int grid = p.n_items < num_sms ? p.n_items : num_sms;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  return launch_pdl(prefill_kernel, dim3(unsigned(grid)), dim3(THREADS), SMEM_BYTES, stream, tmap_x, tmap_w0, tmap_w1,
                    p);
}

cudaError_t launch_prefill(const uint16_t* X, int64_t M, const patch_weight& W, uint16_t* Y, void* workspace,
                           size_t workspace_bytes, int32_t* status, int num_sms, uint64_t limit_ns, int inject,
                           cudaStream_t stream) {
  return launch_prefill_impl(X, M, W, W, false, Y, workspace, workspace_bytes, status, num_sms, limit_ns, inject,
                             stream);
}

cudaError_t launch_prefill_mlp(const uint16_t* X, int64_t M, const patch_weight& W_gate, const patch_weight& W_up,
                               uint16_t* H, int32_t* status, int num_sms, uint64_t limit_ns, cudaStream_t stream) {
  return launch_prefill_impl(X, M, W_gate, W_up, true, H, nullptr, 0, status, num_sms, limit_ns, 0, stream);
}

}  // namespace patch
