// Prefill path of patch_gemm (M > 16), patch_gemm_mlp and patch_gemm_group:
// a persistent, warp-specialised TMA + tcgen05 kernel for sm_100a in which
// dense tiles run on the dense tensor-core MMA and 2:4 sparse tiles on the
// structured-sparse MMA, both accumulating into fp32 tiles in tensor memory.
// One launch runs the units of one GEMM, or of a group of independent GEMMs
// (a table of them in the kernel parameters, with a host-balanced list of
// units per CTA).
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

#include <algorithm>
#include <memory>
#include <vector>

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

// One GEMM of a launch.  A launch runs one GEMM (patch_gemm, the gated MLP)
// or a group of independent ones (patch_gemm_group) whose units share the
// CTAs: items [item0, next GEMM's item0) are this GEMM's units.
struct Gemm {
  const uint8_t* meta;
  const patch_tile_desc* desc;
  uint16_t* Y;
  int M, N, Tn, Tk, n_pairs, n_tb;  // units: see unit_of()
  int bt;                      // tokens per unit: a multiple of 16, at most BT
  int item0;
  uint32_t idesc_dense, idesc_sparse;
};

// Positions of a group launch's units: CTA c runs the items at positions c,
// c + grid, c + 2 grid, ... in turn, up to the first kNoItem.
constexpr int kOrderCap = 8192;
constexpr uint16_t kNoItem = 0xFFFF;

template <int G>
struct Params {
  CUtensorMap x[G];            // X of GEMM g: boxes of 64 k x bt tokens
  CUtensorMap w[G];            // W of GEMM g: 16 KiB panels
  CUtensorMap w_up;            // gated MLP: the up weight, read by row 1
  Gemm g[G];
  int n_gemm, n_items;
  int n_pos;                   // positions: n_items for one GEMM (item = position), else order[] entries
  uint16_t order[G > 1 ? kOrderCap : 1];  // groups: the item at each position (host-balanced, see below)
  int mlp;                     // 1 (one GEMM): row 0 = gate, row 1 = up tile row rp; Y = silu(gate) * up
  const uint8_t* meta_up;
  const patch_tile_desc* desc_up;
  int ks;                      // K parts per output block (split K, one GEMM; 1 = whole K per unit)
  float* part;                 // ks > 1: fp32 partials [block][ks][ROWS][bt][128]
  uint32_t* counters;          // ks > 1: arrivals [block][ROWS][4] (zero between calls)
  int staged;                  // 1: every GEMM's descriptor rows fit in shared memory (Tk <= MAXTK)
  uint64_t limit_ns;
  int32_t* status;
  int inject;  // 1: row 0's producer stops after the first K-tile (exercises the timeout path)
};

// The item at position pos, or -1 past the end of this CTA's list.
template <int G>
__device__ __forceinline__ int item_at(const Params<G>& P, int pos) {
  if (pos >= P.n_pos) return -1;
  if constexpr (G == 1) {
    return pos;
  } else {
    return P.order[pos] == kNoItem ? -1 : int(P.order[pos]);
  }
}

// The GEMM of `item`: the last one whose first item is <= item.
template <int G>
__device__ __forceinline__ int gemm_of(const Params<G>& P, int item) {
  int lo = 0, hi = P.n_gemm - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (P.g[mid].item0 <= item) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Row pair rp holds tile rows rp and rp + n_pairs (n_pairs = ceil(Tn / 2);
// the last pair of an odd Tn has one row).  A unit costs the sum of its two
// rows' MMA time, so pairing each row with the one half the layer away keeps
// unit costs even when sparse tiles come in bands of tile rows (a band of half
// the rows puts exactly one row of every pair inside it), where neighbouring
// rows would pair dense with dense and sparse with sparse and a one-wave grid
// would wait for the dense pairs.  A gated-MLP unit is gate and up tile row rp.
__device__ __forceinline__ int rows_of(const Gemm& gm, int mlp, int rp) {
  return mlp ? ROWS : (rp + gm.n_pairs < gm.Tn ? ROWS : 1);
}
// the tile row of its weight that row r of unit row pair rp reads
__device__ __forceinline__ int tile_row(const Gemm& gm, int mlp, int rp, int r) {
  return mlp ? rp : rp + r * gm.n_pairs;
}

// Units run row pair by row pair (all token blocks of a pair are consecutive
// items), so the CTAs of one wave read a few row pairs' W, which stays in L2
// while every token block uses it, instead of every wave reading all of W.
// Units that share an X block (same tb) or W rows (same rp) start their K loop
// at different tiles, so they do not all hit the same L2 lines at the same
// moment; only the order of the fp32 sum changes.  The token blocks of a row
// pair start one K-tile apart, so each W panel's readers follow each other
// within a few steps and W streams through L2 once; the row pairs spread
// evenly over K, so an X block's readers span the whole loop and X stays
// resident (down at M = 2048 holds 45 MB of X but 90 MB of W: with the row
// pairs one tile apart and the token blocks spread, its W panels were
// evicted between readers, 1.5x the layer's bytes from DRAM).
__device__ __forceinline__ int k_rotation(int rp, int tb, int Tk, int n_pairs) {
  const int stride = Tk > n_pairs ? Tk / n_pairs : 1;
  return (rp * stride + tb) % Tk;
}

// Work unit: output block blk = (row pair rp, token block tb) of its GEMM and
// its K part kp, which covers K-tiles [k0, k0 + len).  With ks = 1 a unit is a
// whole output block.  The K loop starts at a rotated tile of the part.
struct Unit {
  int blk, kp, rp, tb, k0, len, rot;
};
__device__ __forceinline__ Unit unit_of(const Gemm& gm, int ks, int item) {
  Unit u;
  const int local = item - gm.item0;
  u.blk = local / ks;
  u.kp = local - u.blk * ks;
  u.rp = u.blk / gm.n_tb;
  u.tb = u.blk - u.rp * gm.n_tb;
  u.k0 = int(int64_t(u.kp) * gm.Tk / ks);
  u.len = int(int64_t(u.kp + 1) * gm.Tk / ks) - u.k0;
  u.rot = k_rotation(u.rp, u.tb, u.len, gm.n_pairs);
  return u;
}

// ---------------------------------------------------------------- roles

// W producer of row r: the row's descriptors, metadata and W panels.  It never
// touches X, so it may run ahead of the previous kernel in the stream (W, the
// metadata and the descriptors are inputs that no kernel triggering an early
// launch writes).
template <int G>
__device__ void producer_w(Shared& s, const Params<G>& P, int r) {
  const bool up = P.mlp && r;  // the gated MLP's row 1 reads the up weight
  const bool staged = P.staged;
  uint32_t a_i = 0, e_i = 0, d_i = 0;  // loads issued per ring / descriptor rows staged
  bool ok = true;
  // stage (or, for a pair without row r, complete with no bytes) the descriptor row of an item
  auto stage_row = [&](int item, int buf) {
    const Gemm& gm = P.g[gemm_of(P, item)];
    const int rp = unit_of(gm, P.ks, item).rp;
    const bool has = r < rows_of(gm, P.mlp, rp);
    const uint32_t row_bytes = uint32_t(gm.Tk * sizeof(patch_tile_desc));
    mbar_expect_tx(&s.pdesc_full[r][buf], has ? row_bytes : 0u);
    if (has)
      bulk_load(s.pdesc[r][buf], (up ? P.desc_up : gm.desc) + int64_t(tile_row(gm, P.mlp, rp, r)) * gm.Tk, row_bytes,
                &s.pdesc_full[r][buf]);
    ++d_i;
  };
  if (staged && item_at(P, blockIdx.x) >= 0) stage_row(item_at(P, blockIdx.x), 0);
  int it = 0;
  for (int pos = blockIdx.x; ok; pos += gridDim.x, ++it) {
    const int item = item_at(P, pos);
    if (item < 0) break;
    const int g = gemm_of(P, item);
    const Gemm& gm = P.g[g];
    const patch_tile_desc* desc = up ? P.desc_up : gm.desc;
    const uint8_t* meta = up ? P.meta_up : gm.meta;
    const CUtensorMap* tmap_w = up ? &P.w_up : &P.w[g];
    const Unit u = unit_of(gm, P.ks, item);
    const int rp = u.rp, tn = tile_row(gm, P.mlp, rp, r);
    const int buf = it & 1;
    if (staged) {
      if (!(ok = wait_bounded(&s.pdesc_full[r][buf], (it >> 1) & 1, &s.abort_flag, P.limit_ns, P.status, false)))
        break;
      // prefetch the next unit's row into the other buffer (its previous row is done)
      const int next = item_at(P, pos + int(gridDim.x));
      if (next >= 0) stage_row(next, buf ^ 1);
    }
    if (r >= rows_of(gm, P.mlp, rp)) continue;
    int kt = u.k0 + u.rot;
    for (int j = 0; ok && j < u.len; ++j, kt = (kt + 1 == u.k0 + u.len ? u.k0 : kt + 1)) {
      if (P.inject && r == 0 && (item != int(blockIdx.x) || j > 0)) {
        ok = false;
        break;
      }
      const patch_tile_desc d = staged ? s.pdesc[r][buf][kt] : desc[int64_t(tn) * gm.Tk + kt];
      if (d.kind) {
        const uint32_t es = e_i % NE;
        if (!(ok = wait_bounded(&s.e_empty[r][es], ((e_i / NE) & 1) ^ 1, &s.abort_flag, P.limit_ns, P.status, false)))
          break;
        mbar_expect_tx(&s.e_full[r][es], E_BYTES);
        bulk_load(s.e[r][es], meta + uint64_t(d.sparse_ordinal) * E_BYTES, E_BYTES, &s.e_full[r][es]);
        ++e_i;
      }
      // a dense tile's 2 panels (one per 64-k half), a sparse tile's one
      const int panel = int(d.val_offset / A_BYTES);
      for (int h = 0; h < (d.kind ? 1 : 2); ++h) {
        const uint32_t as = a_i % NA;
        if (!(ok = wait_bounded(&s.a_empty[r][as], ((a_i / NA) & 1) ^ 1, &s.abort_flag, P.limit_ns, P.status, false)))
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
    wait_bounded(&s.a_full[r][i % NA], (i / NA) & 1, &s.abort_flag, P.limit_ns, P.status, true);
  for (uint32_t i = (e_i > NE ? e_i - NE : 0); i < e_i; ++i)
    wait_bounded(&s.e_full[r][i % NE], (i / NE) & 1, &s.abort_flag, P.limit_ns, P.status, true);
  for (uint32_t i = (d_i > 2 ? d_i - 2 : 0); i < d_i; ++i)
    wait_bounded(&s.pdesc_full[r][i & 1], (i >> 1) & 1, &s.abort_flag, P.limit_ns, P.status, true);
}

// X producer: the two 64-k panels of X per K-tile, in the same rotated K order.
template <int G>
__device__ void producer_x(Shared& s, const Params<G>& P) {
  uint32_t b_i = 0;
  bool ok = true;
  // X may be the previous kernel's output: wait for it before the first X load
  pdl_wait_previous();
  for (int pos = blockIdx.x; ok; pos += gridDim.x) {
    const int item = item_at(P, pos);
    if (item < 0) break;
    const int g = gemm_of(P, item);
    const Gemm& gm = P.g[g];
    const Unit u = unit_of(gm, P.ks, item);
    int kt = u.k0 + u.rot;
    for (int j = 0; ok && j < u.len; ++j, kt = (kt + 1 == u.k0 + u.len ? u.k0 : kt + 1)) {
      for (int h = 0; ok && h < 2; ++h) {
        const uint32_t bs = b_i % NB;
        if (!(ok = wait_bounded(&s.b_empty[bs], ((b_i / NB) & 1) ^ 1, &s.abort_flag, P.limit_ns, P.status, false)))
          break;
        mbar_expect_tx(&s.b_full[bs], uint32_t(gm.bt) * 128u);
        tma_load_2d(s.b[bs], &P.x[g], &s.b_full[bs], kt * kTile + 64 * h, u.tb * gm.bt);
        ++b_i;
      }
    }
  }
  for (uint32_t i = (b_i > NB ? b_i - NB : 0); i < b_i; ++i)
    wait_bounded(&s.b_full[i % NB], (i / NB) & 1, &s.abort_flag, P.limit_ns, P.status, true);
}

// MMA issuer of row r (one thread): each row has its own issuing thread, so
// the two chains' barrier waits, commits and bookkeeping overlap and the
// tensor core, shared by both, stays fed.  Both consume the same X slots; a
// slot is free once both rows' MMAs on it are complete (two commits).
template <int G>
__device__ void mma_issuer(Shared& s, uint32_t tmem, const Params<G>& P, int r) {
  const uint32_t acc = tmem + ACC_STRIDE * r;
  uint32_t a_i = 0, b_i = 0, e_i = 0;
  bool ok = true;
  int it = 0;
  for (int pos = blockIdx.x; ok; pos += gridDim.x, ++it) {
    const int item = item_at(P, pos);
    if (item < 0) break;
    const Gemm& gm = P.g[gemm_of(P, item)];
    const uint32_t idesc_dense = gm.idesc_dense, idesc_sparse = gm.idesc_sparse;
    const Unit u = unit_of(gm, P.ks, item);
    const bool active = r < rows_of(gm, P.mlp, u.rp);
    if (!(ok = wait_bounded(&s.acc_empty[r], (it & 1) ^ 1, &s.abort_flag, P.limit_ns, P.status, false))) break;
    tc_fence_after();
    uint32_t accumulate = 0;
    for (int kt = 0; ok && kt < u.len; ++kt) {
      uint32_t kind = 0, as = 0, es = 0;
      for (int h = 0; h < 2; ++h) {
        // the tile's kind arrives with its first panel; a sparse tile's one
        // panel serves both halves and its metadata goes to TMEM first
        if (active && (h == 0 || !kind)) {
          as = a_i % NA;
          if (!(ok = wait_bounded(&s.a_full[r][as], (a_i / NA) & 1, &s.abort_flag, P.limit_ns, P.status, false)))
            break;
          ++a_i;
          if (h == 0) kind = *reinterpret_cast<volatile uint32_t*>(&s.a_kind[r][as]);
          if (h == 0 && kind) {
            es = e_i % NE;
            if (!(ok = wait_bounded(&s.e_full[r][es], (e_i / NE) & 1, &s.abort_flag, P.limit_ns, P.status, false)))
              break;
            ++e_i;
            tc_fence_after();
            tmem_cp_128x128b(acc + META_COL0 + 4 * es, meta_desc(smem_u32(s.e[r][es])));
          }
        }
        const uint32_t bs = b_i % NB;
        if (!(ok = wait_bounded(&s.b_full[bs], (b_i / NB) & 1, &s.abort_flag, P.limit_ns, P.status, false))) break;
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
                       idesc_sparse | (kb & 1u), accumulate);
            accumulate = 1;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // K = 16 per MMA = 32 B along the swizzled row
            mma_dense(acc, a0 + (j * 32 >> 4), b0 + (j * 32 >> 4), idesc_dense, accumulate);
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
  wait_bounded(&s.drain[r], 0, &s.abort_flag, P.limit_ns, P.status, true);
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
template <int G>
__device__ void epilogue_split(Shared& s, uint32_t tmem, const Params<G>& P, const Gemm& gm, const Unit& u, int g,
                               int q, int lane) {
  const bool has = g < rows_of(gm, P.mlp, u.rp);
  const int row = 32 * q + lane;
  const int64_t n = int64_t(tile_row(gm, P.mlp, u.rp, g)) * BM + row;
  const int m0 = u.tb * gm.bt;
  const int valid = gm.M - m0 < gm.bt ? gm.M - m0 : gm.bt;  // tokens of this block inside X
  const int64_t slot_floats = int64_t(BM) * gm.bt;           // one row g of one unit
  const int64_t blk_base = int64_t(u.blk) * P.ks * ROWS;
  if (has) {
    float* mine = P.part + ((blk_base + int64_t(u.kp) * ROWS + g) * slot_floats) + row;
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
  uint32_t* counter = P.counters + (int64_t(u.blk) * ROWS + g) * 4 + q;
  uint32_t old = 0;
  if (lane == 0) old = atom_add_acq_rel_gpu(counter, 1u);
  old = __shfl_sync(0xFFFFFFFFu, old, 0);
  if (old != uint32_t(P.ks - 1)) return;
  __syncwarp();  // orders lane 0's acquire before every lane's loads
  for (int c = 0; c * YT < valid; ++c) {
    float sum[YT];
#pragma unroll
    for (int j = 0; j < YT; ++j) sum[j] = 0.0f;
    for (int kp = 0; kp < P.ks; ++kp) {
      const float* src = P.part + ((blk_base + int64_t(kp) * ROWS + g) * slot_floats) + int64_t(YT * c) * BM + row;
      float part[YT];
#pragma unroll
      for (int j = 0; j < YT; ++j) part[j] = __ldcg(src + int64_t(j) * BM);
#pragma unroll
      for (int j = 0; j < YT; ++j) sum[j] += part[j];
    }
#pragma unroll
    for (int j = 0; j < YT; ++j)
      if (YT * c + j < valid) gm.Y[int64_t(m0 + YT * c + j) * gm.N + n] = f32_to_bf16_rne(sum[j]);
  }
  if (lane == 0) *counter = 0;  // ready for the next call
}

template <int G>
__device__ void epilogue(Shared& s, uint32_t tmem, const Params<G>& P) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;                  // the TMEM lane quarter this warp may access
  const int g = (warp - EPI_WARP0) >> 2;   // warp group
  const uint32_t bar_id = 1 + g;           // named barrier of the group's 128 threads
  const bool mlp = P.mlp;
  int it = 0;
  for (int pos = blockIdx.x;; pos += gridDim.x, ++it) {
    const int item = item_at(P, pos);
    if (item < 0) break;
    const Gemm& gm = P.g[gemm_of(P, item)];
    const Unit u = unit_of(gm, P.ks, item);
    const int rp = u.rp, tb = u.tb;
    // the four warps of a group take the same decision, so none is left at a barrier
    bool ok = wait_bounded(&s.acc_full[g], it & 1, &s.abort_flag, P.limit_ns, P.status, false);
    if (mlp) ok = ok && wait_bounded(&s.acc_full[g ^ 1], it & 1, &s.abort_flag, P.limit_ns, P.status, false);
    if (!named_bar_and(bar_id, 128, ok)) break;
    tc_fence_after();
    if (P.ks > 1) {  // split K (never with the gated MLP)
      epilogue_split(s, tmem, P, gm, u, g, q, lane);
      continue;
    }
    if (mlp || g < rows_of(gm, mlp, rp)) {
      const int n0 = tile_row(gm, mlp, rp, g) * BM, m0 = tb * gm.bt;
      const int valid = gm.M - m0 < gm.bt ? gm.M - m0 : gm.bt;  // tokens of this unit inside X
      const uint32_t lanes = tmem + (uint32_t(32 * q) << 16);
      const int c0 = mlp ? g : 0, dc = mlp ? 2 : 1;
      const int64_t ldy = gm.N;
      // this thread's feature; a warp's 32 stores of one token fill 64 contiguous bytes of Y
      uint16_t* yp = gm.Y + int64_t(m0) * ldy + n0 + 32 * q + lane;
      for (int c = c0; c * YC < valid; c += dc) {
        uint32_t v[YC];
        if (mlp) {
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
        uint16_t* yr = yp + int64_t(YC * c) * ldy;
        const int nj = valid - YC * c < YC ? valid - YC * c : YC;
#pragma unroll
        for (int j = 0; j < YC; ++j, yr += ldy)
          if (j < nj) *yr = f32_to_bf16_rne(__uint_as_float(v[j]));
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&s.acc_empty[g]);
      if (mlp) mbar_arrive(&s.acc_empty[g ^ 1]);
    }
  }
}

template <int G>
__global__ void __launch_bounds__(THREADS, 1) prefill_kernel(const __grid_constant__ Params<G> P) {
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
      mbar_init(&s.acc_empty[r], P.mlp ? 8 : 4);  // the gated MLP's groups both read both rows
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
    for (int i = 0; i < P.n_gemm; ++i) {
      prefetch_tensormap(&P.x[i]);
      prefetch_tensormap(&P.w[i]);
    }
    if (P.mlp) prefetch_tensormap(&P.w_up);
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
        mma_issuer(s, tmem, P, warp >> 1);
      else
        producer_w(s, P, warp >> 1);
    }
    __syncwarp();
  } else if (warp == 4) {
    if (lane == 0) producer_x(s, P);
    __syncwarp();
  } else if (warp >= EPI_WARP0) {
    epilogue(s, tmem, P);
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

// The values blob of W as a tensor map of 16 KiB panels (rows of 128 B).
static bool make_map_w(CUtensorMap* map, const patch_weight& W) {
  const int64_t T = (W.N / prefill::BM) * (W.K / kTile);
  const uint64_t n_panels = uint64_t(2 * (T - W.n_sparse) + W.n_sparse);
  return make_map_2d_bf16(map, W.values, 64, n_panels * 128, 128, 64, 128);
}

// GEMM i of a launch: Y = X W^T in units of n_pairs row pairs x n_tb token
// blocks of bt tokens x ks K parts, its items starting at item0.
template <int G>
static bool set_gemm(prefill::Params<G>& P, int i, const uint16_t* X, int64_t M, const patch_weight& W, uint16_t* Y,
                     int64_t n_pairs, int bt, int ks, int item0) {
  using namespace prefill;
  Gemm& gm = P.g[i];
  gm.meta = static_cast<const uint8_t*>(W.meta);
  gm.desc = W.desc;
  gm.Y = Y;
  gm.M = int(M);
  gm.N = int(W.N);
  gm.Tn = int(W.N / BM);
  gm.Tk = int(W.K / kTile);
  gm.n_pairs = int(n_pairs);
  gm.n_tb = int((M + bt - 1) / bt);
  gm.bt = bt;
  gm.item0 = item0;
  gm.idesc_dense = tc::idesc_bf16(BM, bt, false);
  gm.idesc_sparse = tc::idesc_bf16(BM, bt, true);
  (void)ks;
  return make_map_2d_bf16(&P.x[i], X, uint64_t(W.K), uint64_t(M), uint64_t(W.K) * 2, 64, uint32_t(bt)) &&
         make_map_w(&P.w[i], W);
}

template <int G>
static void set_launch(prefill::Params<G>& P, int n_gemm, int n_items, int32_t* status, uint64_t limit_ns) {
  P.n_gemm = n_gemm;
  P.n_items = n_items;
  P.n_pos = n_items;
  P.mlp = 0;
  P.meta_up = nullptr;
  P.desc_up = nullptr;
  P.ks = 1;
  P.part = nullptr;
  P.counters = nullptr;
  P.staged = 1;
  for (int i = 0; i < n_gemm; ++i)
    if (P.g[i].Tk > prefill::MAXTK) P.staged = 0;
  P.limit_ns = limit_ns;
  P.status = status;
  P.inject = 0;
}

static_assert(sizeof(prefill::Params<kPrefillGroupMax>) <= 32764, "kernel parameter space");

template <int G>
static cudaError_t launch_params(const prefill::Params<G>& P, int num_sms, cudaStream_t stream) {
  using namespace prefill;
  const int grid = P.n_items < num_sms ? P.n_items : num_sms;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  return launch_pdl(prefill_kernel<G>, dim3(unsigned(grid)), dim3(THREADS), SMEM_BYTES, stream, P);
}

// Shared by the plain GEMM (units of tile rows rp and rp + n_pairs of W) and
// the gated MLP (W0 = gate, W1 = up, units of tile row rp of each).
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
  Params<1> P;
  if (!set_gemm(P, 0, X, M, W0, Y, n_pairs, plan.bt, plan.ks, 0)) return cudaErrorUnknown;
  set_launch(P, 1, int(n_pairs * plan.n_tb * plan.ks), status, limit_ns);
  P.mlp = mlp ? 1 : 0;
  if (mlp) {
    if (!make_map_w(&P.w_up, W1)) return cudaErrorUnknown;
    P.meta_up = static_cast<const uint8_t*>(W1.meta);
    P.desc_up = W1.desc;
  }
  P.ks = plan.ks;
  P.counters = static_cast<uint32_t*>(workspace);  // the fixed counter region at the start (used when ks > 1)
  P.part = plan.ks > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kDecodeCounterBytes) : nullptr;
  P.inject = inject;
  return launch_params(P, num_sms, stream);
}

// Units to CTAs for a group: longest first, each to the CTA with the least
// work so far (ties to the lower index), a unit's work modelled as its
// K-tiles x tokens x tile rows.  Units of one GEMM cost the same, so those of
// the costliest GEMM go out first, round the CTAs, then the next GEMM's fill
// in behind the shortest lists.  CTA c's j-th unit sits at position c + j grid.
// Returns false when the positions do not fit the table.
template <int G>
static bool balance_units(prefill::Params<G>& P, const int64_t* unit_cost, int grid) {
  using namespace prefill;
  std::vector<std::vector<uint16_t>> lists(grid);
  std::vector<std::pair<int64_t, int>> heap;  // (work, cta), a min-heap
  for (int c = 0; c < grid; ++c) heap.push_back({0, c});
  auto later = [](const std::pair<int64_t, int>& a, const std::pair<int64_t, int>& b) { return a > b; };
  for (int i = 0; i < P.n_gemm; ++i) {  // GEMMs are in descending unit cost
    const int n_units = P.g[i].n_pairs * P.g[i].n_tb;
    for (int k = 0; k < n_units; ++k) {
      std::pop_heap(heap.begin(), heap.end(), later);
      lists[heap.back().second].push_back(uint16_t(P.g[i].item0 + k));
      heap.back().first += unit_cost[i];
      std::push_heap(heap.begin(), heap.end(), later);
    }
  }
  size_t rounds = 0;
  for (const auto& l : lists) rounds = l.size() > rounds ? l.size() : rounds;
  if (rounds * size_t(grid) > size_t(kOrderCap)) return false;
  P.n_pos = int(rounds) * grid;
  for (int pos = 0; pos < P.n_pos; ++pos) {
    const auto& l = lists[pos % grid];
    const size_t j = size_t(pos / grid);
    P.order[pos] = j < l.size() ? l[j] : kNoItem;
  }
  return true;
}

// A group of independent GEMMs in one launch (at most kPrefillGroupMax).
// Tokens per unit: the fewest 240-token blocks that hold M, evened out
// (M = 512: 3 blocks of 176, not 240 + 240 + 32), so no block streams its
// weights for a sliver of tokens; the units of all the GEMMs then share the
// CTAs as balance_units assigns them.
cudaError_t launch_prefill_group(const PrefillGroupCall* calls, int n, int32_t* status, int num_sms,
                                 uint64_t limit_ns, cudaStream_t stream) {
  using namespace prefill;
  if (n <= 0) return cudaSuccess;
  if (n > kPrefillGroupMax) return cudaErrorInvalidValue;
  int order[kPrefillGroupMax], bts[kPrefillGroupMax];
  int64_t cost[kPrefillGroupMax];
  for (int i = 0; i < n; ++i) {
    const int64_t M = calls[i].M, Tn = calls[i].W.N / BM, Tk = calls[i].W.K / kTile;
    const int64_t blocks = (M + BT - 1) / BT;
    const int64_t per = (M + blocks - 1) / blocks;
    bts[i] = int((per + 15) / 16 * 16);
    cost[i] = Tk * bts[i] * (Tn > 1 ? ROWS : 1);
    order[i] = i;
  }
  for (int i = 1; i < n; ++i)  // stable insertion sort, costliest units first
    for (int j = i; j > 0 && cost[order[j]] > cost[order[j - 1]]; --j) {
      const int t = order[j];
      order[j] = order[j - 1];
      order[j - 1] = t;
    }
  std::unique_ptr<Params<kPrefillGroupMax>> hold(new Params<kPrefillGroupMax>());  // ~27 KB, copied at launch
  Params<kPrefillGroupMax>& P = *hold;
  int items = 0;
  int64_t unit_cost[kPrefillGroupMax];
  for (int k = 0; k < n; ++k) {
    const PrefillGroupCall& c = calls[order[k]];
    const int64_t n_pairs = (c.W.N / BM + ROWS - 1) / ROWS;
    if (!set_gemm(P, k, c.X, c.M, c.W, c.Y, n_pairs, bts[order[k]], 1, items)) return cudaErrorUnknown;
    items += P.g[k].n_pairs * P.g[k].n_tb;
    unit_cost[k] = cost[order[k]];
  }
  set_launch(P, n, items, status, limit_ns);
  const int grid = items < num_sms ? items : num_sms;
  if (items > kOrderCap || !balance_units(P, unit_cost, grid)) {
    // too many units for the table: the first half of the calls, then the rest;
    // a call alone runs as patch_gemm's prefill path does (no split K)
    if (n < 2)
      return launch_prefill(calls[0].X, calls[0].M, calls[0].W, calls[0].Y, nullptr, 0, status, num_sms, limit_ns, 0,
                            stream);
    const cudaError_t e = launch_prefill_group(calls, n / 2, status, num_sms, limit_ns, stream);
    return e != cudaSuccess ? e : launch_prefill_group(calls + n / 2, n - n / 2, status, num_sms, limit_ns, stream);
  }
  return launch_params(P, num_sms, stream);
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
