// Decode path of patch_gemm (M <= 16 tokens): a stream-K, TMA-fed kernel
// whose job is to move the stored bytes of the packed weight from HBM at
// full bandwidth; the tensor cores do the (small) arithmetic.
//
// Layer: Y[m][n] = sum_k X[m][k] * W_eff[n][k] with W_eff the hybrid weight
// of "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs" (section 2
// "Methodology: PATCH", "Core Mechanism" and "Inference & Deployment": dense
// 128 x 128 tiles on dense tensor-core MMA, 2:4 tiles on the sparse ones).
//
// Work split (stream-K over panels): the values blob is a sequence of P
// panels (16 KiB: a dense tile is 2 panels, a sparse tile 1) in row-major
// tile order.  CTA c of G takes panels [c*P/G, (c+1)*P/G), so
// every CTA streams the same number of panels whatever the sparsity pattern
// (G = 1.5 x the SM count, two CTA slots per SM; see plan()).
// Inside its range a CTA accumulates each tile row's panels into a TMEM
// accumulator (M = 128 rows of W, N = 16 tokens, zero-padded by TMA).  A
// tile row entirely inside one CTA's range is rounded to bf16 and stored
// directly.  A row cut by range boundaries is finished, per 32-row quarter,
// by whichever covering CTA's epilogue warp arrives last: every warp stores
// its fp32 partial sums in the workspace and bumps the quarter's arrival
// counter; the last one adds all partials in CTA order (deterministic),
// stores Y and resets the counter to zero for the next call.
//
// One pipeline stage per panel holds the 16 KiB weight panel, the 64-k
// slices of X it multiplies (1 for a dense panel, 2 for a sparse one) and,
// for a sparse tile, its 2 KiB of metadata, all landing on one mbarrier.
// Roles per CTA (7 warps): warp 0 W producer (weight panels, the stage's
// info word), warp 6 X producer (X slices, metadata), warp 1 MMA issuer and
// TMEM owner (dense panel: 4 x kind::f16 K = 16; sparse tile: tcgen05.cp of
// the metadata, then 4 x kind::f16 .sp K = 32), warps 2-5 epilogue.  Every
// wait is bounded in time as in the prefill kernel.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace patch {
namespace decode_tc {

using namespace tc;

constexpr int BM = 128;
constexpr int BT = 16;                   // MMA N (tokens)
constexpr int NS = 4;                    // pipeline stages per CTA (2 CTAs per SM: ~8 panels in flight)
constexpr int NACC = 2;                  // accumulator buffers (epilogue overlaps the next row)
constexpr int A_BYTES = PATCH_PANEL_BYTES;
constexpr int X_BYTES = BT * 64 * 2;     // one 64-k slice of X (room for 16 token rows)
constexpr int E_BYTES = PATCH_META_TILE_BYTES;
constexpr int THREADS = 224;  // warps: 0 W producer, 1 MMA, 2-5 epilogue, 6 X producer
constexpr uint32_t TMEM_COLS = 128;
constexpr uint32_t META_COL0 = NACC * BT;  // 4 metadata columns per stage after the accumulators
static_assert(META_COL0 + 4 * NS <= TMEM_COLS, "TMEM layout");
constexpr uint32_t IDESC_DENSE = idesc_bf16(BM, BT, false);
constexpr uint32_t IDESC_SPARSE = idesc_bf16(BM, BT, true);
constexpr int WS_FLOATS_PER_CTA = 2 * BT * BM;  // [2 slots][128 rows][16 tokens]
constexpr int DCAP = 256;                       // descriptors of the CTA's tiles staged in shared memory

// stage info word written by the producer, read by the MMA thread
constexpr uint32_t INFO_SPARSE = 1u, INFO_SEG_START = 2u, INFO_SEG_END = 4u;

struct Stage {
  alignas(1024) uint8_t a[A_BYTES];
  alignas(1024) uint8_t x[2][X_BYTES];
  alignas(128) uint8_t e[E_BYTES];
};

struct Shared {
  Stage st[NS];
  uint64_t full[NS], empty[NS];
  uint64_t acc_full[NACC], acc_empty[NACC], drain;
  uint32_t info[NS];
  alignas(16) patch_tile_desc dcache[DCAP];  // tiles t_first .. t_last (when they fit)
  uint32_t tmem_base;
  int abort_flag;
  int t_first, t_last;  // tiles holding the CTA's first and last panel
  int cached;           // dcache holds the CTA's tiles
  int64_t row_lo[2];    // first panel of the CTA's first row, and of the row after it
  int64_t row_hi[2];    // first panel of the CTA's last row, and of the row after it
};
constexpr size_t SMEM_BYTES = sizeof(Shared) + 1024;
// two CTAs fit on an SM, so the next layer's CTAs can start (and stream their
// weight) while this kernel's last CTAs finish
static_assert(2 * (SMEM_BYTES + 1024) <= 228 * 1024, "shared memory budget: 2 CTAs per SM");

struct Args {
  const patch_tile_desc* desc;
  const uint8_t* meta;
  uint16_t* Y;
  float* ws;           // [G][2][128][16] fp32 partials (contents between calls do not matter)
  uint32_t* counters;  // [Tn][4] arrivals per tile row and TMEM lane quarter (zero between calls)
  int M, N, Tk, Tn;
  int64_t P;  // panels in the values blob
  uint64_t limit_ns;
  int32_t* status;
};

__host__ __device__ __forceinline__ int64_t range_begin(int64_t c, int64_t P, int64_t G) { return c * P / G; }
// the CTA whose range holds panel p
__host__ __device__ __forceinline__ int64_t cta_of_panel(int64_t p, int64_t P, int64_t G) {
  return ((p + 1) * G - 1) / P;
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ int64_t panel_of(const patch_tile_desc& d) {
  return int64_t(d.val_offset / PATCH_PANEL_BYTES);
}

// Tiles holding panels pa and pb: the last t with panel_of(desc[t]) <= p.
// Called by every thread of the block.  The first round probes blockDim.x
// consecutive tiles around the proportional estimate p*T/P, which holds the
// answer unless the sparse tiles are very unevenly spread; otherwise each
// further round probes blockDim.x tiles at once and narrows the span by that
// factor, so a search costs a few global latencies, not log2(T) dependent ones.
__device__ void find_tiles(const patch_tile_desc* desc, int T, int64_t P, int64_t pa, int64_t pb, int& ta,
                           int& tb) {
  const int n = blockDim.x, i = threadIdx.x;
  auto window = [&](int64_t p) {
    int64_t w = p * T / P - n / 2;
    if (w > T - n) w = T - n;
    return int(w < 0 ? 0 : w);
  };
  const int wa = window(pa), wb = window(pb);
  const int ca = __syncthreads_count(wa + i < T && panel_of(desc[wa + i]) <= pa);
  const int cb = __syncthreads_count(wb + i < T && panel_of(desc[wb + i]) <= pb);
  const int na = T - wa < n ? T - wa : n, nb = T - wb < n ? T - wb : n;
  if (ca >= 1 && (ca < na || wa + na == T) && cb >= 1 && (cb < nb || wb + nb == T)) {
    ta = wa + ca - 1;
    tb = wb + cb - 1;
    return;
  }
  int lo_a = 0, lo_b = 0, span = T;
  while (span > 1) {
    const int step = (span + n - 1) / n;
    const int ia = lo_a + i * step, ib = lo_b + i * step;
    const bool in = i * step < span;
    const int ka = __syncthreads_count(in && ia < T && panel_of(desc[ia]) <= pa);
    const int kb = __syncthreads_count(in && ib < T && panel_of(desc[ib]) <= pb);
    lo_a += (ka - 1) * step;
    lo_b += (kb - 1) * step;
    span = step;
  }
  ta = lo_a;
  tb = lo_b;
}

// One-round form of the CTA's set-up: every thread loads one descriptor of a
// window of blockDim.x tiles starting one tile row before the proportional
// estimate of the CTA's first tile.  When the window holds the CTA's tiles and
// the first tile of every tile row the epilogue needs (the rows holding the
// CTA's first and last tile, and the rows after them), the tile range, the
// staged descriptors and the row boundaries all come from those registers: one
// global round trip instead of the three of find_tiles, the staging loop and
// the boundary loads.  That is the usual case (even sparse tiles, Tk up to
// about 100); otherwise it writes nothing and returns false (block-uniform).
__device__ bool locate_one_round(Shared& s, const Args& a, int64_t pa, int64_t pb) {
  const int n = blockDim.x, i = threadIdx.x;
  const int T = a.Tn * a.Tk;
  int64_t w64 = pa * T / a.P - a.Tk;
  if (w64 > T - n) w64 = T - n;
  if (w64 < 0) w64 = 0;
  const int w = int(w64), t = w + i;
  const bool in = t < T;
  patch_tile_desc d = {};
  if (in) d = a.desc[t];
  const int64_t pm = in ? panel_of(d) : 0;
  const int ca = __syncthreads_count(in && pm <= pa);
  const int cb = __syncthreads_count(in && pm <= pb);
  const int nv = T - w < n ? T - w : n;  // window entries inside the table
  if (ca < 1 || cb < 1 || ((ca == nv || cb == nv) && w + nv != T)) return false;
  const int ta = w + ca - 1, tb = w + cb - 1;
  const int row_first = ta / a.Tk * a.Tk, row_after = (tb / a.Tk + 1) * a.Tk;
  if (row_first < w || (row_after < T && row_after >= w + nv) || tb - ta + 1 > DCAP) return false;
  if (in && t >= ta && t <= tb) s.dcache[t - ta] = d;
  // first panel of: the first row, the row after it, the last row, the row after that (P past the end)
  const int want[4] = {row_first, row_first + a.Tk, tb / a.Tk * a.Tk, row_after};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    int64_t* dst = k < 2 ? &s.row_lo[k] : &s.row_hi[k - 2];
    if (want[k] >= T) {
      if (i == 0) *dst = a.P;
    } else if (in && t == want[k]) {
      *dst = pm;
    }
  }
  if (i == 0) {
    s.t_first = ta;
    s.t_last = tb;
    s.cached = 1;
  }
  return true;
}

// Descriptor of tile t (staged in shared memory when the CTA's tiles fit).
__device__ __forceinline__ patch_tile_desc tile_desc(const Shared& s, const Args& a, int t) {
  return s.cached ? s.dcache[t - s.t_first] : a.desc[t];
}

// X slice loads of one stage (after the previous kernel in the stream is done)
__device__ __forceinline__ void load_x(Stage& g, uint64_t* full, const CUtensorMap* tmap_x, uint32_t xinfo) {
  const int kt = int(xinfo >> 2), h = int((xinfo >> 1) & 1);
  if (xinfo & 1) {
    tma_load_2d(g.x[0], tmap_x, full, kt * kTile, 0);
    tma_load_2d(g.x[1], tmap_x, full, kt * kTile + 64, 0);
  } else {
    tma_load_2d(g.x[0], tmap_x, full, kt * kTile + 64 * h, 0);
  }
}

// Walks a CTA's panels in order: tile t, K-tile kt, half h of a dense tile.
struct PanelWalk {
  int t, h, kt;
  patch_tile_desc d;
  __device__ __forceinline__ void start(const Shared& s, const Args& a, int64_t p0) {
    t = s.t_first;
    d = tile_desc(s, a, t);
    h = int(p0 - panel_of(d));
    kt = t % a.Tk;
  }
  __device__ __forceinline__ bool sparse() const { return d.kind != 0; }
  __device__ __forceinline__ bool last_of_tile() const { return d.kind != 0 || h == 1; }
  // X slices of this panel: K-tile, half, both halves for a sparse tile
  __device__ __forceinline__ uint32_t xinfo() const {
    return uint32_t(kt) << 2 | uint32_t(h) << 1 | (sparse() ? 1u : 0u);
  }
  __device__ __forceinline__ void next(const Shared& s, const Args& a, bool more) {
    if (last_of_tile()) {
      h = 0;
      ++t;
      if (++kt == a.Tk) kt = 0;
      if (more) d = tile_desc(s, a, t);
    } else {
      h = 1;
    }
  }
};

// Two producer threads fill each stage; the stage barrier counts one arrival
// from each.  One thread issuing every copy spends about as long per panel as
// HBM takes to deliver it.
//
// W producer: the weight panel and the stage's info word.  The panels of the
// first NS stages were requested at kernel entry; for those it only arrives.
__device__ void producer_w(Shared& s, const CUtensorMap* tmap_w, const Args& a, int64_t p0, int64_t p1) {
  PanelWalk w;
  w.start(s, a, p0);
  uint32_t i = 0;
  for (int64_t p = p0; p < p1; ++p, ++i) {
    const uint32_t st = i % NS;
    const bool early = i < NS;
    if (!early && !wait_bounded(&s.empty[st], ((i / NS) & 1) ^ 1, &s.abort_flag, a.limit_ns, a.status, false))
      break;
    uint32_t info = w.sparse() ? INFO_SPARSE : 0u;
    if (p == p0 || (w.kt == 0 && w.h == 0)) info |= INFO_SEG_START;
    if (p + 1 == p1 || (w.kt == a.Tk - 1 && w.last_of_tile())) info |= INFO_SEG_END;
    s.info[st] = info;  // published to the MMA thread by this thread's arrival
    if (early) {
      mbar_arrive(&s.full[st]);
    } else {
      mbar_expect_tx(&s.full[st], A_BYTES);
      tma_load_2d(s.st[st].a, tmap_w, &s.full[st], 0, int(p * 128));
    }
    w.next(s, a, p + 1 < p1);
  }
  // every copy issued must have landed before the CTA may exit
  for (uint32_t j = (i > NS ? i - NS : 0); j < i; ++j)
    wait_bounded(&s.full[j % NS], (j / NS) & 1, &s.abort_flag, a.limit_ns, a.status, true);
}

// X producer: a sparse tile's metadata and the panel's X slices (M token rows
// x 64 k each).  The metadata of the first NS stages is requested before this
// kernel waits for the previous kernel in the stream; X, which may be that
// kernel's output, only after it has completed.
__device__ void producer_x(Shared& s, const CUtensorMap* tmap_x, const Args& a, int64_t p0, int64_t p1) {
  PanelWalk w;
  w.start(s, a, p0);
  const uint32_t xb = uint32_t(a.M) * 128;  // an X slice holds M token rows (rows M..15 of the slot are never read back)
  const int64_t n0 = p1 - p0 < NS ? p1 - p0 : NS;
  uint32_t first[NS];
  uint32_t i = 0;
  int64_t p = p0;
#pragma unroll
  for (int j = 0; j < NS; ++j) {
    if (j >= n0) break;
    const bool sparse = w.sparse();
    mbar_expect_tx(&s.full[j], sparse ? 2 * xb + E_BYTES : xb);
    if (sparse) bulk_load(s.st[j].e, a.meta + uint64_t(w.d.sparse_ordinal) * E_BYTES, E_BYTES, &s.full[j]);
    first[j] = w.xinfo();
    w.next(s, a, p + 1 < p1);
    ++p;
    ++i;
  }
  pdl_wait_previous();
#pragma unroll
  for (int j = 0; j < NS; ++j)
    if (j < n0) load_x(s.st[j], &s.full[j], tmap_x, first[j]);
  for (; p < p1; ++p, ++i) {
    const uint32_t st = i % NS;
    if (!wait_bounded(&s.empty[st], ((i / NS) & 1) ^ 1, &s.abort_flag, a.limit_ns, a.status, false)) break;
    const bool sparse = w.sparse();
    mbar_expect_tx(&s.full[st], sparse ? 2 * xb + E_BYTES : xb);
    if (sparse) bulk_load(s.st[st].e, a.meta + uint64_t(w.d.sparse_ordinal) * E_BYTES, E_BYTES, &s.full[st]);
    load_x(s.st[st], &s.full[st], tmap_x, w.xinfo());
    w.next(s, a, p + 1 < p1);
  }
  for (uint32_t j = (i > NS ? i - NS : 0); j < i; ++j)
    wait_bounded(&s.full[j % NS], (j / NS) & 1, &s.abort_flag, a.limit_ns, a.status, true);
}

__device__ void mma_issuer(Shared& s, uint32_t tmem, const Args& a, int64_t p0, int64_t p1) {
  uint32_t i = 0, seg = 0, acc = tmem, accumulate = 0;
  for (int64_t p = p0; p < p1; ++p, ++i) {
    const uint32_t st = i % NS;
    if (!wait_bounded(&s.full[st], (i / NS) & 1, &s.abort_flag, a.limit_ns, a.status, false)) break;
    const uint32_t info = *reinterpret_cast<volatile uint32_t*>(&s.info[st]);
    if (info & INFO_SEG_START) {  // a new tile row starts a new accumulation segment
      const uint32_t buf = seg % NACC;
      if (!wait_bounded(&s.acc_empty[buf], ((seg / NACC) & 1) ^ 1, &s.abort_flag, a.limit_ns, a.status, false))
        break;
      acc = tmem + buf * BT;
      accumulate = 0;
    }
    tc_fence_after();
    Stage& g = s.st[st];
    const uint64_t a0 = sw128_desc(smem_u32(g.a));
    if (info & INFO_SPARSE) {
      const uint32_t e_tmem = tmem + META_COL0 + 4 * st;
      tmem_cp_128x128b(e_tmem, meta_desc(smem_u32(g.e)));
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {  // 32-k blocks: 16 kept values = 32 B of A; 32 k = 64 B of X
        const uint64_t b = sw128_desc(smem_u32(g.x[kb >> 1])) + ((kb & 1) * 64 >> 4);
        mma_sparse(acc, a0 + (kb * 32 >> 4), b, e_tmem + (kb & 2), IDESC_SPARSE | (kb & 1), accumulate);
        accumulate = 1;
      }
    } else {
      const uint64_t b0 = sw128_desc(smem_u32(g.x[0]));
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // K = 16 per MMA = 32 B along the swizzled row
        mma_dense(acc, a0 + (j * 32 >> 4), b0 + (j * 32 >> 4), IDESC_DENSE, accumulate);
        accumulate = 1;
      }
    }
    tc_commit(&s.empty[st]);
    if (info & INFO_SEG_END) {
      tc_commit(&s.acc_full[seg % NACC]);
      ++seg;
    }
  }
  tc_commit(&s.drain);
  wait_bounded(&s.drain, 0, &s.abort_flag, a.limit_ns, a.status, true);
}

// Sum of the partial rows (row r of the tile row) of covering CTAs c_lo..c_hi,
// in CTA order (deterministic).  B CTAs at a time: all their loads are issued
// before the additions; NV float4s (4 tokens each) per partial row at most.
template <int B, int NV>
__device__ __forceinline__ void sum_partials(const Args& a, int r, int64_t c_lo, int64_t c_hi, int slot_lo, int nv,
                                             float (&sum)[BT]) {
#pragma unroll
  for (int m = 0; m < BT; ++m) sum[m] = 0.0f;
  for (int64_t c0 = c_lo; c0 <= c_hi; c0 += B) {
    float4 part[B][NV];
#pragma unroll
    for (int j = 0; j < B; ++j) {
      const int64_t c = c0 + j;
      const float4* src = reinterpret_cast<const float4*>(
          a.ws + c * WS_FLOATS_PER_CTA + (c == c_lo ? slot_lo : 0) * BT * BM + r * BT);
#pragma unroll
      for (int k = 0; k < NV; ++k)
        part[j][k] = (c <= c_hi && k < nv) ? __ldcg(src + k) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
#pragma unroll
    for (int j = 0; j < B; ++j)
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        sum[4 * k] += part[j][k].x;
        sum[4 * k + 1] += part[j][k].y;
        sum[4 * k + 2] += part[j][k].z;
        sum[4 * k + 3] += part[j][k].w;
      }
  }
}

__device__ void epilogue(Shared& s, uint32_t tmem, const Args& a, int64_t p0, int64_t p1) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;
  const int r = 32 * q + lane;  // tile row (TMEM lane) of this thread
  const int64_t G = gridDim.x;
  const int tn_first = s.t_first / a.Tk, tn_last = s.t_last / a.Tk;
  const patch_tile_desc df = tile_desc(s, a, s.t_first), dl = tile_desc(s, a, s.t_last);
  // does the CTA hold the first panel of its first row / the last panel of its last row?
  const bool first_row_whole = s.t_first % a.Tk == 0 && p0 == panel_of(df);
  const bool last_row_whole = s.t_last % a.Tk == a.Tk - 1 && p1 == panel_of(dl) + (dl.kind ? 1 : 2);
  for (int tn = tn_first; tn <= tn_last; ++tn) {
    const int seg = tn - tn_first, buf = seg % NACC;
    // a warp-uniform decision: the tensor-memory load below is warp-collective
    const bool ok = wait_bounded(&s.acc_full[buf], (seg / NACC) & 1, &s.abort_flag, a.limit_ns, a.status, false);
    if (!__all_sync(0xFFFFFFFFu, ok)) break;
    tc_fence_after();
    uint32_t v[16];
    tmem_ld_16cols(tmem + (uint32_t(32 * q) << 16) + uint32_t(buf * BT), v);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.acc_empty[buf]);
    const int64_t n = int64_t(tn) * BM + r;
    if ((tn > tn_first || first_row_whole) && (tn < tn_last || last_row_whole)) {  // the whole row is ours
#pragma unroll
      for (int m = 0; m < BT; ++m)
        if (m < a.M) a.Y[int64_t(m) * a.N + n] = f32_to_bf16_rne(__uint_as_float(v[m]));
      continue;
    }
    // A cut row: publish this warp's 32 rows (its TMEM lane quarter q) of
    // partial sums and count the arrival; the last covering CTA to arrive for
    // quarter q adds up that quarter's partials (in CTA order) and stores them.
    // partial sums of row r: 16 consecutive floats (all 16 MMA columns)
    float4* mine = reinterpret_cast<float4*>(a.ws + int64_t(blockIdx.x) * WS_FLOATS_PER_CTA +
                                             (tn == tn_first ? 0 : BT * BM) + r * BT);
#pragma unroll
    for (int k = 0; k < BT / 4; ++k)
      if (4 * k < a.M)
        mine[k] = make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                              __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
    const int64_t rb = tn == tn_first ? s.row_lo[0] : s.row_hi[0];
    const int64_t re = tn == tn_first ? s.row_lo[1] : s.row_hi[1];
    const int64_t c_lo = cta_of_panel(rb, a.P, G), c_hi = cta_of_panel(re - 1, a.P, G);
    // the warp's partial stores are ordered before lane 0's release-acquire
    // increment; the last arriver's acquire makes every covering CTA's
    // partials visible to its later (L2) loads
    __syncwarp();
    uint32_t old = 0;
    if (lane == 0) old = atom_add_acq_rel_gpu(&a.counters[4 * tn + q], 1u);
    old = __shfl_sync(0xFFFFFFFFu, old, 0);
    if (old != uint32_t(c_hi - c_lo)) continue;
    __syncwarp();  // orders lane 0's acquire before every lane's loads
    // only the first covering CTA can have started before the row (its "last row" slot)
    const int slot_lo = range_begin(c_lo, a.P, G) < rb ? 1 : 0;
    const int nv = (a.M + 3) / 4;  // float4s per row that carry real tokens
    float sum[BT];
    if (nv <= 2)  // up to 8 tokens: 8 covering CTAs' partials per round of loads
      sum_partials<8, 2>(a, r, c_lo, c_hi, slot_lo, nv, sum);
    else
      sum_partials<4, BT / 4>(a, r, c_lo, c_hi, slot_lo, nv, sum);
#pragma unroll
    for (int m = 0; m < BT; ++m)
      if (m < a.M) a.Y[int64_t(m) * a.N + n] = f32_to_bf16_rne(sum[m]);
    if (lane == 0) a.counters[4 * tn + q] = 0;  // ready for the next call
  }
}

__global__ void __launch_bounds__(THREADS, 2)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const Args a) {
  extern __shared__ uint8_t smem_raw[];
  Shared& s = *reinterpret_cast<Shared*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t p0 = range_begin(blockIdx.x, a.P, G), p1 = range_begin(blockIdx.x + 1, a.P, G);
  pdl_launch_dependents();  // the next kernel may run its prologue as our CTAs finish

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s.full[i], 2);  // one arrival per producer thread
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < NACC; ++i) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 4);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmap_w);
    // The first weight panels need nothing but their index: request them now,
    // before the tile search, so HBM is busy from the CTA's first microsecond.
    // Their stages expect the rest of their bytes when the producer arms them.
    const int64_t n0 = p1 - p0 < NS ? p1 - p0 : NS;
    for (int j = 0; j < n0; ++j) {
      mbar_add_tx(&s.full[j], A_BYTES);
      tma_load_2d(s.st[j].a, &tmap_w, &s.full[j], 0, int((p0 + j) * 128));
    }
    prefetch_tensormap(&tmap_x);
  }
  // locate the CTA's first and last tile, stage their descriptors and the
  // tile-row boundaries the epilogue needs for rows cut by this CTA's range
  // (G <= P, so every CTA has at least one panel)
  if (!locate_one_round(s, a, p0, p1 - 1)) {
    int ta, tb;
    find_tiles(a.desc, a.Tn * a.Tk, a.P, p0, p1 - 1, ta, tb);
    const int count = tb - ta + 1;
    if (threadIdx.x == 0) {
      s.t_first = ta;
      s.t_last = tb;
      s.cached = count <= DCAP;
    }
    if (count <= DCAP)
      for (int i = threadIdx.x; i < count; i += blockDim.x) s.dcache[i] = a.desc[ta + i];
    if (threadIdx.x < 4) {
      const int tn = (threadIdx.x < 2 ? ta : tb) / a.Tk + (threadIdx.x & 1);
      const int64_t v = tn < a.Tn ? panel_of(a.desc[int64_t(tn) * a.Tk]) : a.P;
      if (threadIdx.x < 2)
        s.row_lo[threadIdx.x] = v;
      else
        s.row_hi[threadIdx.x - 2] = v;
    }
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    if (lane == 0) producer_w(s, &tmap_w, a, p0, p1);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_issuer(s, tmem, a, p0, p1);
    __syncwarp();
  } else if (warp == 6) {
    if (lane == 0) producer_x(s, &tmap_x, a, p0, p1);
    __syncwarp();
  } else {
    epilogue(s, tmem, a, p0, p1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

struct Plan {
  int64_t Tn, Tk, P, G;
  size_t ws_floats_bytes;
};

static Plan plan(const patch_weight& W, int num_sms) {
  Plan p;
  p.Tn = W.N / kTile;
  p.Tk = W.K / kTile;
  const int64_t T = p.Tn * p.Tk;
  p.P = 2 * (T - W.n_sparse) + W.n_sparse;
  // 1.5 CTAs per SM: with two CTA slots per SM, half the SMs run two of this
  // kernel's CTAs (8 stages in flight) while the other half keep a slot for
  // the next kernel's CTAs to fetch their first panels early.  Measured on the
  // LLaMA-2-7B decode step: 1x 3410 GB/s, 1.3-1.75x 3580-3610, 2x 3420.
  const int64_t g = int64_t(num_sms) * 3 / 2;
  p.G = p.P < g ? p.P : g;
  p.ws_floats_bytes = size_t(p.G) * WS_FLOATS_PER_CTA * sizeof(float);
  return p;
}

}  // namespace decode_tc

size_t decode_tc_workspace_bytes(int64_t M, const patch_weight& W, int num_sms) {
  (void)M;
  const decode_tc::Plan p = decode_tc::plan(W, num_sms);
  return kDecodeCounterBytes + p.ws_floats_bytes;
}

cudaError_t launch_decode_tc(const uint16_t* X, int64_t M, const patch_weight& W, uint16_t* Y, void* workspace,
                             int32_t* status, int num_sms, uint64_t limit_ns, cudaStream_t stream) {
  using namespace decode_tc;
  const Plan pl = plan(W, num_sms);
  if (pl.Tn > kDecodeMaxTileRows) return cudaErrorInvalidValue;
  CUtensorMap tmap_x, tmap_w;
  // X boxes carry exactly the M token rows: the MMA still reads 16 rows (N = 16),
  // but accumulator columns >= M are never stored, so rows >= M may hold anything
  if (!make_map_2d_bf16(&tmap_x, X, uint64_t(W.K), uint64_t(M), uint64_t(W.K) * 2, 64, uint32_t(M)))
    return cudaErrorUnknown;
  if (!make_map_2d_bf16(&tmap_w, W.values, 64, uint64_t(pl.P) * 128, 128, 64, 128)) return cudaErrorUnknown;
  Args a;
  a.desc = W.desc;
  a.meta = static_cast<const uint8_t*>(W.meta);
  a.Y = Y;
  a.counters = static_cast<uint32_t*>(workspace);
  a.ws = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kDecodeCounterBytes);
  a.M = int(M);
  a.N = int(W.N);
  a.Tk = int(pl.Tk);
  a.Tn = int(pl.Tn);
  a.P = pl.P;
  a.limit_ns = limit_ns;
  a.status = status;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_tc_kernel, dim3(unsigned(pl.G)), dim3(THREADS), SMEM_BYTES, stream, tmap_x, tmap_w, a);
}

}  // namespace patch
