// patch_gemm64: the hybrid layer Y[m][n] = sum_k X[m][k] * W_eff[n][k] on
// 64 x 64 execution tiles ("PATCH: Learnable Tile-level Hybrid Sparsity for
// LLMs", section 4 "Experimental Results", "Ablation Studies": the tile size
// trades finer control over where the 2:4 pattern applies against hardware
// efficiency; section 2 "Inference & Deployment": dense tiles on the dense
// tensor-core MMA, 2:4 tiles on the sparse one).
//
// The packed weight is a sequence of P panels of 4 KiB (64 rows x 32 bf16,
// 64-byte rows): a dense 64 x 64 tile is 2 consecutive panels, a sparse one
// 1 panel of kept values plus a 512-byte metadata block.  A dense tile is
// four M = 64 kind::f16 K = 16 MMAs, a sparse one two .sp K = 32 MMAs.
//
// Work split (stream-K): the tokens are cut into J blocks of BT (16 when
// M <= 16, else 256).  Over the sequence of (token block, tile) pairs, the
// position of a pair is that of its tile's first panel (j * P + panel), V =
// J * P positions in all; CTA c of G takes the pairs whose
// position lies in [c*V/G, (c+1)*V/G), so every CTA streams the same number
// of stored bytes to within one panel.  A CTA accumulates each (token block,
// tile row) segment of its share in tensor memory; a segment inside one share
// is rounded to bf16 and stored, a cut one is finished by the last covering
// CTA to arrive, which adds the fp32 partials in CTA order (deterministic)
// and resets its arrival counter.
//
// One pipeline stage per tile: its weight (one TMA copy of 8 or 4 KiB,
// 64-byte swizzle), its 64-k slice of X (one TMA copy, 128-byte swizzle) and,
// for a sparse tile, its metadata block (one bulk copy).  A thread issuing
// copies, or MMAs, spends about 100 ns on each, so the work is spread out.
// Warps: 0 W producer, 1 X producer (writes each stage's info word), 2
// metadata producer (each walks the tile kinds itself), 3 and 12 the MMA
// issuers (issuer u takes every NISS-th K step of a tile into its own
// accumulator; warp 3 owns tensor memory), 4-7 epilogue (lane quarter
// q = warp % 4), 8-11 metadata stagers: the M = 64 sparse MMA reads its
// metadata from the first 16 lanes of each 32-lane quarter, a placement no
// shared-to-tensor-memory copy shape produces from a compact block, so each
// stager warp moves its quarter's 128 bytes with one 32-lane, 2-column
// tensor-memory store.  Every wait is bounded in time (PATCH_DEV_TIMEOUT).
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace patch {
namespace g64 {

using namespace tc;

constexpr int BM = 64;                              // tile rows = MMA M
constexpr uint32_t PANEL = PATCH_PANEL64_BYTES;     // 64 rows x 32 bf16
constexpr uint32_t META = PATCH_META_TILE64_BYTES;  // metadata of one sparse tile
constexpr int THREADS = 13 * 32;
constexpr uint32_t FULL_MASK = 0xFFFFFFFFu;
constexpr uint32_t INFO_SPARSE = 1u, INFO_SEG_START = 2u, INFO_SEG_END = 4u;

// BT = 16 (decode): two CTAs per SM, two MMA issuers each (a 4-8 KiB tile is
// little work for the ~100 ns a thread spends per MMA, per copy and per loop
// turn, so two CTAs' control threads run side by side); BT = 256 (prefill):
// one CTA per SM, one issuer whose four N = 256 MMAs per tile take about as
// long to issue as to run.
template <int BT>
struct Cfg {
  static constexpr int CTAS_PER_SM = BT == 16 ? 2 : 1;
  static constexpr int NISS = BT == 16 ? 2 : 1;   // MMA-issuing threads
  static constexpr int NS = BT == 16 ? 8 : 5;     // pipeline stages (tiles)
  static constexpr int NACC = BT == 16 ? 2 : 1;   // accumulator buffers per issuer
  static constexpr int X_BYTES = BT * 128;        // one 64-k slice of X: BT token rows x 128 B
  static constexpr uint32_t META_COL0 = uint32_t(NACC * NISS * BT);  // then 4 columns per stage
  static constexpr uint32_t TMEM_COLS = META_COL0 + 4 * NS <= 256 ? 256u : 512u;
  static constexpr uint32_t IDESC_DENSE = idesc_bf16(BM, BT, false);
  static constexpr uint32_t IDESC_SPARSE = idesc_bf16(BM, BT, true);
  static_assert(META_COL0 + 4 * NS <= TMEM_COLS && TMEM_COLS <= 512, "tensor memory layout");
};

template <int BT>
struct Stage {
  alignas(1024) uint8_t a[2 * PANEL];  // a dense tile's 2 panels (k 0..31, 32..63), or a sparse tile's 1
  alignas(1024) uint8_t x[Cfg<BT>::X_BYTES];
  alignas(16) uint8_t e[META];
};

template <int BT>
struct Shared {
  static constexpr int NS = Cfg<BT>::NS, NACC = Cfg<BT>::NACC;
  Stage<BT> st[NS];
  uint64_t full[NS], ready[NS], empty[NS];
  uint64_t acc_full[NACC], acc_empty[NACC], drain[2];
  uint32_t info[NS];
  uint32_t tmem_base;
  int abort_flag;
  int64_t vt_first, n_tiles;  // the share: n_tiles (token block, tile) pairs from virtual tile vt_first
};
template <int BT>
constexpr size_t smem_bytes() {
  return sizeof(Shared<BT>) + 1024;
}
static_assert(2 * (smem_bytes<16>() + 1024) <= 228 * 1024 && smem_bytes<256>() <= 227 * 1024,
              "shared memory budget");

struct Args {
  const patch_tile_desc* desc;
  const uint8_t* meta;
  uint16_t* Y;
  float* ws;           // [G][2][64][BT] fp32 partials (contents between calls do not matter)
  uint32_t* counters;  // [J][Tn][4] arrivals per segment and lane quarter (zero between calls)
  int M, N, Tk, Tn, J;
  int T;      // tiles of the weight
  int64_t P;  // panels of the weight
  int64_t V;  // J * P
  uint64_t limit_ns;
  uint64_t drain_ns;  // limit of the final waits for copies and MMAs in flight (at least 20 ms)
  int32_t* status;
};

__host__ __device__ __forceinline__ int64_t range_begin(int64_t c, int64_t V, int64_t G) { return c * V / G; }
// the CTA whose range of positions holds position v
__host__ __device__ __forceinline__ int64_t cta_of(int64_t v, int64_t V, int64_t G) {
  return ((v + 1) * G - 1) / V;
}

__device__ __forceinline__ int64_t panel_of(const patch_tile_desc* desc, int64_t t) {
  return int64_t(desc[t].val_offset / PANEL);
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// The tiles holding panels pa and pb (the last t with panel_of(t) <= p),
// found by the whole block: first a window of blockDim.x tiles around the
// proportional estimate p*T/P (enough unless the sparse tiles are very
// unevenly spread), else rounds of blockDim.x evenly spaced probes, each
// narrowing the span by that factor.
__device__ void find_tiles(const patch_tile_desc* desc, int T, int64_t P, int64_t pa, int64_t pb, int& ta,
                           int& tb) {
  const int n = blockDim.x, i = threadIdx.x;
  auto window = [&](int64_t p) {
    int64_t w = p * T / P - n / 2;
    if (w > T - n) w = T - n;
    return int(w < 0 ? 0 : w);
  };
  const int wa = window(pa), wb = window(pb);
  const int ca = __syncthreads_count(wa + i < T && panel_of(desc, wa + i) <= pa);
  const int cb = __syncthreads_count(wb + i < T && panel_of(desc, wb + i) <= pb);
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
    const int ka = __syncthreads_count(in && ia < T && panel_of(desc, ia) <= pa);
    const int kb = __syncthreads_count(in && ib < T && panel_of(desc, ib) <= pb);
    lo_a += (ka - 1) * step;
    lo_b += (kb - 1) * step;
    span = step;
  }
  ta = lo_a;
  tb = lo_b;
}

// A producer warp's walk over its share's tiles: token block j, tile t (its
// K-tile kt), its first panel p and metadata ordinal, and the kinds of the 32
// tiles around t, loaded by the whole warp (one descriptor per lane, the next
// 32 prefetched).  Every lane holds the same state.
struct Walk {
  int64_t j, p;
  int t, kt;
  uint32_t ord;        // sparse tiles before t
  uint32_t kinds;      // bit i: tile (t & ~31) + i is sparse
  uint32_t next_kind;  // this lane's tile of the next 32

  __device__ __forceinline__ void load_batch(const Args& a, int base) {
    const int lane = threadIdx.x & 31;
    kinds = __ballot_sync(FULL_MASK, base + lane < a.T && a.desc[base + lane].kind != 0);
    next_kind = base + 32 + lane < a.T ? a.desc[base + 32 + lane].kind : 0u;
  }
  __device__ __forceinline__ void start(const Args& a, int64_t vt) {
    j = vt / a.T;
    t = int(vt - j * a.T);
    p = panel_of(a.desc, t);
    kt = t % a.Tk;
    ord = uint32_t(2 * int64_t(t) - p);  // a dense tile before t is 2 panels, a sparse one 1
    load_batch(a, t & ~31);
  }
  __device__ __forceinline__ bool sparse() const { return (kinds >> (t & 31)) & 1u; }
  __device__ __forceinline__ uint32_t info(bool first, bool last, int Tk) const {
    uint32_t v = sparse() ? INFO_SPARSE : 0u;
    if (first || kt == 0) v |= INFO_SEG_START;
    if (last || kt == Tk - 1) v |= INFO_SEG_END;
    return v;
  }
  __device__ __forceinline__ void next(const Args& a) {
    const bool sp = sparse();
    ord += sp ? 1u : 0u;
    p += sp ? 1 : 2;
    ++t;
    if (++kt == a.Tk) kt = 0;
    if (t == a.T) {  // next token block
      t = 0;
      p = 0;
      ++j;
      ord = 0;
      load_batch(a, 0);
    } else if ((t & 31) == 0) {
      const int lane = threadIdx.x & 31;
      kinds = __ballot_sync(FULL_MASK, next_kind != 0);
      next_kind = t + 32 + lane < a.T ? a.desc[t + 32 + lane].kind : 0u;
    }
  }
};

// The three producers share this loop: stage i of the share is armed by
// `issue` once the MMAs of stage i - NS have released it (the first NS
// without waiting).  The warp's lane 0 waits and issues; every lane walks.
// Every copy issued lands before the CTA exits.
template <int BT, typename Issue>
__device__ void produce(Shared<BT>& s, const Args& a, Issue&& issue) {
  constexpr int NS = Cfg<BT>::NS;
  const int lane = threadIdx.x & 31;
  Walk w;
  w.start(a, s.vt_first);
  int64_t i = 0;
  for (; i < s.n_tiles; ++i) {
    const int st = int(i % NS);
    bool ok = true;
    if (lane == 0 && i >= NS)
      ok = wait_bounded(&s.empty[st], uint32_t((i / NS) & 1) ^ 1u, &s.abort_flag, a.limit_ns, a.status, false);
    if (!__shfl_sync(FULL_MASK, ok, 0)) break;
    if (lane == 0) issue(st, i, w);
    w.next(a);
  }
  if (lane == 0)
    for (int64_t k = i > NS ? i - NS : 0; k < i; ++k)
      wait_bounded(&s.full[k % NS], uint32_t((k / NS) & 1), &s.abort_flag, a.drain_ns, a.status, true);
}

// Metadata stager (4 warps, lane quarter q): for a sparse stage, the 8 bytes
// of lane i < 16 of quarter q go to tensor-memory lane 32q + i, columns
// META_COL0 + 4*stage + 0..1 (lanes 16..31 get zeros the MMA never reads).
// Every stage, dense or not, is passed on to the MMA issuers through `ready`.
template <int BT>
__device__ void meta_stager(Shared<BT>& s, uint32_t tmem, const Args& a) {
  using C = Cfg<BT>;
  const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) & 3;
  for (int64_t i = 0; i < s.n_tiles; ++i) {
    const int st = int(i % C::NS);
    const bool ok =
        wait_bounded(&s.full[st], uint32_t((i / C::NS) & 1), &s.abort_flag, a.limit_ns, a.status, false);
    if (!__all_sync(FULL_MASK, ok)) break;
    const uint32_t info = *reinterpret_cast<volatile uint32_t*>(&s.info[st]);
    if (info & INFO_SPARSE) {
      uint2 m = make_uint2(0u, 0u);
      if (lane < 16) m = *reinterpret_cast<const uint2*>(s.st[st].e + 128 * q + 8 * lane);
      __syncwarp();  // converged for the warp-collective store
      tmem_st_32x32b_x2(tmem + (uint32_t(32 * q) << 16) + C::META_COL0 + 4u * uint32_t(st), m.x, m.y);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.ready[st]);
  }
}

// MMA issuer u of NISS: the K steps kb = u, u + NISS, ... of a tile (a dense
// tile's four K = 16 steps, a sparse one's two K = 32 steps, step kb reading
// metadata column kb of its stage's slot through the selector), into its own
// accumulator.  `ready` implies `full`: the stagers pass a stage on only
// after waiting for it.
template <int BT>
__device__ void mma_issuer(Shared<BT>& s, uint32_t tmem, const Args& a, int u) {
  using C = Cfg<BT>;
  uint32_t seg = 0, acc = tmem, accumulate = 0;
  for (int64_t i = 0; i < s.n_tiles; ++i) {
    const int st = int(i % C::NS);
    const uint32_t ph = uint32_t((i / C::NS) & 1);
    if (!wait_bounded(&s.ready[st], ph, &s.abort_flag, a.limit_ns, a.status, false)) break;
    const uint32_t info = *reinterpret_cast<volatile uint32_t*>(&s.info[st]);
    if (info & INFO_SEG_START) {  // a new segment starts a new accumulation
      const uint32_t buf = seg % C::NACC;
      if (!wait_bounded(&s.acc_empty[buf], ((seg / C::NACC) & 1) ^ 1u, &s.abort_flag, a.limit_ns, a.status, false))
        break;
      acc = tmem + (buf * C::NISS + uint32_t(u)) * uint32_t(BT);
      accumulate = 0;
    }
    tc_fence_after();
    Stage<BT>& g = s.st[st];
    const uint64_t a0 = sw64_desc(smem_u32(g.a)), b0 = sw128_desc(smem_u32(g.x));
    if (info & INFO_SPARSE) {
      // 32 k per step: 16 kept values = 32 B of each A row, 64 B of each X row
      for (int kb = u; kb < 2; kb += C::NISS) {
        mma_sparse(acc, a0 + uint64_t(kb * 32 >> 4), b0 + uint64_t(kb * 64 >> 4),
                   tmem + C::META_COL0 + 4u * uint32_t(st), C::IDESC_SPARSE | uint32_t(kb), accumulate);
        accumulate = 1;
      }
    } else {
      // 16 k per step: panel kb / 2, 32 B into its rows; 32 B steps along X
      for (int kb = u; kb < 4; kb += C::NISS) {
        mma_dense(acc, a0 + uint64_t(((kb >> 1) * PANEL + (kb & 1) * 32) >> 4), b0 + uint64_t(kb * 32 >> 4),
                  C::IDESC_DENSE, accumulate);
        accumulate = 1;
      }
    }
    tc_commit(&s.empty[st]);
    if (info & INFO_SEG_END) {
      tc_commit(&s.acc_full[seg % C::NACC]);
      ++seg;
    }
  }
  tc_commit(&s.drain[u]);
  wait_bounded(&s.drain[u], 0, &s.abort_flag, a.drain_ns, a.status, true);
}

// CH accumulator columns starting at c0 of this warp's lane quarter, summed
// over the issuers' accumulators (in issuer order).
template <int BT, int CH>
__device__ __forceinline__ void load_acc(uint32_t tmem, int q, uint32_t buf, int c0, float (&v)[CH]) {
  constexpr int NISS = Cfg<BT>::NISS;
#pragma unroll
  for (int u = 0; u < NISS; ++u) {
    uint32_t raw[CH];
    const uint32_t addr = tmem + (uint32_t(32 * q) << 16) + (buf * NISS + uint32_t(u)) * uint32_t(BT) + uint32_t(c0);
    if constexpr (CH == 16)
      tmem_ld_16cols(addr, raw);
    else
      tmem_ld_32cols(addr, raw);
#pragma unroll
    for (int c = 0; c < CH; ++c) v[c] = (u == 0 ? 0.0f : v[c]) + __uint_as_float(raw[c]);
  }
}

// Epilogue (4 warps; lane i < 16 of quarter q holds tile row 16q + i, the M = 64
// accumulator layout).  Segments of the share in order; a whole one is
// stored.  A cut one goes through the partials: a CTA writes its slot 1 for
// the segment that starts inside its share and continues after it, its slot
// 0 for one that started before its share; so the first covering CTA's
// partials are in its slot 1 and every later one's in slot 0.
template <int BT>
__device__ void epilogue(Shared<BT>& s, uint32_t tmem, const Args& a) {
  using C = Cfg<BT>;
  constexpr int CH = BT < 32 ? BT : 32;
  constexpr int NB = BT == 16 ? 2 : 4;  // covering CTAs whose partials are loaded per round
  const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) & 3;
  const int r = 16 * q + lane;
  const bool act = lane < 16;
  const int64_t G = gridDim.x;
  if (s.n_tiles <= 0) return;
  const int64_t vt0 = s.vt_first, vt1 = s.vt_first + s.n_tiles - 1;
  const int64_t s0 = (vt0 / a.T) * a.Tn + (vt0 % a.T) / a.Tk;
  const int64_t s1 = (vt1 / a.T) * a.Tn + (vt1 % a.T) / a.Tk;
  for (int64_t sg = s0; sg <= s1; ++sg) {
    const int64_t k = sg - s0, j = sg / a.Tn;
    const int tn = int(sg - j * a.Tn);
    const int64_t t_row = int64_t(tn) * a.Tk;  // first tile of the row
    const int64_t c_lo = cta_of(j * a.P + panel_of(a.desc, t_row), a.V, G);
    const int64_t c_hi = cta_of(j * a.P + panel_of(a.desc, t_row + a.Tk - 1), a.V, G);
    const bool whole = c_lo == c_hi;
    const bool started_before = j * a.T + t_row < vt0;
    const uint32_t buf = uint32_t(k % C::NACC);
    // a warp-uniform decision: the tensor-memory loads below are warp-collective
    const bool ok =
        wait_bounded(&s.acc_full[buf], uint32_t(k / C::NACC) & 1u, &s.abort_flag, a.limit_ns, a.status, false);
    if (!__all_sync(FULL_MASK, ok)) break;
    tc_fence_after();
    const int64_t n = int64_t(tn) * BM + r;
    const int64_t m0 = j * BT;  // first token of the block
    float* mine =
        a.ws + (int64_t(blockIdx.x) * 2 + (started_before ? 0 : 1)) * (BM * BT) + int64_t(r) * BT;
#pragma unroll 1
    for (int c0 = 0; c0 < BT; c0 += CH) {
      float v[CH];
      __syncwarp();  // converged for the warp-collective loads
      load_acc<BT, CH>(tmem, q, buf, c0, v);
      if (!act) continue;
      if (whole) {
#pragma unroll
        for (int c = 0; c < CH; ++c)
          if (m0 + c0 + c < a.M) a.Y[(m0 + c0 + c) * a.N + n] = f32_to_bf16_rne(v[c]);
      } else {
#pragma unroll
        for (int c = 0; c < CH; c += 4)
          if (m0 + c0 + c < a.M)
            *reinterpret_cast<float4*>(mine + c0 + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.acc_empty[buf]);
    if (whole) continue;
    // count this warp's arrival (its 16 rows); the last covering CTA adds
    // every covering CTA's partials in CTA order
    uint32_t* counter = a.counters + (j * a.Tn + tn) * 4 + q;
    uint32_t old = 0;
    if (lane == 0) old = atom_add_acq_rel_gpu(counter, 1u);  // after the warp's partial stores (syncwarp above)
    old = __shfl_sync(FULL_MASK, old, 0);
    if (old != uint32_t(c_hi - c_lo)) continue;
    __syncwarp();  // lane 0's acquire before every lane's loads
#pragma unroll 1
    for (int c0 = 0; c0 < BT; c0 += CH) {
      float sum[CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) sum[c] = 0.0f;
#pragma unroll 1
      for (int64_t cb = c_lo; cb <= c_hi; cb += NB) {
        float4 part[NB][CH / 4];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const int64_t c = cb + b;
          const float4* src = reinterpret_cast<const float4*>(
              a.ws + (c * 2 + (c == c_lo ? 1 : 0)) * (BM * BT) + int64_t(r) * BT + c0);
#pragma unroll
          for (int i4 = 0; i4 < CH / 4; ++i4)
            part[b][i4] = (act && c <= c_hi && m0 + c0 + 4 * i4 < a.M) ? __ldcg(src + i4)
                                                                        : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int i4 = 0; i4 < CH / 4; ++i4) {
            sum[4 * i4] += part[b][i4].x;
            sum[4 * i4 + 1] += part[b][i4].y;
            sum[4 * i4 + 2] += part[b][i4].z;
            sum[4 * i4 + 3] += part[b][i4].w;
          }
      }
      if (act) {
#pragma unroll
        for (int c = 0; c < CH; ++c)
          if (m0 + c0 + c < a.M) a.Y[(m0 + c0 + c) * a.N + n] = f32_to_bf16_rne(sum[c]);
      }
    }
    if (lane == 0) *counter = 0;  // ready for the next call
  }
}

template <int BT>
__global__ void __launch_bounds__(THREADS, Cfg<BT>::CTAS_PER_SM)
    gemm64_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                  const __grid_constant__ CUtensorMap tmap_w2, const Args a) {
  using C = Cfg<BT>;
  extern __shared__ uint8_t smem_raw[];
  Shared<BT>& s =
      *reinterpret_cast<Shared<BT>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t r0 = range_begin(blockIdx.x, a.V, G), r1 = range_begin(blockIdx.x + 1, a.V, G);
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&s.full[i], 3);   // W, X and metadata producers
      mbar_init(&s.ready[i], 4);  // the 4 metadata stagers
      mbar_init(&s.empty[i], C::NISS);
    }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(&s.acc_full[i], C::NISS);
      mbar_init(&s.acc_empty[i], 4);
    }
    for (int i = 0; i < C::NISS; ++i) mbar_init(&s.drain[i], 1);
    s.abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmap_w);
    prefetch_tensormap(&tmap_w2);
    prefetch_tensormap(&tmap_x);
  }
  // The share: tiles whose first panel's position lies in [r0, r1).  The
  // tile holding position r0 belongs to this CTA if it starts there, else
  // (the second panel of a dense tile) to the previous one; the tile holding
  // r1 - 1 starts at or before it and is the share's last.
  {
    int ta, tb;
    find_tiles(a.desc, a.T, a.P, r0 % a.P, (r1 - 1) % a.P, ta, tb);
    if (threadIdx.x == 0) {
      int64_t first = (r0 / a.P) * a.T + ta;
      if (panel_of(a.desc, ta) < r0 % a.P) ++first;
      const int64_t last = ((r1 - 1) / a.P) * a.T + tb;
      s.vt_first = first;
      s.n_tiles = last - first + 1;  // >= 1: the range spans at least 2 positions
    }
  }
  if (warp == 3) tmem_alloc(&s.tmem_base, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const int64_t n = s.n_tiles;

  if (warp == 0) {  // W producer: the tile's panels in one copy
    produce(s, a, [&](int st, int64_t i, const Walk& w) {
      const bool sp = w.sparse();
      mbar_expect_tx(&s.full[st], sp ? PANEL : 2 * PANEL);
      tma_load_2d(s.st[st].a, sp ? &tmap_w : &tmap_w2, &s.full[st], 0, int(w.p * BM));
    });
  } else if (warp == 1) {  // X producer: the stage's info word and 64-k slice of X
    const uint32_t xb = uint32_t(a.M < BT ? a.M : BT) * 128u;
    pdl_wait_previous();  // X may be the previous kernel's output
    produce(s, a, [&](int st, int64_t i, const Walk& w) {
      s.info[st] = w.info(i == 0, i + 1 == n, a.Tk);  // published by this thread's arrival
      mbar_expect_tx(&s.full[st], xb);
      tma_load_2d(s.st[st].x, &tmap_x, &s.full[st], w.kt * 64, int(w.j * BT));
    });
  } else if (warp == 2) {  // metadata producer
    produce(s, a, [&](int st, int64_t i, const Walk& w) {
      if (w.sparse()) {
        mbar_expect_tx(&s.full[st], META);
        bulk_load(s.st[st].e, a.meta + uint64_t(w.ord) * META, META, &s.full[st]);
      } else {
        mbar_arrive(&s.full[st]);
      }
    });
  } else if (warp == 3 || warp == 12) {
    const int u = warp == 3 ? 0 : 1;
    if (lane == 0 && u < C::NISS) mma_issuer(s, tmem, a, u);
    __syncwarp();
  } else if (warp < 8) {
    epilogue(s, tmem, a);
  } else {
    meta_stager(s, tmem, a);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

struct Plan {
  int BT, J;
  int64_t Tn, Tk, T, P, V, G;
  size_t counter_bytes, ws_bytes;
};

static Plan plan(int64_t M, const patch_weight64& W, int num_sms) {
  Plan p;
  p.BT = M <= 16 ? 16 : 256;
  p.J = int((M + p.BT - 1) / p.BT);
  p.Tn = W.N / BM;
  p.Tk = W.K / BM;
  p.T = p.Tn * p.Tk;
  p.P = 2 * (p.T - W.n_sparse) + W.n_sparse;
  p.V = int64_t(p.J) * p.P;
  // every CTA's range spans at least 2 positions, so it holds a tile start and
  // owns a tile: the owners of a segment's tiles are then exactly the CTAs
  // c_lo..c_hi between its first and last tile's owners
  const int64_t gmax = int64_t(num_sms) * (p.BT == 16 ? g64::Cfg<16>::CTAS_PER_SM : g64::Cfg<256>::CTAS_PER_SM);
  p.G = p.V >= 2 ? (p.V / 2 < gmax ? p.V / 2 : gmax) : 1;
  p.counter_bytes = (size_t(p.J) * size_t(p.Tn) * 16 + 255) / 256 * 256;
  p.ws_bytes = size_t(p.G) * 2 * BM * p.BT * sizeof(float);
  return p;
}

template <int BT>
static cudaError_t launch(const CUtensorMap& tmap_x, const CUtensorMap& tmap_w, const CUtensorMap& tmap_w2,
                          const Args& a, int64_t G, cudaStream_t stream) {
  cudaError_t e =
      cudaFuncSetAttribute(gemm64_kernel<BT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_bytes<BT>()));
  if (e != cudaSuccess) return e;
  return launch_pdl(gemm64_kernel<BT>, dim3(unsigned(G)), dim3(THREADS), smem_bytes<BT>(), stream, tmap_x, tmap_w,
                    tmap_w2, a);
}

}  // namespace g64

size_t gemm64_workspace_bytes(int64_t M, const patch_weight64& W, int num_sms) {
  if (M <= 0) return 0;
  const g64::Plan p = g64::plan(M, W, num_sms);
  return p.counter_bytes + p.ws_bytes;
}

cudaError_t launch_gemm64(const uint16_t* X, int64_t M, const patch_weight64& W, uint16_t* Y, void* workspace,
                          int32_t* status, int num_sms, uint64_t limit_ns, cudaStream_t stream) {
  using namespace g64;
  const Plan pl = plan(M, W, num_sms);
  if (pl.P * BM > int64_t(INT32_MAX) || int64_t(pl.J) * pl.BT > int64_t(INT32_MAX) || pl.T > int64_t(INT32_MAX))
    return cudaErrorInvalidValue;
  CUtensorMap tmap_x, tmap_w, tmap_w2;
  // X slices of 64 k x (up to) BT tokens, 128-byte swizzle; the box holds
  // min(M, BT) rows (rows past M in the last block read as zeros, rows the box
  // does not cover are never stored)
  const uint32_t box_rows = uint32_t(M < pl.BT ? M : pl.BT);
  if (!make_map_2d_bf16(&tmap_x, X, uint64_t(W.K), uint64_t(M), uint64_t(W.K) * 2, 64, box_rows))
    return cudaErrorUnknown;
  // the values blob as rows of 64 bytes: a sparse tile is 64 of them, a dense one 128
  if (!make_map_2d_bf16_sw64(&tmap_w, W.values, 32, uint64_t(pl.P) * BM, 64, 32, BM)) return cudaErrorUnknown;
  if (!make_map_2d_bf16_sw64(&tmap_w2, W.values, 32, uint64_t(pl.P) * BM, 64, 32, 2 * BM)) return cudaErrorUnknown;
  Args a;
  a.desc = W.desc;
  a.meta = static_cast<const uint8_t*>(W.meta);
  a.Y = Y;
  a.counters = static_cast<uint32_t*>(workspace);
  a.ws = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + pl.counter_bytes);
  a.M = int(M);
  a.N = int(W.N);
  a.Tk = int(pl.Tk);
  a.Tn = int(pl.Tn);
  a.J = pl.J;
  a.T = int(pl.T);
  a.P = pl.P;
  a.V = pl.V;
  a.limit_ns = limit_ns;
  a.drain_ns = limit_ns > 20000000ull ? limit_ns : 20000000ull;
  a.status = status;
  return pl.BT == 16 ? launch<16>(tmap_x, tmap_w, tmap_w2, a, pl.G, stream)
                     : launch<256>(tmap_x, tmap_w, tmap_w2, a, pl.G, stream);
}

}  // namespace patch
