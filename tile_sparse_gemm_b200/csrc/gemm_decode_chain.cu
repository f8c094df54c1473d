// patch_gemm_chain: a sequence of decode GEMMs (M <= 16 tokens each) run by
// one persistent launch, so that the weight stream of the next call overlaps
// the end of the current one.
//
// Layer: Y[m][n] = sum_k X[m][k] * W_eff[n][k] with W_eff the hybrid weight
// of "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs" (section 2
// "Methodology: PATCH", "Core Mechanism" and "Inference & Deployment": dense
// 128 x 128 tiles on dense tensor-core MMA, 2:4 tiles on the sparse ones).
//
// Why one launch: a decode GEMM of a 4096 x 4096 layer moves ~26 MB, about
// 4 us of HBM time, but as its own kernel it also pays the previous kernel's
// drain, the start of its own CTAs, the X load after its dependency resolves
// and the finish of tile rows cut between CTAs -- a few microseconds in which
// the HBM idles.  Here every CTA stays resident for the whole chain and keeps
// one ring of weight panels across calls: its W producer needs nothing but
// panel indices, so it streams call j+1's panels while call j finishes; only
// the X loads of a dependent call wait for the previous call to complete
// (a grid-wide completion counter per call instead of a kernel boundary).
//
// Work split per call (stream-K over panels, as in the single-call decode
// kernel): the values blob is a sequence of P panels (16 KiB: a dense tile is
// 2 panels, a sparse tile 1) in row-major tile order; CTA c of G takes panels
// [c*P/G, (c+1)*P/G).  A tile row inside one CTA's range is rounded and
// stored directly; a row cut between CTAs is finished, per 32-row quarter, by
// whichever covering CTA's epilogue warp arrives last, which adds all fp32
// partials in CTA order (deterministic).
//
// Launch: a plan kernel first writes, for every panel of every call, the tile
// it belongs to (tile index, half, kind, sparse ordinal); then the chain
// kernel runs cooperatively (all CTAs resident: they wait on each other's
// completion counters), one CTA per SM.  Roles per CTA (9 warps): warp 0 W
// producer, warps 6 and 8 X producers (panel records, metadata, X slices, the
// dependency waits; each takes every other panel: one thread's turn per panel,
// up to three copies and the record bookkeeping, took ~420 ns and set the pace
// of the whole ring at ~5.5 TB/s), warps 1 and 7 MMA issuers (warp 1 owns
// TMEM), each issuing half of every panel's MMAs into its own accumulator (one
// thread issuing all of them caps an SM at ~5.5 TB/s of weight panels, two
// reach the memory's ~7 TB/s), warps 2-5 epilogue.
// Every wait, on an mbarrier or on another CTA's counter, is bounded in time.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace patch {
namespace chain {

using namespace tc;

constexpr int BM = 128;
constexpr int BT = 16;                   // MMA N (tokens)
constexpr int NS = 10;                   // pipeline stages per CTA (one CTA per SM)
constexpr int NACC = 2;                  // accumulator buffers
constexpr int A_BYTES = PATCH_PANEL_BYTES;
constexpr int X_BYTES = BT * 64 * 2;     // one 64-k slice of X (room for 16 token rows)
constexpr int E_BYTES = PATCH_META_TILE_BYTES;
constexpr int NISS = 2;                  // MMA-issuing threads, each half of every panel's K
constexpr int THREADS = 288;             // warps: 0 W producer, 1 and 7 MMA, 2-5 epilogue, 6 and 8 X producers
constexpr uint32_t TMEM_COLS = 256;
// accumulator of segment buffer b, issuer u: columns (NISS b + u) BT; issuer u's
// metadata slot of stage st: META_COL0 + 4 (NS u + st)
constexpr uint32_t META_COL0 = NACC * NISS * BT;
static_assert(META_COL0 + 4 * NS * NISS <= TMEM_COLS, "TMEM layout");
constexpr uint32_t IDESC_DENSE = idesc_bf16(BM, BT, false);
constexpr uint32_t IDESC_SPARSE = idesc_bf16(BM, BT, true);
constexpr int WS_FLOATS_PER_CTA = 2 * BT * BM;  // [2 slots][128 rows][16 tokens]
constexpr int PART_RING = 4;                    // partial-sum buffers, by call index mod 4
constexpr int RECBUF = 128;                     // panel records of one call staged in shared memory
constexpr int JMAX = PATCH_CHAIN_MAX_CALLS;

constexpr uint32_t INFO_SPARSE = 1u, INFO_SEG_START = 2u, INFO_SEG_END = 4u;

// Panel record (written by the plan kernel): x = tile index, y = half (bit 0)
// | sparse (bit 1) | sparse ordinal << 2.
__host__ __device__ __forceinline__ uint32_t rec_info(uint32_t h, uint32_t sparse, uint32_t ord) {
  return h | (sparse << 1) | (ord << 2);
}

struct Stage {
  alignas(1024) uint8_t a[A_BYTES];
  alignas(1024) uint8_t x[2][X_BYTES];
  alignas(128) uint8_t e[E_BYTES];
};

struct Shared {
  Stage st[NS];
  alignas(16) uint2 rec[2][RECBUF + 2];  // the X producer's panel records, by call parity
  uint64_t full[NS], empty[NS];
  uint64_t acc_full[NACC], acc_empty[NACC], drain[NISS], rec_full[2];
  uint64_t rec_empty[2];  // X producer 1 is done with the chunk in buffer b
  uint32_t info[NS];
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t SMEM_BYTES = sizeof(Shared) + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct Call {
  const patch_tile_desc* desc;
  const uint8_t* meta;
  uint16_t* Y;
  const uint2* rec;   // P panel records of this call (workspace)
  int64_t P;          // panels in the values blob
  int M, N, Tk, Tn;
  uint32_t ctr_base;  // this call's row counters: counters[ctr_base + 4 tn + q]
  int after;          // read X only after every earlier call of the launch has completed
  int64_t off;        // first panel of the call in the launch's panel sequence (global split)
};

struct Args {
  Call call[JMAX];
  int J;
  uint32_t* counters;  // fixed region: done[J], exit, then the calls' row counters (zero between launches)
  float* part;         // [PART_RING][G][2][128][16] fp32 partials
  uint64_t limit_ns;
  int32_t* status;
  int global;    // 1: no call waits for another; CTAs split the launch's whole panel sequence
  int64_t Ptot;  // panels of all calls
};

struct Maps {
  CUtensorMap x[JMAX];
  CUtensorMap w[JMAX];
};

__host__ __device__ __forceinline__ int64_t range_begin(int64_t c, int64_t P, int64_t G) { return c * P / G; }
__host__ __device__ __forceinline__ int64_t cta_of_panel(int64_t p, int64_t P, int64_t G) {
  return ((p + 1) * G - 1) / P;
}
// CTAs working on a call of P panels: all G, or P when the call has fewer
// panels than CTAs (so that every working CTA holds at least one panel and
// the CTAs covering a tile row are consecutive); the others idle in it.
__host__ __device__ __forceinline__ int64_t active_ctas(int64_t P, int64_t G) { return P < G ? P : G; }
// Panel range [p0, p1) of CTA c in a call of P panels (empty for an idle CTA).
__device__ __forceinline__ void cta_range(int64_t c, int64_t P, int64_t G, int64_t& p0, int64_t& p1) {
  const int64_t Ga = active_ctas(P, G);
  p0 = c < Ga ? range_begin(c, P, Ga) : P;
  p1 = c < Ga ? range_begin(c + 1, P, Ga) : P;
}
// Panel range [p0, p1) of CTA c in call j: its share of the call (per-call
// split), or, when no call waits for another, the part of call j inside the
// CTA's share of the whole launch's panel sequence (global split: a CTA then
// streams one contiguous run of panels across call boundaries, and only the
// rows at the two ends of its run are cut).  Empty ranges are [P, P).
__device__ __forceinline__ void call_range(const Args& a, int j, int64_t c, int64_t G, int64_t& p0, int64_t& p1) {
  const Call& cl = a.call[j];
  if (!a.global) {
    cta_range(c, cl.P, G, p0, p1);
    return;
  }
  int64_t g0, g1;
  cta_range(c, a.Ptot, G, g0, g1);
  const int64_t lo = g0 > cl.off ? g0 : cl.off, hi = g1 < cl.off + cl.P ? g1 : cl.off + cl.P;
  p0 = lo < hi ? lo - cl.off : cl.P;
  p1 = lo < hi ? hi - cl.off : cl.P;
}
__device__ __forceinline__ int64_t panel_of(const patch_tile_desc& d) {
  return int64_t(d.val_offset / PATCH_PANEL_BYTES);
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Order this thread's generic-proxy accesses to global memory with its
// async-proxy (TMA) accesses: Y written by plain stores in one CTA is read by
// TMA loads in another.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Limit of the exit-time waits for this CTA's copies in flight: the caller's
// limit, but never less than 20 ms, so that a short limit (which makes the
// other waits give up early) still lets every issued copy land before exit.
__device__ __forceinline__ uint64_t drain_limit(const Args& a) {
  return a.limit_ns > 20000000ull ? a.limit_ns : 20000000ull;
}

// Wait until calls 0..j have completed on every CTA (done[j] == G).  Bounded
// in time: on expiry the CTA's abort flag and PATCH_DEV_TIMEOUT are set.
__device__ bool wait_calls_done(const Args& a, Shared& s, int j, uint32_t G) {
  const uint32_t* done = a.counters + j;
  if (ld_acquire_gpu(done) >= G) return true;
  const uint64_t t0 = globaltimer_ns();
  volatile int* abort_flag = &s.abort_flag;
  for (uint32_t spin = 1;; ++spin) {
    if (ld_acquire_gpu(done) >= G) return true;
    if ((spin & 15u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > a.limit_ns) {
        *abort_flag = 1;
        set_status(a.status, PATCH_DEV_TIMEOUT);
        return false;
      }
    }
    __nanosleep(64);
  }
}

// ---------------------------------------------------------------- plan kernel

struct PlanArgs {
  const patch_tile_desc* desc[JMAX];
  uint2* rec[JMAX];
  int64_t tile_end[JMAX];  // prefix sums of the calls' tile counts
  int J;
};

// Panel records of every call: each tile writes its 1 (sparse) or 2 (dense)
// panels' records at the panel index its descriptor gives.
__global__ void __launch_bounds__(256) chain_plan_kernel(const __grid_constant__ PlanArgs pa) {
  const int64_t total = pa.tile_end[pa.J - 1];
  for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < total;
       g += int64_t(gridDim.x) * blockDim.x) {
    int j = 0;
    while (g >= pa.tile_end[j]) ++j;
    const int64_t t = g - (j ? pa.tile_end[j - 1] : 0);
    const patch_tile_desc d = pa.desc[j][t];
    const int64_t p = panel_of(d);
    const uint32_t sparse = d.kind ? 1u : 0u;
    const uint32_t ord = sparse ? d.sparse_ordinal : 0u;
    pa.rec[j][p] = make_uint2(uint32_t(t), rec_info(0, sparse, ord));
    if (!sparse) pa.rec[j][p + 1] = make_uint2(uint32_t(t), rec_info(1, 0, 0));
  }
}

// ---------------------------------------------------------------- roles

// W producer: the weight panels of every call, in order, by index only.
__device__ void producer_w(Shared& s, const Maps& maps, const Args& a) {
  const int64_t G = gridDim.x, c = blockIdx.x;
  uint32_t i = 0;
  bool ok = true;
  for (int j = 0; ok && j < a.J; ++j) {
    const Call& cl = a.call[j];
    int64_t p0, p1;
    call_range(a, j, c, G, p0, p1);
    for (int64_t p = p0; p < p1; ++p, ++i) {
      const uint32_t st = i % NS;
      if (!(ok = wait_bounded(&s.empty[st], ((i / NS) & 1) ^ 1, &s.abort_flag, a.limit_ns, a.status, false)))
        break;
      mbar_expect_tx(&s.full[st], A_BYTES);
      tma_load_2d(s.st[st].a, &maps.w[j], &s.full[st], 0, int(p * 128));
    }
  }
  // every copy issued must have landed before the CTA may exit
  for (uint32_t k = (i > NS ? i - NS : 0); k < i; ++k)
    wait_bounded(&s.full[k % NS], (k / NS) & 1, &s.abort_flag, drain_limit(a), a.status, true);
}

// X slice loads of one stage
__device__ __forceinline__ void load_x(Stage& g, uint64_t* full, const CUtensorMap* tmap_x, int kt, int h,
                                       bool sparse) {
  if (sparse) {
    tma_load_2d(g.x[0], tmap_x, full, kt * kTile, 0);
    tma_load_2d(g.x[1], tmap_x, full, kt * kTile + 64, 0);
  } else {
    tma_load_2d(g.x[0], tmap_x, full, kt * kTile + 64 * h, 0);
  }
}

// The X producer's panel records, staged in shared memory in chunks of at
// most RECBUF records (a run of one call's panels), one chunk ahead, in two
// buffers.  A chunk's bulk copy starts at the even record q0 <= its first
// panel and covers whole 16-byte units (a call's records are padded to an
// even count), so record p sits at p - q0 of its buffer.
struct ChunkIter {
  int j;          // call (a.J: past the end)
  int64_t p, p1;  // the chunk's first panel; end of the CTA's range in call j
};

__device__ __forceinline__ void chunk_first(const Args& a, ChunkIter& it) {
  const int64_t G = gridDim.x, c = blockIdx.x;
  for (it.j = 0; it.j < a.J; ++it.j) {
    int64_t p0;
    call_range(a, it.j, c, G, p0, it.p1);
    it.p = p0;
    if (p0 < it.p1) return;
  }
}

__device__ __forceinline__ void chunk_next(const Args& a, ChunkIter& it) {
  const int64_t G = gridDim.x, c = blockIdx.x;
  it.p += RECBUF;
  if (it.p < it.p1) return;
  for (++it.j; it.j < a.J; ++it.j) {
    int64_t p0;
    call_range(a, it.j, c, G, p0, it.p1);
    it.p = p0;
    if (p0 < it.p1) return;
  }
}

__device__ __forceinline__ void stage_chunk(Shared& s, const Args& a, const ChunkIter& it, uint32_t k) {
  const Call& cl = a.call[it.j];
  const int64_t e = it.p + RECBUF < it.p1 ? it.p + RECBUF : it.p1;
  const int64_t q0 = it.p & ~int64_t(1);
  const uint32_t bytes = uint32_t(((e - q0) * 8 + 15) & ~int64_t(15));  // <= (RECBUF + 2) * 8
  mbar_expect_tx(&s.rec_full[k & 1], bytes);
  bulk_load(s.rec[k & 1], cl.rec + q0, bytes, &s.rec_full[k & 1]);
}

// X producer `par` (0 or 1): for the CTA's panels i with i % 2 == par, the
// panel's record (tile, half, kind), the stage's info word, a sparse tile's
// metadata and the panel's X slices.  A call that reads the output of earlier
// calls loads its X slices only after they have completed on every CTA.
// Producer 0 stages the record chunks, producer 1 tells it (rec_empty) when it
// is done with a buffer, so the chunk two ahead may overwrite it.
__device__ void producer_x(Shared& s, const Maps& maps, const Args& a, int par) {
  const int64_t G = gridDim.x, c = blockIdx.x;
  uint32_t i = 0;
  bool ok = true;
  uint32_t staged = 0, waited = 0;  // record chunks copied / waited for; chunk n uses buffer n & 1
  ChunkIter cur;
  chunk_first(a, cur);
  if (par == 0 && cur.j < a.J) stage_chunk(s, a, cur, staged++);
  while (ok && cur.j < a.J) {
    // stage the chunk after this one into the other buffer, once producer 1
    // is done with the chunk before this one, which that buffer held
    ChunkIter nxt = cur;
    chunk_next(a, nxt);
    if (par == 0 && nxt.j < a.J) {
      if (staged >= 2 && !(ok = wait_bounded(&s.rec_empty[staged & 1], ((staged >> 1) - 1) & 1, &s.abort_flag,
                                             a.limit_ns, a.status, false)))
        break;
      stage_chunk(s, a, nxt, staged++);
    }
    if (!(ok = wait_bounded(&s.rec_full[waited & 1], (waited >> 1) & 1, &s.abort_flag, a.limit_ns, a.status, false)))
      break;
    const uint2* recs = s.rec[waited & 1];
    ++waited;
    const int j = cur.j;
    const Call& cl = a.call[j];
    int64_t p0, p1;  // the CTA's whole range in call j (segment boundaries); the chunk is [cb, ce)
    call_range(a, j, c, G, p0, p1);
    const int64_t cb = cur.p, ce = cur.p + RECBUF < cur.p1 ? cur.p + RECBUF : cur.p1;
    const int64_t q0 = cb & ~int64_t(1);
    const uint32_t xb = uint32_t(cl.M) * 128;  // an X slice holds M token rows
    bool dep_ok = !cl.after || j == 0 || cb > p0;  // waited for at the call's first chunk
    for (int64_t p = cb; p < ce; ++p, ++i) {
      if ((i & 1u) != uint32_t(par)) continue;  // the other producer's panel
      const uint32_t st = i % NS;
      if (!(ok = wait_bounded(&s.empty[st], ((i / NS) & 1) ^ 1, &s.abort_flag, a.limit_ns, a.status, false)))
        break;
      const uint2 r = recs[p - q0];
      const int t = int(r.x), kt = t % cl.Tk, h = int(r.y & 1u);
      const bool sparse = (r.y >> 1) & 1u;
      uint32_t info = sparse ? INFO_SPARSE : 0u;
      if (p == p0 || (kt == 0 && h == 0)) info |= INFO_SEG_START;
      if (p + 1 == p1 || (kt == cl.Tk - 1 && (sparse || h == 1))) info |= INFO_SEG_END;
      s.info[st] = info;  // published to the MMA thread by this thread's arrival
      if (!dep_ok) {  // X is earlier calls' output: wait until they are complete everywhere
        if (!wait_calls_done(a, s, j - 1, uint32_t(G))) {
          // arrive without bytes, so the stage completes once its weight panel
          // has landed and the exit-time drain does not wait for it in vain
          mbar_arrive(&s.full[st]);
          ok = false;
          ++i;
          break;
        }
        fence_proxy_async_global();
        dep_ok = true;
      }
      mbar_expect_tx(&s.full[st], sparse ? 2 * xb + E_BYTES : xb);
      if (sparse) bulk_load(s.st[st].e, cl.meta + uint64_t(r.y >> 2) * E_BYTES, E_BYTES, &s.full[st]);
      load_x(s.st[st], &s.full[st], &maps.x[j], kt, h, sparse);
    }
    if (par == 1) mbar_arrive(&s.rec_empty[(waited - 1) & 1]);  // done with this chunk's buffer
    cur = nxt;
  }
  // every copy issued must have landed before the CTA may exit
  for (uint32_t k = waited; k < staged; ++k)
    wait_bounded(&s.rec_full[k & 1], (k >> 1) & 1, &s.abort_flag, drain_limit(a), a.status, true);
  for (uint32_t k = (i > NS ? i - NS : 0); k < i; ++k)
    if ((k & 1u) == uint32_t(par))
      wait_bounded(&s.full[k % NS], (k / NS) & 1, &s.abort_flag, drain_limit(a), a.status, true);
}

// MMA issuer u (one thread each, u = 0, 1): every panel's four MMAs are split
// between the two threads by K (u = 0 the first half, u = 1 the second), each
// into its own accumulator, so that issuing them -- a long-latency instruction
// each -- takes half as long per panel; the epilogue adds the two halves.
// Both wait for every stage and both commit to its release (empty: 2 arrivals).
__device__ void mma_issuer(Shared& s, uint32_t tmem, const Args& a, int u) {
  const int64_t G = gridDim.x, c = blockIdx.x;
  uint32_t i = 0, seg = 0, acc = tmem, accumulate = 0;
  bool ok = true;
  for (int j = 0; ok && j < a.J; ++j) {
    const Call& cl = a.call[j];
    int64_t p0, p1;
    call_range(a, j, c, G, p0, p1);
    for (int64_t p = p0; p < p1; ++p, ++i) {
      const uint32_t st = i % NS;
      if (!(ok = wait_bounded(&s.full[st], (i / NS) & 1, &s.abort_flag, a.limit_ns, a.status, false))) break;
      const uint32_t info = *reinterpret_cast<volatile uint32_t*>(&s.info[st]);
      if (info & INFO_SEG_START) {  // a new tile row starts a new accumulation segment
        const uint32_t buf = seg % NACC;
        if (!(ok = wait_bounded(&s.acc_empty[buf], ((seg / NACC) & 1) ^ 1, &s.abort_flag, a.limit_ns, a.status,
                                false)))
          break;
        acc = tmem + (NISS * buf + u) * BT;
        accumulate = 0;
      }
      tc_fence_after();
      Stage& g = s.st[st];
      const uint64_t a0 = sw128_desc(smem_u32(g.a));
      if (info & INFO_SPARSE) {
        // each issuer copies the metadata into its own columns: no ordering across threads needed
        const uint32_t e_tmem = tmem + META_COL0 + 4 * (NS * u + st);
        tmem_cp_128x128b(e_tmem, meta_desc(smem_u32(g.e)));
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // 32-k blocks kb = 2u, 2u + 1: 16 kept values = 32 B of A; 32 k = 64 B of X
          const int kb = 2 * u + h;
          const uint64_t b = sw128_desc(smem_u32(g.x[u])) + (h * 64 >> 4);
          mma_sparse(acc, a0 + (kb * 32 >> 4), b, e_tmem + (kb & 2), IDESC_SPARSE | (kb & 1), accumulate);
          accumulate = 1;
        }
      } else {
        const uint64_t b0 = sw128_desc(smem_u32(g.x[0]));
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // K = 16 per MMA = 32 B along the swizzled row
          const int k = 2 * u + h;
          mma_dense(acc, a0 + (k * 32 >> 4), b0 + (k * 32 >> 4), IDESC_DENSE, accumulate);
          accumulate = 1;
        }
      }
      tc_commit(&s.empty[st]);
      if (info & INFO_SEG_END) {
        tc_commit(&s.acc_full[seg % NACC]);
        ++seg;
      }
    }
  }
  tc_commit(&s.drain[u]);
  wait_bounded(&s.drain[u], 0, &s.abort_flag, a.limit_ns, a.status, true);
}

// Sum of the partial rows (row r of the tile row) of covering CTAs c_lo..c_hi
// in one partial-sum buffer, in CTA order (deterministic).
template <int B, int NV>
__device__ __forceinline__ void sum_partials(const float* ring, int r, int64_t c_lo, int64_t c_hi, int slot_lo, int nv,
                                             float (&sum)[BT]) {
#pragma unroll
  for (int m = 0; m < BT; ++m) sum[m] = 0.0f;
  for (int64_t c0 = c_lo; c0 <= c_hi; c0 += B) {
    float4 part[B][NV];
#pragma unroll
    for (int k2 = 0; k2 < B; ++k2) {
      const int64_t cc = c0 + k2;
      const float4* src = reinterpret_cast<const float4*>(ring + cc * WS_FLOATS_PER_CTA +
                                                          (cc == c_lo ? slot_lo : 0) * BT * BM + r * BT);
#pragma unroll
      for (int k = 0; k < NV; ++k)
        part[k2][k] = (cc <= c_hi && k < nv) ? __ldcg(src + k) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
#pragma unroll
    for (int k2 = 0; k2 < B; ++k2)
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        sum[4 * k] += part[k2][k].x;
        sum[4 * k + 1] += part[k2][k].y;
        sum[4 * k + 2] += part[k2][k].z;
        sum[4 * k + 3] += part[k2][k].w;
      }
  }
}

// Epilogue warps (one TMEM lane quarter each): per call, the CTA's tile rows
// in order; then, once all four warps are done with the call, one arrival on
// the call's completion counter.
__device__ void epilogue(Shared& s, uint32_t tmem, const Args& a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;
  const int r = 32 * q + lane;  // tile row (TMEM lane) of this thread
  const int64_t G = gridDim.x, c = blockIdx.x;
  const bool leader = warp == 2 && lane == 0;
  uint32_t seg = 0;
  bool ok = true, seen = false;
  for (int j = 0; j < a.J; ++j) {
    const Call& cl = a.call[j];
    int64_t p0, p1;
    call_range(a, j, c, G, p0, p1);
    const bool first_call = p1 > p0 && !seen;  // the call holding the CTA's first segment
    seen = seen || p1 > p0;
    if (ok && p1 > p0) {
      // the CTA's first and last panel records and the boundaries of the rows they lie in
      const uint2 r0 = __ldcg(cl.rec + p0), r1 = __ldcg(cl.rec + p1 - 1);
      const int t0 = int(r0.x), t1 = int(r1.x);
      const int tn_first = t0 / cl.Tk, tn_last = t1 / cl.Tk;
      const bool first_row_whole = t0 % cl.Tk == 0 && (r0.y & 1u) == 0;
      const bool last_row_whole = t1 % cl.Tk == cl.Tk - 1 && (((r1.y >> 1) & 1u) || (r1.y & 1u));
      auto row_start = [&](int tn) -> int64_t {
        return tn < cl.Tn ? panel_of(cl.desc[int64_t(tn) * cl.Tk]) : cl.P;
      };
      int64_t row_lo[2] = {0, 0}, row_hi[2] = {0, 0};
      if (!first_row_whole || tn_first == tn_last) {
        row_lo[0] = row_start(tn_first);
        row_lo[1] = row_start(tn_first + 1);
      }
      if (!last_row_whole) {
        row_hi[0] = row_start(tn_last);
        row_hi[1] = row_start(tn_last + 1);
      }
      // per-call split: partial buffer j % 4, which last served call j - 4; global
      // split: one buffer (a CTA cuts only its first and last segment of the launch)
      float* ring = a.part + (a.global ? 0 : int64_t(j % PART_RING) * G * WS_FLOATS_PER_CTA);
      bool guard_done = a.global || j < PART_RING;
      for (int tn = tn_first; tn <= tn_last; ++tn, ++seg) {
        const uint32_t buf = seg % NACC;
        // a warp-uniform decision: the tensor-memory loads below are warp-collective
        ok = __all_sync(0xFFFFFFFFu,
                        wait_bounded(&s.acc_full[buf], (seg / NACC) & 1, &s.abort_flag, a.limit_ns, a.status, false));
        if (!ok) break;
        tc_fence_after();
        uint32_t v[16], w[16];
        tmem_ld_16cols(tmem + (uint32_t(32 * q) << 16) + uint32_t(NISS * buf * BT), v);
        tmem_ld_16cols(tmem + (uint32_t(32 * q) << 16) + uint32_t((NISS * buf + 1) * BT), w);
#pragma unroll
        for (int m = 0; m < BT; ++m) v[m] = __float_as_uint(__uint_as_float(v[m]) + __uint_as_float(w[m]));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.acc_empty[buf]);
        const int64_t n = int64_t(tn) * BM + r;
        if ((tn > tn_first || first_row_whole) && (tn < tn_last || last_row_whole)) {  // the whole row is ours
#pragma unroll
          for (int m = 0; m < BT; ++m)
            if (m < cl.M) cl.Y[int64_t(m) * cl.N + n] = f32_to_bf16_rne(__uint_as_float(v[m]));
          continue;
        }
        if (!guard_done) {  // every CTA has finished call j - 4, whose last arrivers read this buffer
          if (!(ok = wait_calls_done(a, s, j - PART_RING, uint32_t(G)))) break;
          guard_done = true;
        }
        const bool first_seg = tn == tn_first && (!a.global || first_call);
        float4* mine = reinterpret_cast<float4*>(ring + c * WS_FLOATS_PER_CTA + (first_seg ? 0 : BT * BM) + r * BT);
#pragma unroll
        for (int k = 0; k < BT / 4; ++k)
          if (4 * k < cl.M)
            mine[k] = make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                  __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
        // the row's panels in the split's index space (the call's, or the launch's)
        const int64_t base = a.global ? cl.off : 0, Pspace = a.global ? a.Ptot : cl.P;
        const int64_t rb = base + (tn == tn_first ? row_lo[0] : row_hi[0]);
        const int64_t re = base + (tn == tn_first ? row_lo[1] : row_hi[1]);
        const int64_t Ga = active_ctas(Pspace, G);
        const int64_t c_lo = cta_of_panel(rb, Pspace, Ga), c_hi = cta_of_panel(re - 1, Pspace, Ga);
        uint32_t* counter = a.counters + cl.ctr_base + 4 * tn + q;
        __syncwarp();
        uint32_t old = 0;
        if (lane == 0) old = atom_add_acq_rel_gpu(counter, 1u);
        old = __shfl_sync(0xFFFFFFFFu, old, 0);
        if (old != uint32_t(c_hi - c_lo)) continue;
        __syncwarp();
        const int slot_lo = range_begin(c_lo, Pspace, Ga) < rb ? 1 : 0;
        const int nv = (cl.M + 3) / 4;
        float sum[BT];
        if (nv <= 2)
          sum_partials<8, 2>(ring, r, c_lo, c_hi, slot_lo, nv, sum);
        else
          sum_partials<4, BT / 4>(ring, r, c_lo, c_hi, slot_lo, nv, sum);
#pragma unroll
        for (int m = 0; m < BT; ++m)
          if (m < cl.M) cl.Y[int64_t(m) * cl.N + n] = f32_to_bf16_rne(sum[m]);
        if (lane == 0) *counter = 0;  // ready for the next launch
      }
    }
    // all four warps' stores of call j are done (each thread orders its own Y
    // stores before the TMA reads of later calls): one release arrival on done[j]
    fence_proxy_async_global();
    named_bar_sync(1, 128);
    if (leader) red_release_gpu_add(a.counters + j, 1u);
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    chain_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Args a) {
  extern __shared__ uint8_t smem_raw[];
  Shared& s = *reinterpret_cast<Shared*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int k = 0; k < NS; ++k) {
      mbar_init(&s.full[k], 2);      // one arrival per producer thread
      mbar_init(&s.empty[k], NISS);  // one commit per MMA issuer
    }
    for (int k = 0; k < NACC; ++k) {
      mbar_init(&s.acc_full[k], NISS);
      mbar_init(&s.acc_empty[k], 4);
    }
    mbar_init(&s.drain[0], 1);
    mbar_init(&s.drain[1], 1);
    mbar_init(&s.rec_full[0], 1);
    mbar_init(&s.rec_full[1], 1);
    mbar_init(&s.rec_empty[0], 1);
    mbar_init(&s.rec_empty[1], 1);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < a.J) {
    prefetch_tensormap(&maps.w[threadIdx.x]);
    prefetch_tensormap(&maps.x[threadIdx.x]);
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    if (lane == 0) producer_w(s, maps, a);
    __syncwarp();
  } else if (warp == 1 || warp == 7) {
    if (lane == 0) mma_issuer(s, tmem, a, warp == 1 ? 0 : 1);
    __syncwarp();
  } else if (warp == 6 || warp == 8) {
    if (lane == 0) producer_x(s, maps, a, warp == 6 ? 0 : 1);
    __syncwarp();
  } else {
    epilogue(s, tmem, a);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  // the last CTA to leave clears the completion counters for the next launch
  // (every CTA has read them for the last time before it arrives here)
  if (threadIdx.x == 0) {
    uint32_t* exit_ctr = a.counters + a.J;
    const uint32_t old = atom_add_acq_rel_gpu(exit_ctr, 1u);
    if (old == gridDim.x - 1) {
      for (int j = 0; j < a.J; ++j) a.counters[j] = 0;
      *exit_ctr = 0;
    }
  }
}

}  // namespace chain

// ---------------------------------------------------------------- host side

namespace {

struct ChainGeometry {
  int64_t P, Tn, Tk;
};

ChainGeometry geometry(const patch_weight& W) {
  ChainGeometry g;
  g.Tn = W.N / kTile;
  g.Tk = W.K / kTile;
  const int64_t T = g.Tn * g.Tk;
  g.P = 2 * (T - W.n_sparse) + W.n_sparse;
  return g;
}

// Counter words a launch of calls [j0, j1) needs in the fixed region: one
// completion counter per call, one exit counter, four per tile row per call.
int64_t counter_words(const patch_chain_call* calls, int64_t j0, int64_t j1) {
  int64_t w = (j1 - j0) + 1;
  for (int64_t j = j0; j < j1; ++j) w += 4 * (calls[j].W.N / kTile);
  return w;
}

}  // namespace

int64_t chain_launch_end(const patch_chain_call* calls, int64_t j0, int64_t n) {
  int64_t j1 = j0 + 1;  // a single call always fits (N <= 524288 is checked)
  while (j1 < n && j1 - j0 < chain::JMAX &&
         counter_words(calls, j0, j1 + 1) * 4 <= int64_t(kDecodeCounterBytes))
    ++j1;
  return j1;
}

size_t chain_workspace_bytes(const patch_chain_call* calls, int64_t n, int num_sms) {
  size_t rec_max = 0;
  for (int64_t j0 = 0; j0 < n;) {
    const int64_t j1 = chain_launch_end(calls, j0, n);
    size_t rec = 0;
    for (int64_t j = j0; j < j1; ++j) rec += size_t((geometry(calls[j].W).P + 1) & ~int64_t(1)) * 8;
    if (rec > rec_max) rec_max = rec;
    j0 = j1;
  }
  const size_t part = size_t(chain::PART_RING) * size_t(num_sms) * chain::WS_FLOATS_PER_CTA * sizeof(float);
  return kDecodeCounterBytes + part + rec_max;
}

cudaError_t launch_chain(const patch_chain_call* calls, int64_t j0, int64_t j1, void* workspace, int32_t* status,
                         int num_sms, uint64_t limit_ns, cudaStream_t stream) {
  using namespace chain;
  const int J = int(j1 - j0);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t part_bytes = size_t(PART_RING) * size_t(num_sms) * WS_FLOATS_PER_CTA * sizeof(float);
  uint2* rec = reinterpret_cast<uint2*>(ws + kDecodeCounterBytes + part_bytes);

  Maps maps;  // kernel parameters: copied at launch
  Args args;
  PlanArgs pa;
  uint32_t ctr = uint32_t(J + 1);
  int64_t rec_off_panels = 0;  // the calls' panels, one after another
  bool any_after = false;
  int64_t tiles = 0, rec_off = 0;
  for (int j = 0; j < J; ++j) {
    const patch_chain_call& cl = calls[j0 + j];
    const ChainGeometry g = geometry(cl.W);
    if (!make_map_2d_bf16(&maps.x[j], cl.X, uint64_t(cl.W.K), uint64_t(cl.M), uint64_t(cl.W.K) * 2, 64,
                          uint32_t(cl.M)))
      return cudaErrorUnknown;
    if (!make_map_2d_bf16(&maps.w[j], cl.W.values, 64, uint64_t(g.P) * 128, 128, 64, 128)) return cudaErrorUnknown;
    Call& c = args.call[j];
    c.desc = cl.W.desc;
    c.meta = static_cast<const uint8_t*>(cl.W.meta);
    c.Y = cl.Y;
    c.rec = rec + rec_off;
    c.P = g.P;
    c.M = int(cl.M);
    c.N = int(cl.W.N);
    c.Tk = int(g.Tk);
    c.Tn = int(g.Tn);
    c.ctr_base = ctr;
    c.after = cl.after_previous && j > 0 ? 1 : 0;  // the launch's first call never waits
    c.off = rec_off_panels;
    rec_off_panels += g.P;
    any_after = any_after || c.after;
    ctr += uint32_t(4 * g.Tn);
    pa.desc[j] = cl.W.desc;
    pa.rec[j] = rec + rec_off;
    tiles += g.Tn * g.Tk;
    pa.tile_end[j] = tiles;
    rec_off += (g.P + 1) & ~int64_t(1);  // keeps every call's records 16-byte aligned
  }
  args.J = J;
  args.counters = static_cast<uint32_t*>(workspace);
  args.part = reinterpret_cast<float*>(ws + kDecodeCounterBytes);
  args.limit_ns = limit_ns;
  args.status = status;
  // when no call waits for another, the CTAs split the whole panel sequence
  args.global = any_after ? 0 : 1;
  args.Ptot = rec_off_panels;
  pa.J = J;

  int plan_blocks = int((tiles + 255) / 256);
  if (plan_blocks > 4 * num_sms) plan_blocks = 4 * num_sms;
  chain_plan_kernel<<<plan_blocks, 256, 0, stream>>>(pa);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  e = cudaFuncSetAttribute(chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chain_kernel, THREADS, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  // every CTA must be resident at once: they wait on each other's counters
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(num_sms));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, chain_kernel, maps, args);
}

}  // namespace patch
