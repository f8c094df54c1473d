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
// tile order.  CTA c of G (one per SM) takes panels [c*P/G, (c+1)*P/G), so
// every CTA streams the same number of panels whatever the sparsity pattern.
// Inside its range a CTA accumulates each tile row's panels into a TMEM
// accumulator (M = 128 rows of W, N = 16 tokens, zero-padded by TMA).  A
// tile row entirely inside one CTA's range is rounded to bf16 and stored
// directly; a row cut by a range boundary leaves fp32 partial sums in the
// workspace ([G][2][16][128]: each CTA has at most a first and a last cut
// row), which decode_fixup_kernel adds in CTA order (deterministic).
//
// Roles per CTA (6 warps): warp 0 TMA producer (A ring of 10 weight panels,
// B ring of 2 KiB X panels, metadata ring), warp 1 MMA issuer and TMEM owner
// (dense panel: 4 x kind::f16 K = 16; sparse tile: tcgen05.cp of its metadata,
// then 4 x kind::f16 .sp K = 32), warps 2-5 epilogue (tcgen05.ld of 128 x 16
// fp32).  Waits are bounded in time exactly as in the prefill kernel.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace patch {
namespace decode_tc {

using namespace tc;

constexpr int BM = 128;
constexpr int BT = 16;                  // MMA N (tokens)
constexpr int NA = 10;                  // weight panels in flight per SM
constexpr int NB = 12;
constexpr int NE = 4;
constexpr int NACC = 2;                 // accumulator buffers (epilogue overlaps the next row)
constexpr int A_BYTES = PATCH_PANEL_BYTES;
constexpr int B_BYTES = BT * 64 * 2;
constexpr int E_BYTES = PATCH_META_TILE_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 64;
constexpr uint32_t META_COL0 = NACC * BT;
constexpr uint32_t IDESC_DENSE = idesc_bf16(BM, BT, false);
constexpr uint32_t IDESC_SPARSE = idesc_bf16(BM, BT, true);
constexpr int WS_FLOATS_PER_CTA = 2 * BT * BM;  // [2 slots][16 tokens][128 rows]
constexpr int DCAP = 1024;               // descriptors of the CTA's tiles staged in shared memory

struct Shared {
  alignas(1024) uint8_t a[NA][A_BYTES];
  alignas(1024) uint8_t b[NB][B_BYTES];
  alignas(128) uint8_t e[NE][E_BYTES];
  uint64_t a_full[NA], a_empty[NA], b_full[NB], b_empty[NB], e_full[NE], e_empty[NE];
  uint64_t acc_full[NACC], acc_empty[NACC], drain;
  alignas(16) patch_tile_desc dcache[DCAP];  // tiles t_first .. t_last (when they fit)
  uint32_t tmem_base;
  int abort_flag;
  int t_first, t_last;  // tiles holding the CTA's first and last panel
  int cached;           // dcache holds the CTA's tiles
};
constexpr size_t SMEM_BYTES = sizeof(Shared) + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct Args {
  const patch_tile_desc* desc;
  const uint8_t* meta;
  uint16_t* Y;
  float* ws;
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

__device__ __forceinline__ int64_t panel_of(const patch_tile_desc& d) {
  return int64_t(d.val_offset / PATCH_PANEL_BYTES);
}

// Tiles holding panels pa and pb: the last t with panel_of(desc[t]) <= p.
// Called by every thread of the block: each round probes blockDim.x tiles at
// once and narrows the span by that factor, so a search costs a few global
// latencies instead of log2(T) dependent ones.
__device__ void find_tiles(const patch_tile_desc* desc, int T, int64_t pa, int64_t pb, int& ta, int& tb) {
  const int n = blockDim.x, i = threadIdx.x;
  int lo_a = 0, lo_b = 0, span = T;
  while (span > 1) {
    const int step = (span + n - 1) / n;
    const int ia = lo_a + i * step, ib = lo_b + i * step;
    const bool in = i * step < span;
    const int ca = __syncthreads_count(in && ia < T && panel_of(desc[ia]) <= pa);
    const int cb = __syncthreads_count(in && ib < T && panel_of(desc[ib]) <= pb);
    lo_a += (ca - 1) * step;
    lo_b += (cb - 1) * step;
    span = step;
  }
  ta = lo_a;
  tb = lo_b;
}

// Descriptor of tile t (staged in shared memory when the CTA's tiles fit).
__device__ __forceinline__ patch_tile_desc tile_desc(const Shared& s, const Args& a, int t) {
  return s.cached ? s.dcache[t - s.t_first] : a.desc[t];
}

__device__ __forceinline__ void advance(const patch_tile_desc& d, int& t, int& h) {
  if (d.kind || h == 1) {
    ++t;
    h = 0;
  } else {
    h = 1;
  }
}

__device__ void producer(Shared& s, const CUtensorMap* tmap_x, const CUtensorMap* tmap_w, const Args& a,
                         int64_t p0, int64_t p1) {
  uint32_t a_i = 0, b_i = 0, e_i = 0;
  int t = s.t_first;
  int h = p0 < p1 ? int(p0 - panel_of(tile_desc(s, a, t))) : 0;
  bool ok = true;
  for (int64_t p = p0; ok && p < p1; ++p) {
    const patch_tile_desc d = tile_desc(s, a, t);
    const int kt = t % a.Tk;
    if (d.kind) {
      const uint32_t es = e_i % NE;
      if (!(ok = wait_bounded(&s.e_empty[es], ((e_i / NE) & 1) ^ 1, &s.abort_flag, a.limit_ns, a.status, false)))
        break;
      mbar_expect_tx(&s.e_full[es], E_BYTES);
      bulk_load(s.e[es], a.meta + uint64_t(d.sparse_ordinal) * E_BYTES, E_BYTES, &s.e_full[es]);
      ++e_i;
    }
    const uint32_t as = a_i % NA;
    if (!(ok = wait_bounded(&s.a_empty[as], ((a_i / NA) & 1) ^ 1, &s.abort_flag, a.limit_ns, a.status, false)))
      break;
    mbar_expect_tx(&s.a_full[as], A_BYTES);
    tma_load_2d(s.a[as], tmap_w, &s.a_full[as], 0, int(p * 128));
    ++a_i;
    const int nb = d.kind ? 2 : 1;
    for (int j = 0; j < nb; ++j) {
      const uint32_t bs = b_i % NB;
      if (!(ok = wait_bounded(&s.b_empty[bs], ((b_i / NB) & 1) ^ 1, &s.abort_flag, a.limit_ns, a.status, false)))
        break;
      mbar_expect_tx(&s.b_full[bs], B_BYTES);
      tma_load_2d(s.b[bs], tmap_x, &s.b_full[bs], kt * kTile + 64 * (d.kind ? j : h), 0);
      ++b_i;
    }
    advance(d, t, h);
  }
  for (uint32_t i = (a_i > NA ? a_i - NA : 0); i < a_i; ++i)
    wait_bounded(&s.a_full[i % NA], (i / NA) & 1, &s.abort_flag, a.limit_ns, a.status, true);
  for (uint32_t i = (b_i > NB ? b_i - NB : 0); i < b_i; ++i)
    wait_bounded(&s.b_full[i % NB], (i / NB) & 1, &s.abort_flag, a.limit_ns, a.status, true);
  for (uint32_t i = (e_i > NE ? e_i - NE : 0); i < e_i; ++i)
    wait_bounded(&s.e_full[i % NE], (i / NE) & 1, &s.abort_flag, a.limit_ns, a.status, true);
}

__device__ void mma_issuer(Shared& s, uint32_t tmem, const Args& a, int64_t p0, int64_t p1) {
  uint32_t a_i = 0, b_i = 0, e_i = 0;
  int t = s.t_first;
  int h = p0 < p1 ? int(p0 - panel_of(tile_desc(s, a, t))) : 0;
  int seg = -1, cur_tn = -1;
  uint32_t acc = tmem, accumulate = 0;
  bool ok = true;
  for (int64_t p = p0; ok && p < p1; ++p) {
    const patch_tile_desc d = tile_desc(s, a, t);
    const int tn = t / a.Tk;
    if (tn != cur_tn) {  // a new tile row starts a new accumulation segment
      ++seg;
      cur_tn = tn;
      const int buf = seg % NACC;
      if (!(ok = wait_bounded(&s.acc_empty[buf], ((seg / NACC) & 1) ^ 1, &s.abort_flag, a.limit_ns, a.status,
                              false)))
        break;
      tc_fence_after();
      acc = tmem + uint32_t(buf * BT);
      accumulate = 0;
    }
    const uint32_t as = a_i % NA;
    if (d.kind) {
      const uint32_t es = e_i % NE;
      if (!(ok = wait_bounded(&s.e_full[es], (e_i / NE) & 1, &s.abort_flag, a.limit_ns, a.status, false))) break;
      if (!(ok = wait_bounded(&s.a_full[as], (a_i / NA) & 1, &s.abort_flag, a.limit_ns, a.status, false))) break;
      tc_fence_after();
      const uint32_t e_tmem = tmem + META_COL0 + 4 * es;
      tmem_cp_128x128b(e_tmem, meta_desc(smem_u32(s.e[es])));
      const uint64_t a0 = sw128_desc(smem_u32(s.a[as]));
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t bs = b_i % NB;
        if (!(ok = wait_bounded(&s.b_full[bs], (b_i / NB) & 1, &s.abort_flag, a.limit_ns, a.status, false))) break;
        tc_fence_after();
        const uint64_t b0 = sw128_desc(smem_u32(s.b[bs]));
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t kb = 2 * hh + j;
          mma_sparse(acc, a0 + (kb * 32 >> 4), b0 + (j * 64 >> 4), e_tmem + (kb & 2u), IDESC_SPARSE | (kb & 1u),
                     accumulate);
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
      const uint32_t bs = b_i % NB;
      if (!(ok = wait_bounded(&s.a_full[as], (a_i / NA) & 1, &s.abort_flag, a.limit_ns, a.status, false))) break;
      if (!(ok = wait_bounded(&s.b_full[bs], (b_i / NB) & 1, &s.abort_flag, a.limit_ns, a.status, false))) break;
      tc_fence_after();
      const uint64_t a0 = sw128_desc(smem_u32(s.a[as]));
      const uint64_t b0 = sw128_desc(smem_u32(s.b[bs]));
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        mma_dense(acc, a0 + (j * 32 >> 4), b0 + (j * 32 >> 4), IDESC_DENSE, accumulate);
        accumulate = 1;
      }
      tc_commit(&s.a_empty[as]);
      ++a_i;
      tc_commit(&s.b_empty[bs]);
      ++b_i;
    }
    advance(d, t, h);
    // the segment ends with the CTA's range or with the tile row
    if (p + 1 == p1 || t / a.Tk != cur_tn) tc_commit(&s.acc_full[seg % NACC]);
  }
  tc_commit(&s.drain);
  wait_bounded(&s.drain, 0, &s.abort_flag, a.limit_ns, a.status, true);
}

__device__ void epilogue(Shared& s, uint32_t tmem, const Args& a, int64_t p0, int64_t p1) {
  if (p0 >= p1) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;
  const int tn_first = s.t_first / a.Tk, tn_last = s.t_last / a.Tk;
  float* ws_cta = a.ws + int64_t(blockIdx.x) * WS_FLOATS_PER_CTA;
  for (int tn = tn_first; tn <= tn_last; ++tn) {
    const int seg = tn - tn_first, buf = seg % NACC;
    if (!wait_bounded(&s.acc_full[buf], (seg / NACC) & 1, &s.abort_flag, a.limit_ns, a.status, false)) break;
    tc_fence_after();
    uint32_t v[16];
    tmem_ld_16cols(tmem + (uint32_t(32 * q) << 16) + uint32_t(buf * BT), v);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.acc_empty[buf]);
    const int r = 32 * q + lane;
    // does this CTA hold the row's first and last panel?
    const patch_tile_desc df = tile_desc(s, a, s.t_first), dl = tile_desc(s, a, s.t_last);
    const bool starts = tn > tn_first || (s.t_first % a.Tk == 0 && p0 == panel_of(df));
    const bool ends = tn < tn_last || (s.t_last % a.Tk == a.Tk - 1 && p1 == panel_of(dl) + (dl.kind ? 1 : 2));
    if (starts && ends) {  // the whole row is ours
      const int64_t n = int64_t(tn) * BM + r;
#pragma unroll
      for (int m = 0; m < BT; ++m)
        if (m < a.M) a.Y[int64_t(m) * a.N + n] = f32_to_bf16_rne(__uint_as_float(v[m]));
    } else {
      float* slot = ws_cta + (tn == tn_first ? 0 : BT * BM);
#pragma unroll
      for (int m = 0; m < BT; ++m)
        if (m < a.M) slot[m * BM + r] = __uint_as_float(v[m]);
    }
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const Args a) {
  extern __shared__ uint8_t smem_raw[];
  Shared& s = *reinterpret_cast<Shared*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t p0 = range_begin(blockIdx.x, a.P, G), p1 = range_begin(blockIdx.x + 1, a.P, G);

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
    s.abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmap_x);
    prefetch_tensormap(&tmap_w);
  }
  // locate the CTA's first and last tile, then stage their descriptors
  if (p0 < p1) {
    int ta, tb;
    find_tiles(a.desc, a.Tn * a.Tk, p0, p1 - 1, ta, tb);
    const int count = tb - ta + 1;
    if (threadIdx.x == 0) {
      s.t_first = ta;
      s.t_last = tb;
      s.cached = count <= DCAP;
    }
    if (count <= DCAP)
      for (int i = threadIdx.x; i < count; i += blockDim.x) s.dcache[i] = a.desc[ta + i];
  } else if (threadIdx.x == 0) {
    s.t_first = s.t_last = 0;
    s.cached = 0;
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    if (lane == 0) producer(s, &tmap_x, &tmap_w, a, p0, p1);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_issuer(s, tmem, a, p0, p1);
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

// Rows cut by range boundaries: Y = bf16(sum over the covering CTAs, in CTA order).
__global__ void __launch_bounds__(256) decode_fixup_kernel(const patch_tile_desc* __restrict__ desc,
                                                           const float* __restrict__ ws, uint16_t* __restrict__ Y,
                                                           int M, int N, int Tk, int Tn, int64_t P, int64_t G) {
  const int tn = blockIdx.x;
  const int64_t rb = panel_of(desc[int64_t(tn) * Tk]);
  const int64_t re = tn + 1 < Tn ? panel_of(desc[int64_t(tn + 1) * Tk]) : P;
  const int64_t c_lo = cta_of_panel(rb, P, G), c_hi = cta_of_panel(re - 1, P, G);
  if (c_lo == c_hi) return;  // written directly by its CTA
  for (int i = threadIdx.x; i < M * BM; i += blockDim.x) {
    const int m = i / BM, r = i - m * BM;
    float sum = 0.0f;
    for (int64_t c = c_lo; c <= c_hi; ++c) {
      const int slot = range_begin(c, P, G) >= rb ? 0 : 1;  // this row is c's first row, or its last
      sum += ws[c * WS_FLOATS_PER_CTA + slot * BT * BM + m * BM + r];
    }
    Y[int64_t(m) * N + int64_t(tn) * BM + r] = f32_to_bf16_rne(sum);
  }
}

}  // namespace decode_tc

size_t decode_tc_workspace_bytes(int64_t M, const patch_weight& W, int num_sms) {
  (void)M;
  const int64_t Tn = W.N / kTile, Tk = W.K / kTile, T = Tn * Tk;
  const int64_t P = 2 * (T - W.n_sparse) + W.n_sparse;
  const int64_t G = P < num_sms ? P : num_sms;
  return size_t(G) * decode_tc::WS_FLOATS_PER_CTA * sizeof(float);
}

cudaError_t launch_decode_tc(const uint16_t* X, int64_t M, const patch_weight& W, uint16_t* Y, void* workspace,
                             int32_t* status, int num_sms, uint64_t limit_ns, cudaStream_t stream) {
  using namespace decode_tc;
  const int64_t Tn = W.N / kTile, Tk = W.K / kTile, T = Tn * Tk;
  const int64_t P = 2 * (T - W.n_sparse) + W.n_sparse;
  const int64_t G = P < num_sms ? P : num_sms;
  CUtensorMap tmap_x, tmap_w;
  if (!make_map_2d_bf16(&tmap_x, X, uint64_t(W.K), uint64_t(M), uint64_t(W.K) * 2, 64, BT)) return cudaErrorUnknown;
  if (!make_map_2d_bf16(&tmap_w, W.values, 64, uint64_t(P) * 128, 128, 64, 128)) return cudaErrorUnknown;
  Args a;
  a.desc = W.desc;
  a.meta = static_cast<const uint8_t*>(W.meta);
  a.Y = Y;
  a.ws = static_cast<float*>(workspace);
  a.M = int(M);
  a.N = int(W.N);
  a.Tk = int(Tk);
  a.Tn = int(Tn);
  a.P = P;
  a.limit_ns = limit_ns;
  a.status = status;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  decode_tc_kernel<<<int(G), THREADS, SMEM_BYTES, stream>>>(tmap_x, tmap_w, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_fixup_kernel<<<int(Tn), 256, 0, stream>>>(W.desc, a.ws, Y, int(M), int(W.N), int(Tk), int(Tn), P, G);
  return cudaGetLastError();
}

}  // namespace patch
