"""CPU oracle for the PATCH hybrid tile-sparse linear layer (test infrastructure).

Only the test suite, the package smoke check and the benchmark's CPU-baseline
leg may import this package.  The arithmetic lives in ``patch_oracle.c``
(plain C, fp64, OpenMP over output elements); this module only compiles it
with gcc and marshals numpy arrays, except the gated MLP's SiLU and product
(``hybrid_mlp``), written here in fp64 numpy on top of the C GEMM.  It shares
no code with the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "patch_oracle.c"
_LIB = _HERE / "liboracle.so"

TILE = 128
_lib = None


def build(force: bool = False) -> Path:
    """Compile patch_oracle.c into liboracle.so (gcc -O2 -fopenmp)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.{os.getpid()}.tmp")
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
                        "-o", str(tmp), str(_SRC)], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(str(build()))
        P, I64 = ctypes.c_void_p, ctypes.c_int64
        for name, args in {
            "oracle_apply_mask": [P, I64, I64, P, P, P],
            "oracle_hard_mask": [P, I64, I64, P, P, P, P, P],
            "oracle_hard_mask_tiles": [P, I64, I64, I64, P, P, P, P, P],
            "oracle_exec_tiles": [P, I64, I64, I64, P, P],
            "oracle_pack": [P, I64, I64, P, P, I64, P, P, P],
            "oracle_unpack": [P, P, P, I64, I64, P],
            "oracle_gemm_rows": [P, I64, P, I64, P, I64, I64, P],
            "oracle_hybrid_gemm": [P, I64, P, I64, P, I64, I64, P, P, P],
            "oracle_apply_mask_tiles": [P, I64, I64, I64, P, P, P],
            "oracle_exec_tiles_e": [P, I64, I64, I64, I64, P, P],
            "oracle_pack64": [P, I64, I64, P, P, I64, P, P, P],
            "oracle_unpack64": [P, P, P, I64, I64, P],
        }.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        lib.oracle_pack_sizes.argtypes = [I64, I64, I64, P, P, P]
        lib.oracle_pack_sizes.restype = None
        lib.oracle_pack64_sizes.argtypes = [I64, I64, I64, P, P, P]
        lib.oracle_pack64_sizes.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = None
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: oracle error {rc}")


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    """OpenMP threads for the following oracle calls (CPU-baseline timing only)."""
    _load().oracle_set_num_threads(int(n))


def apply_mask(w: np.ndarray, bitmap: np.ndarray, pat_id: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w, np.uint16)
    N, K = w.shape
    out = np.empty_like(w)
    _check(_load().oracle_apply_mask(_ptr(w), N, K, _ptr(np.ascontiguousarray(bitmap, np.uint8)),
                                     _ptr(np.ascontiguousarray(pat_id, np.uint8)), _ptr(out)),
           "apply_mask")
    return out


def hard_mask(w: np.ndarray, tile_logits: np.ndarray, pattern_logits: np.ndarray):
    """Returns (W_masked, bitmap [Tn][Tk] u8, pat_id [N][K/4] u8)."""
    w = np.ascontiguousarray(w, np.uint16)
    N, K = w.shape
    wm = np.empty_like(w)
    bitmap = np.empty((N // TILE, K // TILE), np.uint8)
    pid = np.empty((N, K // 4), np.uint8)
    _check(_load().oracle_hard_mask(_ptr(w), N, K, _ptr(np.ascontiguousarray(tile_logits, np.float32)),
                                    _ptr(np.ascontiguousarray(pattern_logits, np.float32)),
                                    _ptr(wm), _ptr(bitmap), _ptr(pid)), "hard_mask")
    return wm, bitmap, pid


def hard_mask_tiles(w: np.ndarray, tile_logits: np.ndarray, pattern_logits: np.ndarray, mask_tile: int):
    """Hard mask with b x b mask tiles (b = mask_tile, 4..128): returns
    (W_masked, bitmap [N/b][K/b] u8, pat_id [N][K/4] u8)."""
    w = np.ascontiguousarray(w, np.uint16)
    N, K = w.shape
    b = int(mask_tile)
    wm = np.empty_like(w)
    bitmap = np.empty((N // b, K // b), np.uint8)
    pid = np.empty((N, K // 4), np.uint8)
    _check(_load().oracle_hard_mask_tiles(_ptr(w), N, K, b, _ptr(np.ascontiguousarray(tile_logits, np.float32)),
                                          _ptr(np.ascontiguousarray(pattern_logits, np.float32)),
                                          _ptr(wm), _ptr(bitmap), _ptr(pid)), "hard_mask_tiles")
    return wm, bitmap, pid


def exec_tiles(bitmap: np.ndarray, N: int, K: int, mask_tile: int):
    """128 x 128 execution tiles of a b x b mask bitmap: (exec [N/128][K/128] u8, n_sparse)."""
    bitmap = np.ascontiguousarray(bitmap, np.uint8)
    ex = np.empty((N // TILE, K // TILE), np.uint8)
    n = ctypes.c_int64()
    _check(_load().oracle_exec_tiles(_ptr(bitmap), N, K, int(mask_tile), _ptr(ex), ctypes.byref(n)), "exec_tiles")
    return ex, n.value


def pack_sizes(N: int, K: int, n_sparse: int):
    v, m, d = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _load().oracle_pack_sizes(N, K, n_sparse, ctypes.byref(v), ctypes.byref(m), ctypes.byref(d))
    return v.value, m.value, d.value


def pack(w: np.ndarray, bitmap: np.ndarray, pat_id: np.ndarray):
    """Returns (values u8, meta u8, desc u8) blobs of the packed format."""
    w = np.ascontiguousarray(w, np.uint16)
    N, K = w.shape
    bitmap = np.ascontiguousarray(bitmap, np.uint8)
    ns = int(np.count_nonzero(bitmap))
    vb, mb, db = pack_sizes(N, K, ns)
    values = np.zeros(vb, np.uint8)
    meta = np.zeros(max(mb, 1), np.uint8)
    desc = np.zeros(db, np.uint8)
    _check(_load().oracle_pack(_ptr(w), N, K, _ptr(bitmap), _ptr(np.ascontiguousarray(pat_id, np.uint8)),
                               ns, _ptr(values), _ptr(meta), _ptr(desc)), "pack")
    return values, meta[:mb], desc


def unpack(values: np.ndarray, meta: np.ndarray, desc: np.ndarray, N: int, K: int) -> np.ndarray:
    out = np.empty((N, K), np.uint16)
    meta = np.ascontiguousarray(meta, np.uint8) if meta.size else np.zeros(1, np.uint8)
    _check(_load().oracle_unpack(_ptr(np.ascontiguousarray(values, np.uint8)), _ptr(meta),
                                 _ptr(np.ascontiguousarray(desc, np.uint8)), N, K, _ptr(out)), "unpack")
    return out


# ---- 64 x 64 execution tiles ("Ablation Studies", tile size)

TILE64 = 64


def apply_mask_tiles(w: np.ndarray, bitmap: np.ndarray, pat_id: np.ndarray, mask_tile: int) -> np.ndarray:
    """The hybrid mask with b x b tiles (bitmap [N/b][K/b]) applied to W."""
    w = np.ascontiguousarray(w, np.uint16)
    N, K = w.shape
    out = np.empty_like(w)
    _check(_load().oracle_apply_mask_tiles(_ptr(w), N, K, int(mask_tile),
                                           _ptr(np.ascontiguousarray(bitmap, np.uint8)),
                                           _ptr(np.ascontiguousarray(pat_id, np.uint8)), _ptr(out)),
           "apply_mask_tiles")
    return out


def exec_tiles_e(bitmap: np.ndarray, N: int, K: int, mask_tile: int, exec_tile: int):
    """E x E execution tiles (E = 64 or 128) of a b x b mask bitmap: (exec [N/E][K/E] u8, n_sparse)."""
    bitmap = np.ascontiguousarray(bitmap, np.uint8)
    E = int(exec_tile)
    ex = np.empty((N // E, K // E), np.uint8)
    n = ctypes.c_int64()
    _check(_load().oracle_exec_tiles_e(_ptr(bitmap), N, K, int(mask_tile), E, _ptr(ex), ctypes.byref(n)),
           "exec_tiles_e")
    return ex, n.value


def pack64_sizes(N: int, K: int, n_sparse: int):
    v, m, d = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _load().oracle_pack64_sizes(N, K, n_sparse, ctypes.byref(v), ctypes.byref(m), ctypes.byref(d))
    return v.value, m.value, d.value


def pack64(w: np.ndarray, bitmap: np.ndarray, pat_id: np.ndarray):
    """Blobs (values, meta, desc) of the 64 x 64 execution-tile format; bitmap [N/64][K/64]."""
    w = np.ascontiguousarray(w, np.uint16)
    N, K = w.shape
    bitmap = np.ascontiguousarray(bitmap, np.uint8)
    ns = int(np.count_nonzero(bitmap))
    vb, mb, db = pack64_sizes(N, K, ns)
    values = np.zeros(vb, np.uint8)
    meta = np.zeros(max(mb, 1), np.uint8)
    desc = np.zeros(db, np.uint8)
    _check(_load().oracle_pack64(_ptr(w), N, K, _ptr(bitmap), _ptr(np.ascontiguousarray(pat_id, np.uint8)),
                                 ns, _ptr(values), _ptr(meta), _ptr(desc)), "pack64")
    return values, meta[:mb], desc


def unpack64(values: np.ndarray, meta: np.ndarray, desc: np.ndarray, N: int, K: int) -> np.ndarray:
    out = np.empty((N, K), np.uint16)
    meta = np.ascontiguousarray(meta, np.uint8) if meta.size else np.zeros(1, np.uint8)
    _check(_load().oracle_unpack64(_ptr(np.ascontiguousarray(values, np.uint8)), _ptr(meta),
                                   _ptr(np.ascontiguousarray(desc, np.uint8)), N, K, _ptr(out)), "unpack64")
    return out


def gemm(x: np.ndarray, w_eff: np.ndarray, rows: np.ndarray | None = None) -> np.ndarray:
    """fp64 Y = X * W_eff^T over bf16 bit inputs (optionally only the given rows of X)."""
    x = np.ascontiguousarray(x, np.uint16)
    w_eff = np.ascontiguousarray(w_eff, np.uint16)
    M, K = x.shape
    N = w_eff.shape[0]
    r = None if rows is None else np.ascontiguousarray(rows, np.int64)
    R = M if r is None else r.size
    y = np.empty((R, N), np.float64)
    _check(_load().oracle_gemm_rows(_ptr(x), M, _ptr(r), 0 if r is None else r.size,
                                    _ptr(w_eff), N, K, _ptr(y)), "gemm")
    return y


def hybrid_gemm(x: np.ndarray, w: np.ndarray, bitmap: np.ndarray, pat_id: np.ndarray,
                rows: np.ndarray | None = None) -> np.ndarray:
    """The layer: hybrid mask applied to W, then fp64 Y = X * W_eff^T."""
    x = np.ascontiguousarray(x, np.uint16)
    w = np.ascontiguousarray(w, np.uint16)
    M, K = x.shape
    N = w.shape[0]
    r = None if rows is None else np.ascontiguousarray(rows, np.int64)
    R = M if r is None else r.size
    y = np.empty((R, N), np.float64)
    _check(_load().oracle_hybrid_gemm(_ptr(x), M, _ptr(r), 0 if r is None else r.size, _ptr(w), N, K,
                                      _ptr(np.ascontiguousarray(bitmap, np.uint8)),
                                      _ptr(np.ascontiguousarray(pat_id, np.uint8)), _ptr(y)),
           "hybrid_gemm")
    return y


def chain(x0: np.ndarray, layers) -> list:
    """Hybrid layers run back to back ("Experimental Results" -> "Speedup &
    Efficiency": the model's linear layers executed in sequence): layer i
    multiplies the previous layer's output, rounded once to bf16 (nearest
    even) as a bf16 activation is, by its hybrid weight.  layers: list of
    (w, bitmap, pat_id); x0 bf16 bits [M][K0].  Returns every layer's output:
    fp64, unrounded (for comparison), and the bf16 bits fed to the next."""
    outs, x = [], np.ascontiguousarray(x0, np.uint16)
    for w, bm, ids in layers:
        y = hybrid_gemm(x, w, bm, ids)
        outs.append(y)
        x = _f64_to_bf16_rne(y)
    return outs


def bf16_rne(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bits, round to nearest even (the rounding of every output)."""
    return _f64_to_bf16_rne(x)


def silu(z):
    """SiLU, z * sigmoid(z), in fp64: the gate activation of LLaMA's gated MLP
    (the linears of the pages' LLaMA-2 7B end-to-end runs, "Experimental
    Results" -> "Speedup & Efficiency"; the activation itself is LLaMA's, the
    pages do not state it)."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def hybrid_mlp(x: np.ndarray, gate, up, rows: np.ndarray | None = None) -> np.ndarray:
    """H = silu(X W_gate_eff^T) * (X W_up_eff^T) in fp64, the gated MLP's first
    half on two hybrid weights; gate and up are (w, bitmap, pat_id)."""
    g = hybrid_gemm(x, *gate, rows=rows)
    u = hybrid_gemm(x, *up, rows=rows)
    return silu(g) * u


# patterns as keep-position pairs, numbered lexicographically (the library's reading)
_PAIRS = ((0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3))


def soft_mask(w: np.ndarray, tile_logits: np.ndarray, pattern_logits: np.ndarray, tau: float,
              tile_noise: np.ndarray | None = None, pattern_noise: np.ndarray | None = None):
    """The training-time (soft) hybrid mask of "Core Mechanism" / "Learnable
    Distributions", in fp64, following its steps:
      1. tile choice:    p = softmax((tile_logits + tile_noise) / tau) over (dense, sparse);
      2. pattern choice: q = softmax((pattern_logits + pattern_noise) / tau) over the 6 patterns;
      3. hybrid mask:    M[n][k] = p_dense + p_sparse * sum_j q_j [k mod 4 in pattern j];
      4. soft weight:    W_soft = W * M, rounded once to bf16 (nearest even).
    The noise is the caller's (Gumbel samples; zero when None).  Returns
    (W_soft bf16 bits [N][K], M fp64 [N][K])."""
    N, K = w.shape
    Tn, Tk = N // TILE, K // TILE
    tl = tile_logits.astype(np.float64) + (0.0 if tile_noise is None else tile_noise.astype(np.float64))
    pl = pattern_logits.astype(np.float64) + (0.0 if pattern_noise is None else pattern_noise.astype(np.float64))

    def softmax(z):
        z = z / tau
        z = z - z.max(axis=-1, keepdims=True)
        e = np.exp(z)
        return e / e.sum(axis=-1, keepdims=True)

    p = softmax(tl.reshape(Tn, Tk, 2))                         # [Tn][Tk][2]
    q = softmax(pl.reshape(N, K // 4, 6))                      # [N][K/4][6]
    keep = np.zeros((N, K // 4, 4))
    for j, (a, b) in enumerate(_PAIRS):
        keep[:, :, a] += q[:, :, j]
        keep[:, :, b] += q[:, :, j]
    keep = keep.reshape(N, K)
    pd = np.repeat(np.repeat(p[:, :, 0], TILE, axis=0), TILE, axis=1)
    ps = np.repeat(np.repeat(p[:, :, 1], TILE, axis=0), TILE, axis=1)
    m = pd + ps * keep
    wf = (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return _f64_to_bf16_rne(wf * m), m


def _f64_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bits, round to nearest even.  Goes through fp32 (nearest
    even); that double rounding can only go wrong when the fp32 value lands
    exactly half way between two bf16 values, and those cases are settled by
    comparing the fp64 value with that midpoint."""
    f = np.asarray(x, np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    hi = u >> 16
    r = ((u + 0x7FFF + (hi & 1)) >> 16).astype(np.uint16)
    mid = (u & 0xFFFF) == 0x8000
    if np.any(mid):
        xm, fm = np.asarray(x, np.float64)[mid], f[mid].astype(np.float64)
        res = r[mid]
        res = np.where(np.abs(xm) > np.abs(fm), (hi[mid] + 1).astype(np.uint16), res)
        res = np.where(np.abs(xm) < np.abs(fm), hi[mid].astype(np.uint16), res)
        r[mid] = res
    return r
