"""Seeded synthetic inputs for the PATCH hybrid tile-sparse linear layer.

This module only draws random inputs and encodes them the way the layer's
interface expects; it computes none of the layer's results.  Both the CPU
oracle (tests, bench baseline) and the CUDA path (tests, bench) are fed the
same bytes from here.

Recipe (one independent PCG64 stream per input):
    seed = 20250927 + 1000*config + 10*shape_idx + stream
    stream 0 = X, 1 = W, 2 = tile choice, 3 = tile logits, 4 = pattern logits

* X ~ N(0, 1) and W ~ N(0, 0.02) are drawn in fp32 and rounded to bf16
  (round to nearest, ties to even) on the bit pattern.
* Tile choice (dense = 0 / 2:4 sparse = 1 per 128x128 tile): Bernoulli(p)
  per tile, an exact count at seeded random positions, or one contiguous run
  of tiles in row-major order at a seeded offset ("clustered").
* Pattern ids: magnitude top-2 per group of 4 along K (the two largest |w|,
  ties to the lower index), the stand-in for a one-shot pruner's patterns.
  The id of a kept pair (i0, i1), i0 < i1, is its index in lexicographic
  order: (0,1)=0 (0,2)=1 (0,3)=2 (1,2)=3 (1,3)=4 (2,3)=5.
* Tile logits [Tn][Tk][2] and pattern logits [N][K/4][6] ~ N(0, 1) fp32.
"""
from __future__ import annotations

import numpy as np

TILE = 128
BASE_SEED = 20250927

STREAM_X, STREAM_W, STREAM_TILES, STREAM_TILE_LOGITS, STREAM_PAT_LOGITS = range(5)

# lexicographic numbering of the kept pair of a 2:4 group (input encoding)
_PAIR_ID = {(0, 1): 0, (0, 2): 1, (0, 3): 2, (1, 2): 3, (1, 3): 4, (2, 3): 5}


def rng(config: int, shape_idx: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(BASE_SEED + 1000 * config + 10 * shape_idx + stream))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def gen_x(M: int, K: int, config: int = 0, shape_idx: int = 0) -> np.ndarray:
    """Activations X [M][K] as bf16 bits, N(0, 1)."""
    r = rng(config, shape_idx, STREAM_X)
    return f32_to_bf16_bits(r.standard_normal((M, K), dtype=np.float32))


def gen_w(N: int, K: int, config: int = 0, shape_idx: int = 0, std: float = 0.02) -> np.ndarray:
    """Weights W [N][K] as bf16 bits, N(0, std)."""
    r = rng(config, shape_idx, STREAM_W)
    return f32_to_bf16_bits(r.standard_normal((N, K), dtype=np.float32) * np.float32(std))


def tiles_bernoulli(N: int, K: int, p: float, config: int = 0, shape_idx: int = 0) -> np.ndarray:
    """Tile kinds [Tn][Tk] uint8, each sparse with probability p."""
    r = rng(config, shape_idx, STREAM_TILES)
    return (r.random((N // TILE, K // TILE)) < p).astype(np.uint8)


def exact_sparse_count(T: int, frac: float) -> int:
    return min(T, int(np.floor(frac * T + 0.5)))


def tiles_exact(N: int, K: int, frac: float, config: int = 0, shape_idx: int = 0) -> np.ndarray:
    """Tile kinds with exactly floor(frac*T + 0.5) sparse tiles at seeded random positions."""
    Tn, Tk = N // TILE, K // TILE
    T = Tn * Tk
    ns = exact_sparse_count(T, frac)
    r = rng(config, shape_idx, STREAM_TILES)
    kinds = np.zeros(T, dtype=np.uint8)
    kinds[r.permutation(T)[:ns]] = 1
    return kinds.reshape(Tn, Tk)


def tiles_clustered(N: int, K: int, frac: float, config: int = 0, shape_idx: int = 0) -> np.ndarray:
    """One contiguous run of floor(frac*T + 0.5) sparse tiles in row-major tile order."""
    Tn, Tk = N // TILE, K // TILE
    T = Tn * Tk
    ns = exact_sparse_count(T, frac)
    r = rng(config, shape_idx, STREAM_TILES)
    start = int(r.integers(0, T - ns + 1))
    kinds = np.zeros(T, dtype=np.uint8)
    kinds[start:start + ns] = 1
    return kinds.reshape(Tn, Tk)


def mask_tiles(N: int, K: int, b: int, frac: float, clustered: bool, config: int = 0,
               shape_idx: int = 0) -> np.ndarray:
    """Kinds [N/b][K/b] uint8 of b x b mask tiles with exactly floor(frac*T_b + 0.5)
    sparse: at seeded random positions, or as one contiguous run in row-major
    tile order starting at a seeded offset (full-width bands of tile rows)."""
    Tn, Tk = N // b, K // b
    T = Tn * Tk
    ns = exact_sparse_count(T, frac)
    r = rng(config, shape_idx, STREAM_TILES)
    kinds = np.zeros(T, dtype=np.uint8)
    if clustered:
        start = int(r.integers(0, T - ns + 1))
        kinds[start:start + ns] = 1
    else:
        kinds[r.permutation(T)[:ns]] = 1
    return kinds.reshape(Tn, Tk)


def choice_logits(kinds: np.ndarray) -> np.ndarray:
    """Tile logits [..][..][2] fp32 whose argmax is the given kind: (1, 0) for a
    dense tile, (0, 1) for a sparse one."""
    out = np.zeros(kinds.shape + (2,), np.float32)
    out[..., 0] = (kinds == 0)
    out[..., 1] = (kinds != 0)
    return out


def patterns_top2(w_bits: np.ndarray) -> np.ndarray:
    """Pattern ids [N][K/4] uint8: keep the two largest |w| of each group of 4 (ties -> lower index)."""
    N, K = w_bits.shape
    mag = (w_bits.astype(np.uint16) & np.uint16(0x7FFF)).reshape(N, K // 4, 4).astype(np.int32)  # |w| order
    first = np.argmax(mag, axis=2)                      # largest, lowest index among equals
    np.put_along_axis(mag, first[:, :, None], -1, axis=2)
    second = np.argmax(mag, axis=2)                     # next largest, lowest index among equals
    lo, hi = np.minimum(first, second), np.maximum(first, second)
    table = np.full((4, 4), 255, dtype=np.uint8)
    for (a, b), pid in _PAIR_ID.items():
        table[a, b] = pid
    return table[lo, hi]


def gen_w_device(N: int, K: int, config: int, shape_idx: int, device, std: float = 0.02):
    """Weights W [N][K] as a bf16 torch tensor drawn on `device` with torch's
    generator seeded like gen_w: the same distribution, N(0, std) rounded to
    bf16 to nearest even, but not the same numbers (a different generator).
    For workloads too large to draw on the host (the 32-layer stack)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(BASE_SEED + 1000 * config + 10 * shape_idx + STREAM_W)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * std
    return w.to(torch.bfloat16)  # round to nearest even


def patterns_top2_torch(w):
    """patterns_top2 of a bf16 torch tensor, on its device: keep the two largest
    |w| of each group of 4 (ties -> lower index), lexicographic pair id."""
    import torch
    N, K = w.shape
    mag = (w.view(torch.int16).to(torch.int32) & 0x7FFF).view(N, K // 4, 4)  # |w| order on the bit pattern
    # rank key: larger magnitude first, then lower index
    key = mag * 4 + (3 - torch.arange(4, device=w.device, dtype=torch.int32))
    top = torch.topk(key, 2, dim=2).indices
    lo, hi = torch.minimum(top[..., 0], top[..., 1]), torch.maximum(top[..., 0], top[..., 1])
    table = torch.full((4, 4), 255, dtype=torch.uint8, device=w.device)
    for (a, b), pid in _PAIR_ID.items():
        table[a, b] = pid
    return table[lo, hi]


def gen_tile_logits(N: int, K: int, config: int = 0, shape_idx: int = 0, tile: int = TILE) -> np.ndarray:
    r = rng(config, shape_idx, STREAM_TILE_LOGITS)
    return r.standard_normal((N // tile, K // tile, 2), dtype=np.float32)


def gen_pattern_logits(N: int, K: int, config: int = 0, shape_idx: int = 0) -> np.ndarray:
    r = rng(config, shape_idx, STREAM_PAT_LOGITS)
    return r.standard_normal((N, K // 4, 6), dtype=np.float32)


# ---------------------------------------------------------------------------
# Workload tables (shapes are N x K of each linear layer)

LLAMA2_7B = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
             ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
LLAMA3_8B = [("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
             ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336)]
QWEN25_05B = [("q", 896, 896), ("k", 128, 896), ("v", 128, 896), ("o", 896, 896),
              ("gate", 4864, 896), ("up", 4864, 896), ("down", 896, 4864)]
# Gemma-3-1B linears (hidden 1152, 4 query heads and 1 key/value head of 256, MLP 6912),
# another of the model families the pages evaluate
GEMMA3_1B = [("q", 1024, 1152), ("k", 256, 1152), ("v", 256, 1152), ("o", 1152, 1024),
             ("gate", 6912, 1152), ("up", 6912, 1152), ("down", 1152, 6912)]


def stack_fraction(layer: int, proj: str, n_layers: int = 32) -> float:
    """Non-uniform sparse-tile fraction of the 32-layer stack: 0.1 in the first and
    last 4 layers, 0.7 in the middle ones, +0.1 for MLP matrices, capped at 1."""
    base = 0.1 if (layer < 4 or layer >= n_layers - 4) else 0.7
    if proj in ("gate", "up", "down"):
        base += 0.1
    return min(1.0, base)


def layer_inputs(N: int, K: int, M: int, tiles: np.ndarray, config: int, shape_idx: int):
    """(X, W, tile kinds, pattern ids) for one layer."""
    x = gen_x(M, K, config, shape_idx) if M > 0 else np.zeros((0, K), np.uint16)
    w = gen_w(N, K, config, shape_idx)
    return x, w, tiles, patterns_top2(w)
