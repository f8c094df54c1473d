"""Pins of the CPU oracle against facts fixed outside it (no GPU needed).

Each test checks the oracle against something it does not compute itself:
the method's invariants (PATCH: Learnable Tile-level Hybrid Sparsity for LLMs,
section 2 "Methodology: PATCH"), brute force over the 6 patterns, numpy's
library matmul / argmax, closed-form sizes, and the pattern table under
tests/golden/.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
import synth_inputs as si
from _util import bf16_to_f64

TILE = 128
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pattern_codes.txt")
PAIRS = list(itertools.combinations(range(4), 2))  # lexicographic, library-generated
ONE = np.uint16(0x3F80)  # bf16 1.0


def golden_codes():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                i, a, b, c = line.split()
                rows.append((int(i), int(a), int(b), int(c, 16)))
    return rows


def mask_from_pairs(bitmap, pat_id, N, K):
    """Keep-mask built from the itertools pair list (independent of the oracle's table)."""
    keep = np.ones((N, K), bool)
    pos = np.arange(K) % 4
    for n in range(N):
        for tk in range(K // TILE):
            if bitmap[n // TILE, tk]:
                sl = slice(tk * TILE, (tk + 1) * TILE)
                ids = np.repeat(pat_id[n, tk * 32:(tk + 1) * 32], 4)
                a = np.array([PAIRS[i][0] for i in ids])
                b = np.array([PAIRS[i][1] for i in ids])
                keep[n, sl] = (pos[sl] == a) | (pos[sl] == b)
    return keep


def f64(bits):
    return si.bf16_bits_to_f32(bits).astype(np.float64)


# ---------------------------------------------------------------- hard mask


@pytest.mark.parametrize("pid", range(6))
def test_hard_mask_one_hot_pattern(pid):
    N = K = TILE
    w = np.full((N, K), ONE, np.uint16)
    tl = np.zeros((1, 1, 2), np.float32)
    tl[..., 1] = 1.0  # sparse
    pl = np.zeros((N, K // 4, 6), np.float32)
    pl[..., pid] = 1.0
    wm, bm, ids = oracle.hard_mask(w, tl, pl)
    assert bm.tolist() == [[1]]
    assert np.all(ids == pid)
    keep = np.zeros(4, bool)
    keep[list(PAIRS[pid])] = True
    expect = np.where(np.tile(keep, K // 4)[None, :], ONE, np.uint16(0))
    assert np.array_equal(wm, np.broadcast_to(expect, (N, K)))


def test_hard_mask_tile_choice_and_ties():
    N, K = 2 * TILE, 2 * TILE
    w = np.full((N, K), ONE, np.uint16)
    tl = np.array([[[1.0, 0.0], [0.0, 1.0]], [[0.5, 0.5], [-1.0, -0.5]]], np.float32)
    pl = np.zeros((N, K // 4, 6), np.float32)  # all tied -> pattern 0
    wm, bm, ids = oracle.hard_mask(w, tl, pl)
    assert bm.tolist() == [[0, 1], [0, 1]]  # tie -> dense (index 0)
    assert np.all(ids == 0)
    # sparse tiles keep positions 0,1 of each group; dense tiles keep all
    assert np.all(wm[:TILE, :TILE] == ONE)
    assert np.all(wm[:TILE, TILE:].reshape(TILE, -1, 4)[:, :, 2:] == 0)
    assert np.all(wm[:TILE, TILE:].reshape(TILE, -1, 4)[:, :, :2] == ONE)


def test_hard_mask_pattern_ties_and_nan_reading():
    N = K = TILE
    w = np.full((N, K), ONE, np.uint16)
    tl = np.array([[[0.0, 1.0]]], np.float32)
    pl = np.zeros((N, K // 4, 6), np.float32)
    pl[0, 0] = [0, 1, 1, 0, 0, 0]          # tie between 1 and 2 -> 1
    pl[0, 1] = [np.nan, 5, 6, 7, 8, 9]     # NaN first: no later value beats it -> 0
    pl[0, 2] = [0, np.nan, 1, 0, 0, 0]     # NaN later never wins -> 2
    pl[0, 3] = [-3, -2, -1, -1, -5, -1]    # first maximum -> 2
    _, _, ids = oracle.hard_mask(w, tl, pl)
    assert ids[0, :4].tolist() == [1, 0, 2, 2]


def test_hard_mask_matches_numpy_argmax_random():
    N, K = 256, 384
    w = si.gen_w(N, K, 1, 0)
    tl = si.gen_tile_logits(N, K, 1, 0)
    pl = si.gen_pattern_logits(N, K, 1, 0)
    wm, bm, ids = oracle.hard_mask(w, tl, pl)
    assert np.array_equal(bm, np.argmax(tl, axis=-1).astype(np.uint8))
    assert np.array_equal(ids, np.argmax(pl, axis=-1).astype(np.uint8))
    keep = mask_from_pairs(bm, ids, N, K)
    assert np.array_equal(wm, np.where(keep, w, np.uint16(0)))


def test_pruned_weights_are_positive_zero():
    N = K = TILE
    w = np.full((N, K), np.uint16(0xBF80), np.uint16)  # -1.0
    bm = np.ones((1, 1), np.uint8)
    ids = np.full((N, K // 4), 5, np.uint8)
    wm = oracle.apply_mask(w, bm, ids)
    g = wm.reshape(N, -1, 4)
    assert np.all(g[:, :, :2] == 0x0000) and np.all(g[:, :, 2:] == 0xBF80)


# --------------------------------------------------------------- invariants


@pytest.mark.parametrize("frac", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_two_of_four_and_global_sparsity(frac):
    N, K = 3 * TILE, 4 * TILE
    w = np.full((N, K), ONE, np.uint16)
    bm = si.tiles_exact(N, K, frac, 3, 7)
    ids = np.random.default_rng(5).integers(0, 6, (N, K // 4)).astype(np.uint8)
    wm = oracle.apply_mask(w, bm, ids)
    nz = (wm != 0).reshape(N // TILE, TILE, K // TILE, TILE // 4, 4).sum(-1)
    for tn in range(N // TILE):
        for tk in range(K // TILE):
            expect = 2 if bm[tn, tk] else 4
            assert np.all(nz[tn, :, tk, :] == expect)
    T = bm.size
    ns = int(bm.sum())
    pruned = int(np.count_nonzero(wm == 0))
    assert pruned * 2 * T == N * K * ns  # sparsity == 0.5 * ns / T exactly
    assert 0.0 <= pruned / (N * K) <= 0.5


# ---------------------------------------------------------------- packing


def test_pack_sizes_closed_form():
    for N, K, ns in [(128, 128, 0), (128, 128, 1), (4096, 4096, 512), (11008, 4096, 1376)]:
        T = (N // TILE) * (K // TILE)
        assert oracle.pack_sizes(N, K, ns) == ((T - ns) * 32768 + ns * 16384, ns * 2048, 16 * T)


@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_pack_unpack_round_trip(frac):
    N, K = 3 * TILE, 5 * TILE
    w = si.gen_w(N, K, 2, 1)
    bm = si.tiles_exact(N, K, frac, 2, 1)
    ids = si.patterns_top2(w)
    values, meta, desc = oracle.pack(w, bm, ids)
    vb, mb, db = oracle.pack_sizes(N, K, int(bm.sum()))
    assert (values.size, meta.size, desc.size) == (vb, mb, db)
    w_eff = oracle.unpack(values, meta, desc, N, K)
    assert np.array_equal(w_eff, oracle.apply_mask(w, bm, ids))
    # masked and unmasked W pack to the same bytes
    v2, m2, d2 = oracle.pack(oracle.apply_mask(w, bm, ids), bm, ids)
    assert np.array_equal(values, v2) and np.array_equal(meta, m2) and np.array_equal(desc, d2)


def test_descriptor_table():
    N, K = 2 * TILE, 3 * TILE
    w = si.gen_w(N, K)
    bm = np.array([[1, 0, 1], [0, 0, 1]], np.uint8)
    _, _, desc = oracle.pack(w, bm, si.patterns_top2(w))
    d = desc.reshape(-1, 16)
    kinds = d[:, 0:4].copy().view("<u4").ravel()
    ords = d[:, 4:8].copy().view("<u4").ravel()
    offs = d[:, 8:16].copy().view("<u8").ravel()
    assert kinds.tolist() == [1, 0, 1, 0, 0, 1]
    assert ords.tolist() == [0, 0xFFFFFFFF, 1, 0xFFFFFFFF, 0xFFFFFFFF, 2]
    sizes = [16384 if k else 32768 for k in kinds]
    assert offs.tolist() == list(np.concatenate([[0], np.cumsum(sizes)[:-1]]))


def spec_values_blob(w, bm, ids, desc_offsets):
    """The values blob restated from the packed format's text (a panel is 128
    rows x 64 bf16 with 128-byte rows; a dense tile is 2 panels, k 0..63 then
    k 64..127; a sparse tile is 1 panel whose row r holds group g's two kept
    values in ascending k at positions 2g, 2g + 1), placed at each tile's
    val_offset.  Written with numpy slicing, independently of the C oracle."""
    N, K = w.shape
    Tn, Tk = N // TILE, K // TILE
    size = int(sum(16384 if bm[tn, tk] else 32768 for tn in range(Tn) for tk in range(Tk)))
    blob = np.zeros(size // 2, np.uint16)
    for tn in range(Tn):
        for tk in range(Tk):
            o = int(desc_offsets[tn * Tk + tk]) // 2
            tile = w[tn * TILE:(tn + 1) * TILE, tk * TILE:(tk + 1) * TILE]
            if not bm[tn, tk]:
                for h in range(2):
                    panel = tile[:, 64 * h:64 * (h + 1)]                    # 128 rows x 64 values
                    blob[o + 8192 * h:o + 8192 * (h + 1)] = panel.reshape(-1)  # row-major, 128-byte rows
            else:
                groups = tile.reshape(TILE, 32, 4)
                pid = ids[tn * TILE:(tn + 1) * TILE, tk * 32:(tk + 1) * 32]
                first = np.array([PAIRS[i][0] for i in pid.ravel()]).reshape(TILE, 32)
                second = np.array([PAIRS[i][1] for i in pid.ravel()]).reshape(TILE, 32)
                kept = np.stack([np.take_along_axis(groups, first[..., None], 2)[..., 0],
                                 np.take_along_axis(groups, second[..., None], 2)[..., 0]], axis=2)
                blob[o:o + 8192] = kept.reshape(-1)                         # row r: g0a g0b g1a g1b ...
    return blob.view(np.uint8)


def test_values_blob_layout_against_the_format_text():
    # every weight a distinct bf16 bit pattern, so a byte in the wrong place
    # (panel order, row stride, kept-value order) cannot match by accident
    N, K = 2 * TILE, 2 * TILE
    w = np.arange(N * K, dtype=np.uint32).astype(np.uint16).reshape(N, K)
    assert len(np.unique(w)) == N * K
    rng = np.random.default_rng(7)
    ids = rng.integers(0, 6, size=(N, K // 4)).astype(np.uint8)
    for bm in (np.array([[0, 1], [1, 0]], np.uint8), np.array([[1, 1], [0, 0]], np.uint8),
               np.zeros((2, 2), np.uint8), np.ones((2, 2), np.uint8)):
        values, _, desc = oracle.pack(w, bm, ids)
        offs = desc.reshape(-1, 16)[:, 8:16].copy().view("<u8").ravel()
        expect = spec_values_blob(w, bm, ids, offs)
        assert values.size == expect.size
        assert np.array_equal(values, expect), bm.tolist()
    # a few bytes spelled out: dense tile (0, 0), panel 1, row 3, value 5 is W[3][64 + 5]
    bm = np.array([[0, 1], [1, 0]], np.uint8)
    values, _, desc = oracle.pack(w, bm, ids)
    v16 = values.view(np.uint16)
    assert v16[(16384 + 3 * 128 + 5 * 2) // 2] == w[3, 69]
    # sparse tile (0, 1) starts after the 32 KiB dense tile; its row 7, group 9 keeps PAIRS[id]
    a, b = PAIRS[ids[7, 32 + 9]]
    assert v16[(32768 + 7 * 128 + 9 * 4) // 2] == w[7, 128 + 36 + a]
    assert v16[(32768 + 7 * 128 + 9 * 4 + 2) // 2] == w[7, 128 + 36 + b]


def test_pattern_codes_against_golden():
    codes = golden_codes()
    assert [(a, b) for _, a, b, _ in codes] == PAIRS
    N = K = TILE
    w = np.full((N, K), ONE, np.uint16)
    bm = np.ones((1, 1), np.uint8)
    for pid, a, b, code in codes:
        assert code == a | (b << 2)
        _, meta, _ = oracle.pack(w, bm, np.full((N, K // 4), pid, np.uint8))
        assert np.all(meta == (code | (code << 4)))


def hw_meta_position(r, g):
    """Byte and nibble of group g of tile row r, restated from the tensor-memory
    placement the 16-bit sparse MMA (M = 128) reads: lane = r%8 + 8*((k//16)%2)
    + 16*(r//16), 32-bit column = k//32, byte in column = (k%16)//8 + 2*((r//8)%2),
    nibble = (k//4)%2, with k = 4g; a tcgen05.cp 128x128b copy puts 16 bytes per lane."""
    k = 4 * g
    lane = r % 8 + 8 * ((k // 16) % 2) + 16 * (r // 16)
    col = k // 32
    byte = (k % 16) // 8 + 2 * ((r // 8) % 2)
    return lane * 16 + col * 4 + byte, (k // 4) % 2


def test_metadata_layout_positions():
    N = K = TILE
    w = np.full((N, K), ONE, np.uint16)
    bm = np.ones((1, 1), np.uint8)
    seen = set()
    rng = np.random.default_rng(11)
    cells = [(r, g) for r in range(TILE) for g in range(32)]
    for idx in rng.permutation(len(cells))[:512]:
        r, g = cells[idx]
        ids = np.zeros((N, K // 4), np.uint8)  # code 0x4 everywhere
        ids[r, g] = 5                          # code 0xE at one group
        _, meta, _ = oracle.pack(w, bm, ids)
        byte, nib = hw_meta_position(r, g)
        assert (meta[byte] >> (4 * nib)) & 0xF == 0xE
        others = meta.copy()
        others[byte] &= ~np.uint8(0xF << (4 * nib))
        others[byte] |= np.uint8(0x4 << (4 * nib))
        assert np.all(others == 0x44)
        seen.add((byte, nib))
    assert len(seen) == 512
    # the restated placement is a bijection onto the 2048 bytes x 2 nibbles
    allpos = {hw_meta_position(r, g) for r, g in cells}
    assert len(allpos) == TILE * 32


# ------------------------------------------------------------------- GEMM


def test_gemm_all_dense_is_dense_matmul():
    M, N, K = 5, 2 * TILE, 3 * TILE
    x, w = si.gen_x(M, K, 4, 0), si.gen_w(N, K, 4, 0)
    bm = np.zeros((N // TILE, K // TILE), np.uint8)
    y = oracle.hybrid_gemm(x, w, bm, si.patterns_top2(w))
    ref = f64(x) @ f64(w).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_gemm_all_sparse_is_24_matmul():
    M, N, K = 4, 2 * TILE, 2 * TILE
    x, w = si.gen_x(M, K, 4, 1), si.gen_w(N, K, 4, 1)
    bm = np.ones((N // TILE, K // TILE), np.uint8)
    ids = np.random.default_rng(3).integers(0, 6, (N, K // 4)).astype(np.uint8)
    y = oracle.hybrid_gemm(x, w, bm, ids)
    keep = mask_from_pairs(bm, ids, N, K)
    ref = f64(x) @ np.where(keep, f64(w), 0.0).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_gemm_one_hot_columns_brute_force():
    N = K = TILE
    w = si.gen_w(N, K, 4, 2)
    bm = np.ones((1, 1), np.uint8)
    ids = (np.arange(N * (K // 4)) % 6).astype(np.uint8).reshape(N, K // 4)  # all 6 patterns
    x = np.zeros((K, K), np.uint16)
    x[np.arange(K), np.arange(K)] = ONE       # row m is the unit vector e_m
    y = oracle.hybrid_gemm(x, w, bm, ids)     # y[m][n] = W_eff[n][m]
    for n in range(N):
        for g in range(K // 4):
            a, b = PAIRS[ids[n, g]]
            for i in range(4):
                expect = f64(w[n, 4 * g + i]) if i in (a, b) else 0.0
                assert y[4 * g + i, n] == expect


def test_gemm_linear_over_tiles():
    M, N, K = 3, 3 * TILE, 3 * TILE
    x, w = si.gen_x(M, K, 4, 3), si.gen_w(N, K, 4, 3)
    bm = si.tiles_exact(N, K, 0.5, 4, 3)
    ids = si.patterns_top2(w)
    y = oracle.hybrid_gemm(x, w, bm, ids)
    tile_is_sparse = np.kron(bm, np.ones((TILE, TILE), np.uint8)).astype(bool)
    keep = mask_from_pairs(bm, ids, N, K)
    w_dense_part = np.where(~tile_is_sparse, f64(w), 0.0)
    w_sparse_part = np.where(tile_is_sparse & keep, f64(w), 0.0)
    ref = f64(x) @ w_dense_part.T + f64(x) @ w_sparse_part.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_gemm_row_sample_equals_full():
    M, N, K = 9, TILE, 2 * TILE
    x, w = si.gen_x(M, K, 4, 4), si.gen_w(N, K, 4, 4)
    bm = si.tiles_bernoulli(N, K, 0.5, 4, 4)
    ids = si.patterns_top2(w)
    full = oracle.hybrid_gemm(x, w, bm, ids)
    rows = np.array([8, 0, 3])
    assert np.array_equal(oracle.hybrid_gemm(x, w, bm, ids, rows=rows), full[rows])


# ---------------------------------------------------------- input recipe


def test_top2_patterns_are_magnitude_argmax():
    """Generator's top-2 ids == argmax over the 6 pairs of |wi|+|wj| (fp64, ties low)."""
    w = si.gen_w(TILE, TILE, 6, 0)
    w[0, :4] = [0x3F80, 0xBF80, 0x3F80, 0x0000]  # |1|,|-1|,|1|,0 -> tie resolved to (0,1)
    ids = si.patterns_top2(w)
    mag = np.abs(f64(w)).reshape(TILE, -1, 4)
    score = np.stack([mag[:, :, a] + mag[:, :, b] for a, b in PAIRS], axis=-1)
    assert np.array_equal(ids, np.argmax(score, axis=-1).astype(np.uint8))
    assert ids[0, 0] == 0


def test_bf16_rounding_is_rne():
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e-3], np.float32)
    b = si.f32_to_bf16_bits(f)
    assert b.tolist()[:4] == [0x3F80, 0x3F80, 0x3F82, 0xC020]  # ties go to even
    assert abs(si.bf16_bits_to_f32(b)[4] - 3.0e-3) < 3.0e-3 * 2 ** -8


def test_bf16_rne_from_fp64_ties_and_double_rounding():
    one = 1.0
    ulp = 2.0 ** -7  # bf16 spacing at 1
    # exact ties go to even; just above / below a tie go up / down
    x = np.array([one + ulp / 2, one + 3 * ulp / 2, one + ulp / 2 + 2 ** -40, one + ulp / 2 - 2 ** -40, -2.5, 0.0])
    assert oracle.bf16_rne(x).tolist() == [0x3F80, 0x3F82, 0x3F81, 0x3F80, 0xC020, 0x0000]
    # a value whose fp32 rounding lands exactly on a bf16 midpoint (double rounding) still rounds by the fp64 value
    x = np.array([one + ulp / 2 + 2 ** -30])  # fp32 rounds it to the midpoint 1 + ulp/2
    assert np.float32(x[0]) == np.float32(one + ulp / 2)
    assert oracle.bf16_rne(x).tolist() == [0x3F81]


def _identity_layer(n):
    w = np.zeros((n, n), np.uint16)
    w[np.arange(n), np.arange(n)] = ONE
    return w, np.zeros((n // TILE, n // TILE), np.uint8), np.zeros((n, n // 4), np.uint8)


def test_chain_composes_layers_in_order_with_bf16_between():
    M, K = 3, TILE
    x0 = si.gen_x(M, K, 9, 0)
    w1 = si.gen_w(K, K, 9, 1)
    bm1 = np.ones((1, 1), np.uint8)
    ids1 = si.patterns_top2(w1)
    # one layer: the hybrid GEMM itself
    (y,) = oracle.chain(x0, [(w1, bm1, ids1)])
    assert np.array_equal(y, oracle.hybrid_gemm(x0, w1, bm1, ids1))
    # identity after it: the first output rounded once to bf16, exactly
    y1, y2 = oracle.chain(x0, [(w1, bm1, ids1), _identity_layer(K)])
    assert np.array_equal(y2, f64(oracle.bf16_rne(y1)))
    # a permutation before it: the same as permuting X's columns
    perm = np.random.default_rng(3).permutation(K)
    wp = np.zeros((K, K), np.uint16)
    wp[np.arange(K), perm] = ONE  # (X Wp^T)[m][n] = X[m][perm[n]]
    zero_bm, zero_ids = np.zeros((1, 1), np.uint8), np.zeros((K, K // 4), np.uint8)
    _, y = oracle.chain(x0, [(wp, zero_bm, zero_ids), (w1, bm1, ids1)])
    assert np.array_equal(y, oracle.hybrid_gemm(x0[:, perm], w1, bm1, ids1))


# ---------------------------------------------------------------- gated MLP


def test_silu_closed_forms_and_identities():
    """silu against an independent form: z * (1 + tanh(z / 2)) / 2, plus
    silu(0) = 0, silu(1) = e / (1 + e), silu(z) - silu(-z) = z and the limits."""
    z = np.linspace(-30.0, 30.0, 2001)
    tanh_form = z * (1.0 + np.tanh(z / 2.0)) / 2.0
    # (the tanh form loses relative accuracy to cancellation for very negative z)
    assert np.allclose(oracle.silu(z), tanh_form, rtol=1e-12, atol=1e-14)
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(1.0) == pytest.approx(math.e / (1.0 + math.e), rel=1e-15)
    assert np.allclose(oracle.silu(z) - oracle.silu(-z), z, rtol=1e-13, atol=1e-12)
    assert oracle.silu(800.0) == 800.0 and oracle.silu(-800.0) == 0.0


def test_hybrid_mlp_on_one_hot_inputs():
    """Brute force on a one-hot X column: H[m][n] = silu(Wg_eff[n][k]) * Wu_eff[n][k]
    for every kept k, with the activation evaluated through tanh instead."""
    N, K = 128, 256
    wg = si.gen_w(N, K, 0, 5, std=0.5)
    wu = si.gen_w(N, K, 0, 6, std=0.5)
    bmg = np.array([[0, 1]], np.uint8)
    bmu = np.array([[1, 0]], np.uint8)
    idg, idu = si.patterns_top2(wg), si.patterns_top2(wu)
    ks = [0, 5, 130, 255]
    x = np.zeros((len(ks), K), np.uint16)
    for m, k in enumerate(ks):
        x[m, k] = 0x3F80  # 1.0
    h = oracle.hybrid_mlp(x, (wg, bmg, idg), (wu, bmu, idu))
    geff = bf16_to_f64(oracle.apply_mask(wg, bmg, idg))
    ueff = bf16_to_f64(oracle.apply_mask(wu, bmu, idu))
    for m, k in enumerate(ks):
        g, u = geff[:, k], ueff[:, k]
        assert np.allclose(h[m], g * (1.0 + np.tanh(g / 2.0)) / 2.0 * u, rtol=1e-12, atol=1e-15)


# ------------------------------------------------- soft (training-time) hybrid mask


def _distinct_int_logits(shape, seed):
    """Logits whose entries along the last axis are distinct integers (gaps >= 1)."""
    rng = np.random.default_rng(seed)
    n = shape[-1]
    base = np.argsort(rng.random(shape), axis=-1).astype(np.float32)  # a permutation of 0..n-1
    return base - n / 2


def test_soft_mask_cold_limit_is_the_hard_mask():
    """tau -> 0 with integer-separated logits: the soft mask becomes the
    hard mask's 0/1 keep mask and W_soft to the hard-masked W, bit for bit."""
    N, K = 256, 384
    w = si.gen_w(N, K, 3, 0)
    tl = _distinct_int_logits((N // TILE, K // TILE, 2), 1)
    pl = _distinct_int_logits((N, K // 4, 6), 2)
    ws, m = oracle.soft_mask(w, tl, pl, tau=1e-3)  # e^-(gap/tau) underflows to exactly 0
    wm, bm, ids = oracle.hard_mask(w, tl, pl)
    keep = np.zeros((N, K))
    for n in range(0, N, 37):
        for g in range(K // 4):
            t = bm[n // TILE, (4 * g) // TILE]
            kept = PAIRS[ids[n, g]] if t else (0, 1, 2, 3)
            for i in kept:
                keep[n, 4 * g + i] = 1.0
        assert np.allclose(m[n], keep[n], atol=1e-15)
    # W * 0 is -0 for a negative weight (a product); the hard mask selects +0
    assert np.array_equal(np.where(ws == 0x8000, np.uint16(0), ws), wm)


def test_soft_mask_hot_limit_and_group_sums():
    """tau -> infinity: p = 1/2, q = 1/6, each position lies in 3 of the 6
    patterns, so M = 1/2 + 1/2 * 3/6 = 3/4.  At any tau the 4 entries of a
    group sum to 4 p_dense + 2 p_sparse, with p_sparse = 1 / (1 + e^((l_d - l_s)/tau))."""
    N, K = 128, 256
    w = si.gen_w(N, K, 4, 0)
    tl = si.gen_tile_logits(N, K, 4, 0)
    pl = si.gen_pattern_logits(N, K, 4, 0)
    _, m_hot = oracle.soft_mask(w, tl, pl, tau=1e12)
    assert np.allclose(m_hot, 0.75, atol=1e-9)
    tau = 0.7
    _, m = oracle.soft_mask(w, tl, pl, tau=tau)
    assert np.all(m >= 0.0) and np.all(m <= 1.0)
    sums = m.reshape(N, K // 4, 4).sum(axis=2)
    for n in (0, 63, 127):
        for g in (0, 17, 63):
            ld, ls = float(tl[n // TILE, (4 * g) // TILE, 0]), float(tl[n // TILE, (4 * g) // TILE, 1])
            ps = 1.0 / (1.0 + math.exp((ld - ls) / tau))
            assert sums[n, g] == pytest.approx(4.0 * (1.0 - ps) + 2.0 * ps, rel=1e-12)


def test_soft_mask_noise_enters_as_a_sum_and_patterns_map_to_pairs():
    N, K = 128, 128
    w = si.gen_w(N, K, 5, 0)
    rng = np.random.default_rng(7)
    tl = rng.standard_normal((1, 1, 2)).astype(np.float32)
    pl = rng.standard_normal((N, K // 4, 6)).astype(np.float32)
    tg = rng.gumbel(size=(1, 1, 2)).astype(np.float32)
    pg = rng.gumbel(size=(N, K // 4, 6)).astype(np.float32)
    a = oracle.soft_mask(w, tl, pl, 0.5, tg, pg)
    b = oracle.soft_mask(w, (tl.astype(np.float64) + tg), (pl.astype(np.float64) + pg), 0.5)
    assert np.array_equal(a[0], b[0]) and np.allclose(a[1], b[1], rtol=1e-15)
    # a sparse-only tile and one dominant pattern per group: M = its keep mask
    tl1 = np.array([[[-1e3, 1e3]]], np.float32)
    for j, pair in enumerate(PAIRS):
        pl1 = np.zeros((N, K // 4, 6), np.float32)
        pl1[:, :, j] = 1e3
        _, m1 = oracle.soft_mask(w, tl1, pl1, 1.0)
        expect = np.array([1.0 if i in pair else 0.0 for i in range(4)])
        assert np.allclose(m1.reshape(N, K // 4, 4), expect, atol=1e-12)


# ---- mask tiles smaller than the 128 x 128 execution tile ("Ablation Studies", tile size)

MASK_TILES = [4, 8, 16, 32, 64, 128]


def test_mask_tiles_at_128_are_the_hard_mask():
    """b = 128 reduces to the (separately pinned) 128 x 128 hard mask."""
    N, K = 2 * TILE, 3 * TILE
    w = si.gen_w(N, K, 5, 1)
    tl = si.gen_tile_logits(N, K, 5, 1)
    pl = si.gen_pattern_logits(N, K, 5, 1)
    for a, b in zip(oracle.hard_mask(w, tl, pl), oracle.hard_mask_tiles(w, tl, pl, 128)):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("b", [4, 8, 16, 32, 64])
def test_mask_tiles_keep_exactly_what_each_tile_chose(b):
    """All-ones W, one-hot logits drawn at random: every b x b block is fully kept
    when its tile logit says dense, and keeps exactly its group's pair otherwise
    (the pair read from the lexicographic enumeration of 2-subsets)."""
    N, K = TILE, 2 * TILE
    rng = np.random.default_rng(b)
    choice = rng.integers(0, 2, (N // b, K // b))
    ids = rng.integers(0, 6, (N, K // 4))
    tl = np.zeros((N // b, K // b, 2), np.float32)
    tl[..., 0] = 1.0 - choice
    tl[..., 1] = choice
    pl = np.zeros((N, K // 4, 6), np.float32)
    np.put_along_axis(pl, ids[..., None], 1.0, axis=2)
    w = np.full((N, K), ONE, np.uint16)
    wm, bm, pid = oracle.hard_mask_tiles(w, tl, pl, b)
    assert np.array_equal(bm, choice.astype(np.uint8))
    assert np.array_equal(pid, ids.astype(np.uint8))
    for n in range(0, N, 7):
        for g in range(0, K // 4, 3):
            kept_pos = set(PAIRS[ids[n, g]]) if choice[n // b, (4 * g) // b] else {0, 1, 2, 3}
            row = wm[n, 4 * g:4 * g + 4]
            assert {i for i in range(4) if row[i] == ONE} == kept_pos
            assert all(row[i] == 0 for i in range(4) if i not in kept_pos)


@pytest.mark.parametrize("b", MASK_TILES)
def test_mask_tiles_global_sparsity_is_half_the_sparse_tile_fraction(b):
    N, K = TILE, 2 * TILE
    w = np.full((N, K), ONE, np.uint16)
    rng = np.random.default_rng(100 + b)
    tl = rng.standard_normal((N // b, K // b, 2)).astype(np.float32)
    pl = rng.standard_normal((N, K // 4, 6)).astype(np.float32)
    wm, bm, _ = oracle.hard_mask_tiles(w, tl, pl, b)
    pruned = np.count_nonzero(wm == 0)
    assert pruned * bm.size == N * K * int(bm.sum()) // 2  # pruned/NK == 0.5 * sparse tiles / tiles
    groups = (wm.reshape(N, K // 4, 4) == ONE).sum(axis=2)
    sparse_group = np.repeat(np.repeat(bm, b, axis=0), b // 4, axis=1)  # [N][K/4]: is the group's tile sparse
    assert np.all(groups[sparse_group == 1] == 2) and np.all(groups[sparse_group == 0] == 4)


def test_exec_tiles_all_sixteen_combinations_of_four_64_tiles():
    """A 128 x 128 execution tile holding four 64 x 64 mask tiles is sparse only
    in the one combination where all four are sparse."""
    for combo in range(16):
        bm = np.array([[combo & 1, (combo >> 1) & 1], [(combo >> 2) & 1, (combo >> 3) & 1]], np.uint8)
        ex, n = oracle.exec_tiles(bm, TILE, TILE, 64)
        assert ex.tolist() == [[1 if combo == 15 else 0]] and n == (1 if combo == 15 else 0)


def test_exec_tiles_single_dense_4x4_tile_anywhere_makes_the_tile_dense():
    N, K, b = 2 * TILE, 2 * TILE, 4
    r = TILE // b
    for (i, j) in [(0, 0), (r - 1, r - 1), (r // 2, 3), (r, r), (2 * r - 1, 0)]:
        bm = np.ones((N // b, K // b), np.uint8)
        bm[i, j] = 0
        ex, n = oracle.exec_tiles(bm, N, K, b)
        want = np.ones((2, 2), np.uint8)
        want[i // r, j // r] = 0
        assert np.array_equal(ex, want) and n == 3


def test_exec_tiles_at_128_copy_the_bitmap():
    bm = np.random.default_rng(7).integers(0, 2, (3, 5)).astype(np.uint8)
    ex, n = oracle.exec_tiles(bm, 3 * TILE, 5 * TILE, 128)
    assert np.array_equal(ex, bm) and n == int(bm.sum())


@pytest.mark.parametrize("b", [4, 32, 64])
def test_fine_mask_packs_and_multiplies_as_the_masked_weight(b):
    """Packing W_masked with the execution bitmap loses nothing: the blobs unpack
    to W_masked bit for bit (dense execution tiles carry the pruned zeros), and
    the GEMM on them equals numpy's fp64 matmul of W_masked."""
    N, K, M = 2 * TILE, 2 * TILE, 3
    w = si.gen_w(N, K, 7, b)
    rng = np.random.default_rng(b)
    # mostly-sparse mask tiles, so that some execution tiles come out sparse
    tl = np.zeros((N // b, K // b, 2), np.float32)
    tl[..., 1] = 1.0
    tl[: N // (2 * b), : K // (2 * b), 1] = rng.choice([1.0, -1.0], (N // (2 * b), K // (2 * b)))
    pl = rng.standard_normal((N, K // 4, 6)).astype(np.float32)
    wm, bm, pid = oracle.hard_mask_tiles(w, tl, pl, b)
    ex, ns = oracle.exec_tiles(bm, N, K, b)
    assert 1 <= ns < ex.size
    v, m, d = oracle.pack(wm, ex, pid)
    assert np.array_equal(oracle.unpack(v, m, d, N, K), wm)
    x = si.gen_x(M, K, 7, b)
    y = oracle.gemm(x, oracle.unpack(v, m, d, N, K))
    assert np.allclose(y, f64(x) @ f64(wm).T, rtol=1e-12, atol=1e-12)


# ---- 64 x 64 execution tiles ("Ablation Studies", tile size): the second packed format

T64 = 64


def spec_values_blob64(w, bm, ids, offs):
    """The 64 x 64 values blob, restated from the format text: a dense tile is
    2 panels (k 0..31, then 32..63) of 64 rows x 32 values with 64-byte rows;
    a sparse tile one panel whose row r holds group g's kept pair at 2g, 2g+1."""
    N, K = w.shape
    Tn, Tk = N // T64, K // T64
    size = sum(8192 if not bm[t // Tk, t % Tk] else 4096 for t in range(Tn * Tk))
    blob = np.zeros(size // 2, np.uint16)
    for tn in range(Tn):
        for tk in range(Tk):
            o = int(offs[tn * Tk + tk]) // 2
            tile = w[tn * T64:(tn + 1) * T64, tk * T64:(tk + 1) * T64]
            if not bm[tn, tk]:
                for h in range(2):
                    blob[o + 2048 * h:o + 2048 * (h + 1)] = tile[:, 32 * h:32 * (h + 1)].reshape(-1)
            else:
                for r in range(T64):
                    for g in range(16):
                        a, b = PAIRS[ids[tn * T64 + r, tk * 16 + g]]
                        blob[o + r * 32 + 2 * g] = tile[r, 4 * g + a]
                        blob[o + r * 32 + 2 * g + 1] = tile[r, 4 * g + b]
    return blob.view(np.uint8)


def test_pack64_values_blob_against_the_format_text():
    N, K = 2 * T64, 3 * T64
    w = np.arange(N * K, dtype=np.uint32).astype(np.uint16).reshape(N, K)  # distinct bit patterns
    assert len(np.unique(w)) == N * K
    ids = np.random.default_rng(17).integers(0, 6, size=(N, K // 4)).astype(np.uint8)
    for bm in (np.array([[0, 1, 0], [1, 0, 1]], np.uint8), np.array([[1, 1, 0], [0, 0, 1]], np.uint8),
               np.zeros((2, 3), np.uint8), np.ones((2, 3), np.uint8)):
        values, meta, desc = oracle.pack64(w, bm, ids)
        d = desc.reshape(-1, 16)
        kinds = d[:, 0:4].copy().view("<u4").ravel()
        ords = d[:, 4:8].copy().view("<u4").ravel()
        offs = d[:, 8:16].copy().view("<u8").ravel()
        assert np.array_equal(kinds, bm.ravel())
        sizes = np.where(bm.ravel() == 1, 4096, 8192)
        assert np.array_equal(offs, np.concatenate([[0], np.cumsum(sizes)[:-1]]))
        assert np.array_equal(ords[bm.ravel() == 1], np.arange(int(bm.sum())))
        assert np.all(ords[bm.ravel() == 0] == 0xFFFFFFFF)
        assert values.size == int(sizes.sum()) and meta.size == 512 * int(bm.sum())
        assert np.array_equal(values, spec_values_blob64(w, bm, ids, offs)), bm.tolist()
    # bytes spelled out for bm [[0,1,0],[1,0,1]]: dense tile (0,0), panel 1, row 3, value 5 is W[3][32+5]
    bm = np.array([[0, 1, 0], [1, 0, 1]], np.uint8)
    values, _, _ = oracle.pack64(w, bm, ids)
    v16 = values.view(np.uint16)
    assert v16[(4096 + 3 * 64 + 5 * 2) // 2] == w[3, 37]
    # sparse tile (0,1) starts after the 8 KiB dense tile; row 7, group 9 keeps PAIRS[id]
    a, b = PAIRS[ids[7, 16 + 9]]
    assert v16[(8192 + 7 * 64 + 9 * 4) // 2] == w[7, 64 + 36 + a]
    assert v16[(8192 + 7 * 64 + 9 * 4 + 2) // 2] == w[7, 64 + 36 + b]


def hw_meta64_position(r, g):
    """Byte and nibble of group g of row r in a 64 x 64 tile's metadata block,
    restated from where the 16-bit sparse MMA with M = 64 reads it in tensor
    memory: lane = r%8 + 8*((k//16)%2) + 32*(r//16) (the first 16 lanes of each
    32-lane subpartition), 32-bit column = k//32, byte in column =
    (k%16)//8 + 2*((r//8)%2), nibble = (k//4)%2, with k = 4g; the block stores
    the two columns of lane L at bytes 128*(L//32) + 8*(L%32) .. +7 (a 32-lane,
    2-column store per subpartition moves it without reshuffling)."""
    k = 4 * g
    lane = r % 8 + 8 * ((k // 16) % 2) + 32 * (r // 16)
    col = k // 32
    byte = (k % 16) // 8 + 2 * ((r // 8) % 2)
    return 128 * (lane // 32) + 8 * (lane % 32) + 4 * col + byte, (k // 4) % 2


def test_metadata64_layout_positions():
    w = np.full((T64, T64), ONE, np.uint16)
    bm = np.ones((1, 1), np.uint8)
    seen = set()
    for r in range(T64):
        for g in range(16):
            ids = np.zeros((T64, T64 // 4), np.uint8)  # code 0x4 everywhere
            ids[r, g] = 5                               # code 0xE at one group
            _, meta, _ = oracle.pack64(w, bm, ids)
            byte, nib = hw_meta64_position(r, g)
            assert (meta[byte] >> (4 * nib)) & 0xF == 0xE
            others = meta.copy()
            others[byte] &= ~np.uint8(0xF << (4 * nib))
            others[byte] |= np.uint8(0x4 << (4 * nib))
            assert np.all(others == 0x44)
            seen.add((byte, nib))
    assert len(seen) == 1024  # a bijection onto the 512 bytes x 2 nibbles


def test_pattern_codes64_against_golden():
    w = np.full((T64, T64), ONE, np.uint16)
    bm = np.ones((1, 1), np.uint8)
    for pid, a, b, code in golden_codes():
        _, meta, _ = oracle.pack64(w, bm, np.full((T64, T64 // 4), pid, np.uint8))
        assert meta.size == 512 and np.all(meta == (code | (code << 4)))


def test_pack64_sizes_follow_the_blobs():
    for N, K, ns in ((64, 64, 0), (64, 64, 1), (192, 320, 7), (4096, 4096, 2048)):
        v, m, d = oracle.pack64_sizes(N, K, ns)
        T = (N // 64) * (K // 64)
        assert (v, m, d) == ((T - ns) * 2 * 4096 + ns * 4096, ns * 512, 16 * T)


@pytest.mark.parametrize("frac", [0.0, 0.3, 1.0])
def test_pack64_unpack64_round_trip(frac):
    N, K = 3 * T64, 5 * T64
    w = si.gen_w(N, K, 3, int(frac * 10))
    rng = np.random.default_rng(int(frac * 10))
    bm = (rng.random((N // T64, K // T64)) < frac).astype(np.uint8)
    ids = rng.integers(0, 6, (N, K // 4)).astype(np.uint8)
    v, m, d = oracle.pack64(w, bm, ids)
    wm = oracle.apply_mask_tiles(w, bm, ids, 64)
    assert np.array_equal(oracle.unpack64(v, m, d, N, K), wm)
    # packing the already-masked weight gives the same blobs (pruned values are never stored)
    v2, m2, d2 = oracle.pack64(wm, bm, ids)
    assert np.array_equal(v, v2) and np.array_equal(m, m2) and np.array_equal(d, d2)


def test_apply_mask_tiles_at_128_is_apply_mask_and_agrees_with_hard_mask_tiles():
    N, K = 2 * TILE, 2 * TILE
    w = si.gen_w(N, K, 4, 2)
    rng = np.random.default_rng(21)
    ids = rng.integers(0, 6, (N, K // 4)).astype(np.uint8)
    bm = rng.integers(0, 2, (N // TILE, K // TILE)).astype(np.uint8)
    assert np.array_equal(oracle.apply_mask_tiles(w, bm, ids, 128), oracle.apply_mask(w, bm, ids))
    for b in (4, 16, 64):
        tl = rng.standard_normal((N // b, K // b, 2)).astype(np.float32)
        pl = rng.standard_normal((N, K // 4, 6)).astype(np.float32)
        wm, bmb, pid = oracle.hard_mask_tiles(w, tl, pl, b)
        assert np.array_equal(oracle.apply_mask_tiles(w, bmb, pid, b), wm)


def test_exec_tiles_e_at_128_is_exec_tiles():
    rng = np.random.default_rng(5)
    for b in MASK_TILES:
        bm = (rng.random((2 * TILE // b, 3 * TILE // b)) < 0.9).astype(np.uint8)
        ex, n = oracle.exec_tiles_e(bm, 2 * TILE, 3 * TILE, b, 128)
        ex0, n0 = oracle.exec_tiles(bm, 2 * TILE, 3 * TILE, b)
        assert np.array_equal(ex, ex0) and n == n0


@pytest.mark.parametrize("b", [4, 8, 16, 32, 64])
def test_exec_tiles64_is_all_of_its_mask_tiles(b):
    """Brute force with numpy: the 64 x 64 execution tile is sparse iff all of
    its (64/b)^2 mask tiles are; at b = 64 it is the bitmap itself."""
    N, K = 3 * T64, 2 * T64
    rng = np.random.default_rng(40 + b)
    bm = (rng.random((N // b, K // b)) < 0.85).astype(np.uint8)
    r = T64 // b
    want = bm.reshape(N // T64, r, K // T64, r).all(axis=(1, 3)).astype(np.uint8)
    ex, n = oracle.exec_tiles_e(bm, N, K, b, 64)
    assert np.array_equal(ex, want) and n == int(want.sum())
    if b == 64:
        assert np.array_equal(ex, bm)


def test_exec_tiles64_with_one_dense_4x4_tile():
    N = K = 2 * T64
    r = T64 // 4
    for (i, j) in [(0, 0), (r - 1, r), (2 * r - 1, 2 * r - 1)]:
        bm = np.ones((N // 4, K // 4), np.uint8)
        bm[i, j] = 0
        ex, n = oracle.exec_tiles_e(bm, N, K, 4, 64)
        want = np.ones((2, 2), np.uint8)
        want[i // r, j // r] = 0
        assert np.array_equal(ex, want) and n == 3


def test_gemm64_all_dense_and_all_sparse_are_numpy_matmuls():
    """All-dense 64-tiles multiply as numpy's dense matmul; all-sparse ones as
    numpy's matmul of W with the 2:4 keep-mask built from the itertools pairs."""
    N, K, M = 2 * T64, 3 * T64, 5
    w = si.gen_w(N, K, 6, 0)
    x = si.gen_x(M, K, 6, 0)
    ids = np.random.default_rng(9).integers(0, 6, (N, K // 4)).astype(np.uint8)
    v, m, d = oracle.pack64(w, np.zeros((N // T64, K // T64), np.uint8), ids)
    assert np.allclose(oracle.gemm(x, oracle.unpack64(v, m, d, N, K)), f64(x) @ f64(w).T, rtol=1e-12, atol=1e-12)
    v, m, d = oracle.pack64(w, np.ones((N // T64, K // T64), np.uint8), ids)
    pos = np.arange(K) % 4
    a = np.array([[PAIRS[i][0] for i in row] for row in ids]).repeat(4, axis=1)
    b = np.array([[PAIRS[i][1] for i in row] for row in ids]).repeat(4, axis=1)
    keep = (pos[None, :] == a) | (pos[None, :] == b)
    w24 = np.where(keep, f64(w), 0.0)
    y = oracle.gemm(x, oracle.unpack64(v, m, d, N, K))
    assert np.allclose(y, f64(x) @ w24.T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("b", [4, 32, 64])
def test_fine_mask_packs64_as_the_masked_weight(b):
    """At b <= 64 the 64 x 64 format keeps every all-sparse 64-tile sparse
    (at b = 64, every sparse mask tile) and still unpacks to W_masked."""
    N, K = 2 * TILE, 2 * TILE
    w = si.gen_w(N, K, 8, b)
    rng = np.random.default_rng(60 + b)
    tl = np.zeros((N // b, K // b, 2), np.float32)
    tl[..., 1] = 1.0
    tl[: N // (2 * b), : K // (2 * b), 1] = rng.choice([1.0, -1.0], (N // (2 * b), K // (2 * b)))
    pl = rng.standard_normal((N, K // 4, 6)).astype(np.float32)
    wm, bm, pid = oracle.hard_mask_tiles(w, tl, pl, b)
    ex, ns = oracle.exec_tiles_e(bm, N, K, b, 64)
    ex128, ns128 = oracle.exec_tiles(bm, N, K, b)
    assert ns >= 4 * ns128  # a sparse 128-tile is four sparse 64-tiles
    if b == 64:
        assert ns == int(bm.sum())
    v, m, d = oracle.pack64(wm, ex, pid)
    assert np.array_equal(oracle.unpack64(v, m, d, N, K), wm)
