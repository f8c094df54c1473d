"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

hard mask and pack are compared byte for byte; the GEMM against the fp64
oracle with the layer's tolerance (relative Frobenius error <= 5e-3 and
|err| <= 1e-2 * (1 + |ref|) elementwise).  Sizes here run in seconds on the
oracle and still span several tiles, ragged token counts and the degenerate
all-dense / all-sparse bitmaps; the full-size workloads are in
test_gpu_full_size.py.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import tile_sparse_gemm_b200 as tsg
from _util import bits_of, check_gemm, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu
TILE = 128


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert torch.cuda.get_device_capability()[0] == 10, "GPU tests need an sm_100 device"
    tsg.lib()  # fails loudly when libpatch.so is missing


def pack_on_gpu(w, bm, ids):
    status = tsg.new_status()
    pw = tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids), int(bm.sum()), status=status)
    code, bits = tsg.patch_read_status(status)
    assert code == 0, (code, bits)
    return pw


def gemm_on_gpu(x, pw, path=tsg.PATH_AUTO):
    status = tsg.new_status()
    y = tsg.patch_gemm_ex(to_dev_bf16(x), pw, status=status, path=path)
    code, bits = tsg.patch_read_status(status)
    assert code == 0, (code, bits)
    return bits_of(y)


# ------------------------------------------------------------- hard mask


@pytest.mark.parametrize("N,K,cfg", [(512, 512, 1), (128, 128, 0), (384, 640, 7), (1024, 256, 8)])
def test_hard_mask_bit_exact(N, K, cfg):
    w = si.gen_w(N, K, cfg, 0)
    tl = si.gen_tile_logits(N, K, cfg, 0)
    pl = si.gen_pattern_logits(N, K, cfg, 0)
    wm_ref, bm_ref, id_ref = oracle.hard_mask(w, tl, pl)
    status = tsg.new_status()
    wm, bm, ids = tsg.patch_hard_mask(to_dev_bf16(w), to_dev(tl), to_dev(pl), status=status)
    assert tsg.patch_read_status(status)[0] == 0
    assert np.array_equal(bm.cpu().numpy(), bm_ref)
    assert np.array_equal(ids.cpu().numpy(), id_ref)
    assert np.array_equal(bits_of(wm), wm_ref)


def test_hard_mask_ties_nan_and_negative_weights():
    N = K = 256
    w = np.full((N, K), np.uint16(0xBF80), np.uint16)  # -1.0 everywhere
    tl = np.array([[[0.0, 0.0], [0.0, 1.0]], [[np.nan, 1.0], [1.0, np.nan]]], np.float32)
    rng = np.random.default_rng(0)
    pl = rng.integers(-2, 3, (N, K // 4, 6)).astype(np.float32)  # many ties
    pl[::7, ::5, 3] = np.nan
    pl[::11, ::3, 0] = np.nan
    wm_ref, bm_ref, id_ref = oracle.hard_mask(w, tl, pl)
    wm, bm, ids = tsg.patch_hard_mask(to_dev_bf16(w), to_dev(tl), to_dev(pl))
    assert np.array_equal(bm.cpu().numpy(), bm_ref)
    assert np.array_equal(ids.cpu().numpy(), id_ref)
    assert np.array_equal(bits_of(wm), wm_ref)
    assert bm_ref.tolist() == [[0, 1], [0, 0]]


def test_hard_mask_without_masked_output():
    N, K = 256, 384
    tl = si.gen_tile_logits(N, K, 2, 0)
    pl = si.gen_pattern_logits(N, K, 2, 0)
    _, bm_ref, id_ref = oracle.hard_mask(si.gen_w(N, K, 2, 0), tl, pl)
    wm, bm, ids = tsg.patch_hard_mask(None, to_dev(tl), to_dev(pl), want_masked=False)
    assert wm is None
    assert np.array_equal(bm.cpu().numpy(), bm_ref) and np.array_equal(ids.cpu().numpy(), id_ref)


# ------------------------------------------------------------------ pack


@pytest.mark.parametrize("N,K,kind,frac", [
    (512, 512, "bernoulli", 0.5), (128, 128, "exact", 1.0), (128, 128, "exact", 0.0),
    (384, 640, "exact", 0.5), (640, 384, "clustered", 0.5), (256, 1024, "exact", 0.25)])
def test_pack_bit_exact(N, K, kind, frac):
    w = si.gen_w(N, K, 1, 3)
    bm = {"bernoulli": si.tiles_bernoulli, "exact": si.tiles_exact, "clustered": si.tiles_clustered}[kind](
        N, K, frac, 1, 3)
    ids = si.patterns_top2(w)
    v_ref, m_ref, d_ref = oracle.pack(w, bm, ids)
    pw = pack_on_gpu(w, bm, ids)
    assert np.array_equal(pw.desc.cpu().numpy(), d_ref)
    assert np.array_equal(pw.values.cpu().numpy(), v_ref)
    assert np.array_equal(pw.meta.cpu().numpy(), m_ref)


def test_pack_of_masked_and_random_patterns():
    N, K = 384, 384
    w = si.gen_w(N, K, 5, 0)
    bm = si.tiles_exact(N, K, 0.5, 5, 0)
    ids = np.random.default_rng(9).integers(0, 6, (N, K // 4)).astype(np.uint8)
    v_ref, m_ref, d_ref = oracle.pack(w, bm, ids)
    pw = pack_on_gpu(oracle.apply_mask(w, bm, ids), bm, ids)
    assert np.array_equal(pw.values.cpu().numpy(), v_ref)
    assert np.array_equal(pw.meta.cpu().numpy(), m_ref)
    assert np.array_equal(pw.desc.cpu().numpy(), d_ref)


# ------------------------------------------------- soft (training-time) mask


def _bf16_close(gpu_bits, ref_bits):
    """Equal up to one bf16 rounding step (the GPU multiplies in fp32, the oracle in fp64)."""
    from _util import bf16_to_f64
    g, r = bf16_to_f64(gpu_bits), bf16_to_f64(ref_bits)
    return np.all(np.abs(g - r) <= np.abs(r) * 2.0 ** -7 + 1e-30)


@pytest.mark.parametrize("tau", [0.5, 2.0])
@pytest.mark.parametrize("N,K", [(256, 384), (128, 128)])
def test_soft_mask_matches_oracle(N, K, tau):
    w = si.gen_w(N, K, 13, 0)
    tl = si.gen_tile_logits(N, K, 13, 0)
    pl = si.gen_pattern_logits(N, K, 13, 0)
    rng = np.random.default_rng(13)
    tg = rng.gumbel(size=tl.shape).astype(np.float32)
    pg = rng.gumbel(size=pl.shape).astype(np.float32)
    ws_ref, m_ref = oracle.soft_mask(w, tl, pl, tau, tg, pg)
    ws, m = tsg.patch_soft_mask(to_dev_bf16(w), to_dev(tl), to_dev(pl), tau, to_dev(tg), to_dev(pg))
    m = m.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(m - m_ref) <= 2e-6 + 1e-5 * np.abs(m_ref))
    assert _bf16_close(bits_of(ws), ws_ref)
    # without noise and without the mask output
    ws_ref0, _ = oracle.soft_mask(w, tl, pl, tau)
    ws0, none = tsg.patch_soft_mask(to_dev_bf16(w), to_dev(tl), to_dev(pl), tau, want_mask=False)
    assert none is None and _bf16_close(bits_of(ws0), ws_ref0)


def test_soft_mask_cold_limit_is_the_hard_mask():
    N, K = 256, 256
    w = si.gen_w(N, K, 14, 0)
    rng = np.random.default_rng(14)
    tl = (np.argsort(rng.random((N // TILE, K // TILE, 2)), axis=-1) - 1.0).astype(np.float32)
    pl = (np.argsort(rng.random((N, K // 4, 6)), axis=-1) - 3.0).astype(np.float32)
    wm_ref, _, _ = oracle.hard_mask(w, tl, pl)
    ws, m = tsg.patch_soft_mask(to_dev_bf16(w), to_dev(tl), to_dev(pl), 1e-3)
    b = bits_of(ws)
    assert np.array_equal(np.where(b == 0x8000, np.uint16(0), b), wm_ref)
    mm = m.cpu().numpy()
    assert np.all((mm == 0.0) | (mm == 1.0))


def test_soft_mask_rejects_bad_temperature():
    N = K = 128
    w = to_dev_bf16(si.gen_w(N, K, 1, 0))
    tl, pl = to_dev(si.gen_tile_logits(N, K, 1, 0)), to_dev(si.gen_pattern_logits(N, K, 1, 0))
    for tau in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(tsg.PatchError):
            tsg.patch_soft_mask(w, tl, pl, tau)


# ------------------------------------------------- fused hard mask -> pack


@pytest.mark.parametrize("N,K,cfg", [(512, 512, 1), (128, 128, 0), (384, 640, 7), (1024, 256, 8)])
def test_tile_kinds_and_pack_from_logits_bit_exact(N, K, cfg):
    """Tile kinds from the tile logits and a pack that takes each sparse tile's
    pattern ids as the argmax of its pattern logits: the oracle's hard mask
    followed by its pack, byte for byte, without the masked W or the ids."""
    w = si.gen_w(N, K, cfg, 1)
    tl = si.gen_tile_logits(N, K, cfg, 1)
    pl = si.gen_pattern_logits(N, K, cfg, 1)
    _, bm_ref, id_ref = oracle.hard_mask(w, tl, pl)
    v_ref, m_ref, d_ref = oracle.pack(w, bm_ref, id_ref)
    bitmap, n_dev = tsg.patch_tile_kinds(to_dev(tl))
    assert np.array_equal(bitmap.cpu().numpy(), bm_ref)
    assert int(n_dev.item()) == int(bm_ref.sum())
    status = tsg.new_status()
    pw = tsg.patch_pack_from_logits(to_dev_bf16(w), bitmap, to_dev(pl), int(n_dev.item()), status=status)
    assert tsg.patch_read_status(status)[0] == 0
    assert np.array_equal(pw.desc.cpu().numpy(), d_ref)
    assert np.array_equal(pw.values.cpu().numpy(), v_ref)
    assert np.array_equal(pw.meta.cpu().numpy(), m_ref)


def test_pack_from_logits_ties_and_nan_match_the_hard_mask():
    N = K = 256
    w = si.gen_w(N, K, 6, 0)
    tl = np.array([[[0.0, 0.0], [0.0, 1.0]], [[np.nan, 1.0], [-1.0, 2.0]]], np.float32)
    rng = np.random.default_rng(3)
    pl = rng.integers(-2, 3, (N, K // 4, 6)).astype(np.float32)  # many ties
    pl[::7, ::5, 3] = np.nan
    pl[::11, ::3, 0] = np.nan
    _, bm_ref, id_ref = oracle.hard_mask(w, tl, pl)
    v_ref, m_ref, d_ref = oracle.pack(w, bm_ref, id_ref)
    bitmap, n_dev = tsg.patch_tile_kinds(to_dev(tl))
    pw = tsg.patch_pack_from_logits(to_dev_bf16(w), bitmap, to_dev(pl), int(n_dev.item()))
    assert bm_ref.tolist() == [[0, 1], [0, 1]]
    assert np.array_equal(pw.values.cpu().numpy(), v_ref)
    assert np.array_equal(pw.meta.cpu().numpy(), m_ref)
    assert np.array_equal(pw.desc.cpu().numpy(), d_ref)


def test_fused_and_two_step_mask_pack_agree_and_multiply_alike():
    """hard mask -> pack and tile kinds -> pack-from-logits give the same blobs,
    and a GEMM on them matches the oracle."""
    N, K, M = 384, 512, 8
    w = si.gen_w(N, K, 9, 2)
    tl = si.gen_tile_logits(N, K, 9, 2)
    pl = si.gen_pattern_logits(N, K, 9, 2)
    _, bm2, ids2 = tsg.patch_hard_mask(to_dev_bf16(w), to_dev(tl), to_dev(pl), want_masked=False)
    two = tsg.patch_pack(to_dev_bf16(w), bm2, ids2)
    bitmap, n_dev = tsg.patch_tile_kinds(to_dev(tl))
    one = tsg.patch_pack_from_logits(to_dev_bf16(w), bitmap, to_dev(pl), int(n_dev.item()))
    for a, b in ((one.values, two.values), (one.meta, two.meta), (one.desc, two.desc)):
        assert torch.equal(a, b)
    x = si.gen_x(M, K, 9, 2)
    _, bm_ref, id_ref = oracle.hard_mask(w, tl, pl)
    check_gemm(gemm_on_gpu(x, one), oracle.hybrid_gemm(x, w, bm_ref, id_ref), "fused mask-pack GEMM")


def test_pack_from_logits_count_mismatch_flagged_without_overrun():
    import ctypes
    N = K = 256
    w = si.gen_w(N, K, 4, 0)
    pl = si.gen_pattern_logits(N, K, 4, 0)
    bm = np.array([[1, 1], [0, 1]], np.uint8)  # 3 sparse tiles
    vb, mb, db = tsg.patch_pack_sizes(N, K, 2)
    guard = 4096
    values = torch.full((vb + guard,), 0xAB, dtype=torch.uint8, device="cuda")
    meta = torch.full((mb + guard,), 0xCD, dtype=torch.uint8, device="cuda")
    desc = torch.zeros(db, dtype=torch.uint8, device="cuda")
    status = tsg.new_status()
    rc = tsg.lib().patch_pack_from_logits(
        ctypes.c_void_p(to_dev_bf16(w).data_ptr()), N, K, ctypes.c_void_p(to_dev(bm).data_ptr()),
        ctypes.c_void_p(to_dev(pl).data_ptr()), 2, ctypes.c_void_p(values.data_ptr()),
        ctypes.c_void_p(meta.data_ptr()), ctypes.c_void_p(desc.data_ptr()), ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    code, bits = tsg.patch_read_status(status)
    assert code == 9 and bits & tsg.DEV_COUNT
    assert torch.all(values[vb:] == 0xAB) and torch.all(meta[mb:] == 0xCD)


def test_pack_flags_bad_pattern_id():
    N = K = 256
    w = si.gen_w(N, K, 6, 0)
    bm = np.array([[1, 0], [0, 1]], np.uint8)
    ids = si.patterns_top2(w)
    ids[3, 5] = 9   # inside sparse tile (0, 0)
    ids[3, 40] = 7  # inside dense tile (0, 1): never read
    status = tsg.new_status()
    tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids), 2, status=status)
    code, bits = tsg.patch_read_status(status)
    assert code == 6 and bits == tsg.DEV_BAD_PATTERN


def test_pack_flags_count_mismatch_without_overrun():
    N = K = 256
    w = si.gen_w(N, K, 6, 1)
    bm = np.array([[1, 1], [0, 1]], np.uint8)  # 3 sparse tiles
    ids = si.patterns_top2(w)
    vb, mb, db = tsg.patch_pack_sizes(N, K, 1)
    guard = 4096
    values = torch.full((vb + guard,), 0xAB, dtype=torch.uint8, device="cuda")
    meta = torch.full((mb + guard,), 0xCD, dtype=torch.uint8, device="cuda")
    desc = torch.zeros(db, dtype=torch.uint8, device="cuda")
    status = tsg.new_status()
    import ctypes
    rc = tsg.lib().patch_pack(ctypes.c_void_p(to_dev_bf16(w).data_ptr()), N, K,
                              ctypes.c_void_p(to_dev(bm).data_ptr()), ctypes.c_void_p(to_dev(ids).data_ptr()),
                              1, ctypes.c_void_p(values.data_ptr()), ctypes.c_void_p(meta.data_ptr()),
                              ctypes.c_void_p(desc.data_ptr()), ctypes.c_void_p(status.data_ptr()),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    code, bits = tsg.patch_read_status(status)
    assert code == 9 and bits & tsg.DEV_COUNT
    assert torch.all(values[vb:] == 0xAB) and torch.all(meta[mb:] == 0xCD)


def test_gpu_pack_then_hard_mask_chain():
    """hard mask -> pack on the GPU equals the oracle's chain."""
    N, K = 512, 512
    w = si.gen_w(N, K, 1, 0)
    tl, pl = si.gen_tile_logits(N, K, 1, 0), si.gen_pattern_logits(N, K, 1, 0)
    wm_ref, bm_ref, id_ref = oracle.hard_mask(w, tl, pl)
    v_ref, m_ref, d_ref = oracle.pack(w, bm_ref, id_ref)
    wm, bm, ids = tsg.patch_hard_mask(to_dev_bf16(w), to_dev(tl), to_dev(pl))
    pw = tsg.patch_pack(wm, bm, ids)
    assert np.array_equal(pw.values.cpu().numpy(), v_ref)
    assert np.array_equal(pw.meta.cpu().numpy(), m_ref)
    assert np.array_equal(pw.desc.cpu().numpy(), d_ref)


# ------------------------------------------------------------------ GEMM


def _layer(N, K, M, kind, frac, cfg=3, shape_idx=0):
    x = si.gen_x(M, K, cfg, shape_idx)
    w = si.gen_w(N, K, cfg, shape_idx)
    if kind == "bernoulli":
        bm = si.tiles_bernoulli(N, K, frac, cfg, shape_idx)
    elif kind == "clustered":
        bm = si.tiles_clustered(N, K, frac, cfg, shape_idx)
    else:
        bm = si.tiles_exact(N, K, frac, cfg, shape_idx)
    return x, w, bm, si.patterns_top2(w)


def test_gemm_512x512_bernoulli_tiles_m16():
    """512 x 512 weight, Bernoulli(0.5) tiles, M = 16 tokens."""
    x, w, bm, ids = _layer(512, 512, 16, "bernoulli", 0.5, cfg=1)
    ref = oracle.hybrid_gemm(x, w, bm, ids)
    y = gemm_on_gpu(x, pack_on_gpu(w, bm, ids))
    check_gemm(y, ref, "512 x 512, Bernoulli(0.5) tiles, M = 16")


@pytest.mark.parametrize("path", [tsg.PATH_DECODE, tsg.PATH_DECODE_SIMT])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 7, 8, 13, 16])
@pytest.mark.parametrize("N,K,frac", [(384, 640, 0.5), (256, 1280, 0.0), (640, 256, 1.0)])
def test_gemm_decode_parity(M, N, K, frac, path):
    x, w, bm, ids = _layer(N, K, M, "exact", frac, shape_idx=M)
    ref = oracle.hybrid_gemm(x, w, bm, ids)
    y = gemm_on_gpu(x, pack_on_gpu(w, bm, ids), path)
    check_gemm(y, ref, f"decode path {path} M={M} {N}x{K} f={frac}")


@pytest.mark.parametrize("N,K,frac,kind", [
    (128, 128, 1.0, "exact"),        # 1 panel: most CTAs idle
    (128, 896, 0.5, "clustered"),    # fewer panels than SMs
    (4864, 896, 0.5, "clustered"),   # many tile rows cut between CTAs
    (2048, 4096, 0.3, "bernoulli"),  # mixed kinds, rows longer than a CTA share
    (128, 16384, 0.5, "exact"),      # one tile row shared by every CTA
])
@pytest.mark.parametrize("M", [1, 16])
def test_stream_k_decode_cuts(N, K, frac, kind, M):
    """The stream-K split cuts tile rows anywhere; every cut must be summed exactly once."""
    x, w, bm, ids = _layer(N, K, M, kind, frac, cfg=12, shape_idx=N % 97)
    ref = oracle.hybrid_gemm(x, w, bm, ids)
    y = gemm_on_gpu(x, pack_on_gpu(w, bm, ids), tsg.PATH_DECODE)
    check_gemm(y, ref, f"stream-K {N}x{K} f={frac} M={M}")


@pytest.mark.parametrize("frac", [0.0, 1.0, 0.5])
@pytest.mark.parametrize("M", [17, 129, 256, 300])
def test_gemm_prefill_parity(M, frac):
    N, K = 384, 640
    x, w, bm, ids = _layer(N, K, M, "exact", frac, shape_idx=int(10 * frac))
    ref = oracle.hybrid_gemm(x, w, bm, ids)
    y = gemm_on_gpu(x, pack_on_gpu(w, bm, ids), tsg.PATH_PREFILL)
    check_gemm(y, ref, f"prefill M={M} f={frac}")


@pytest.mark.parametrize("M", [1, 5, 16])
def test_prefill_path_small_m_matches_decode(M):
    x, w, bm, ids = _layer(256, 512, M, "bernoulli", 0.5, cfg=4)
    pw = pack_on_gpu(w, bm, ids)
    ref = oracle.hybrid_gemm(x, w, bm, ids)
    yp = gemm_on_gpu(x, pw, tsg.PATH_PREFILL)
    yd = gemm_on_gpu(x, pw, tsg.PATH_DECODE)
    ys = gemm_on_gpu(x, pw, tsg.PATH_DECODE_SIMT)
    check_gemm(yp, ref, "prefill small M")
    check_gemm(yd, ref, "decode")
    check_gemm(ys, ref, "decode simt")


@pytest.mark.parametrize("N,K,M", [(384, 4096, 17), (384, 4096, 100), (384, 4096, 300), (1024, 4096, 200),
                                   (384, 5376, 50)])
def test_prefill_split_k_matches_oracle_and_whole_k(N, K, M):
    """Few units for the SMs: K is split across CTAs (3 tile rows: a pair with
    one row; ragged token tails; 42 K-tiles in parts of unequal length) and the
    last part of each block adds the parts.  A workspace too small for the
    partials runs whole-K units instead; both match the oracle."""
    x, w, bm, ids = _layer(N, K, M, "exact", 0.5, cfg=16, shape_idx=M % 7)
    pw = pack_on_gpu(w, bm, ids)
    ref = oracle.hybrid_gemm(x, w, bm, ids)
    need = tsg.patch_gemm_workspace_size(M, pw)
    assert need > 65536  # the split plan needs room for its partials
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for it in range(2):
        status = tsg.new_status()
        y = tsg.patch_gemm_ex(to_dev_bf16(x), pw, workspace=ws, status=status, path=tsg.PATH_PREFILL)
        assert tsg.patch_read_status(status)[0] == 0
        check_gemm(bits_of(y), ref, f"split-K prefill {N}x{K} M={M} call {it}")
        assert int(torch.count_nonzero(ws[:65536]).item()) == 0
    status = tsg.new_status()
    y = tsg.patch_gemm_ex(to_dev_bf16(x), pw, workspace=torch.zeros(16, dtype=torch.uint8, device="cuda"),
                          status=status, path=tsg.PATH_PREFILL)
    assert tsg.patch_read_status(status)[0] == 0
    check_gemm(bits_of(y), ref, f"whole-K prefill {N}x{K} M={M}")


def test_split_k_prefill_and_decode_share_one_workspace():
    N, K = 1024, 4096
    x, w, bm, ids = _layer(N, K, 96, "exact", 0.5, cfg=17)
    pw = pack_on_gpu(w, bm, ids)
    ws = torch.zeros(max(tsg.patch_gemm_workspace_size(M, pw) for M in (1, 16, 40, 96)), dtype=torch.uint8,
                     device="cuda")
    for M in (96, 16, 40, 1, 96, 7):
        status = tsg.new_status()
        y = tsg.patch_gemm(to_dev_bf16(x[:M]), pw, workspace=ws, status=status)
        assert tsg.patch_read_status(status)[0] == 0
        check_gemm(bits_of(y), oracle.hybrid_gemm(x[:M], w, bm, ids), f"M={M}")
        assert int(torch.count_nonzero(ws[:65536]).item()) == 0


def test_prefill_many_output_tiles():
    """More work units (row pairs x token blocks) than SMs: the persistent schedule wraps around."""
    N, K, M = 128 * 80, 256, 1100
    x, w, bm, ids = _layer(N, K, M, "exact", 0.5, cfg=5)
    rows = np.array([0, 1, 255, 256, 511, 700, 1023, 1099])
    ref = oracle.hybrid_gemm(x, w, bm, ids, rows=rows)
    y = gemm_on_gpu(x, pack_on_gpu(w, bm, ids), tsg.PATH_PREFILL)
    check_gemm(y[rows], ref, "prefill wrap")


@pytest.mark.parametrize("M", [1, 16, 40])
def test_fused_projection_is_a_gemm_on_row_concatenated_weights(M):
    """q|k|v (or gate|up) fused: one GEMM over the row-concatenated packed
    weight gives the concatenation of the separate layers' outputs."""
    K = 384
    parts = [(256, 0.5), (128, 0.0), (384, 1.0)]
    ws, bms, idss = [], [], []
    for j, (N, f) in enumerate(parts):
        w = si.gen_w(N, K, 11, j)
        ws.append(w)
        bms.append(si.tiles_exact(N, K, f, 11, j))
        idss.append(si.patterns_top2(w))
    x = si.gen_x(M, K, 11, 0)
    w_cat, bm_cat, ids_cat = np.concatenate(ws), np.concatenate(bms), np.concatenate(idss)
    y = gemm_on_gpu(x, pack_on_gpu(w_cat, bm_cat, ids_cat))
    check_gemm(y, oracle.hybrid_gemm(x, w_cat, bm_cat, ids_cat), f"fused projection M={M}")
    n0 = 0
    for w, bm, ids in zip(ws, bms, idss):
        check_gemm(y[:, n0:n0 + w.shape[0]], oracle.hybrid_gemm(x, w, bm, ids), "part")
        n0 += w.shape[0]


@pytest.mark.parametrize("M", [1, 7, 16, 17, 300, 1100])
@pytest.mark.parametrize("N,K", [(384, 640), (256, 256)])
def test_gated_mlp(M, N, K):
    """H = silu(X Wg^T) * (X Wu^T): decode path (two GEMMs + elementwise) for
    M <= 16, one prefill launch with the product in the epilogue above."""
    wg, wu = si.gen_w(N, K, 12, 0, std=0.05), si.gen_w(N, K, 12, 1, std=0.05)
    bmg, bmu = si.tiles_exact(N, K, 0.5, 12, 0), si.tiles_exact(N, K, 0.5, 12, 1)
    idg, idu = si.patterns_top2(wg), si.patterns_top2(wu)
    x = si.gen_x(M, K, 12, 2)
    rows = None if M <= 300 else np.array([0, 1, 239, 240, 700, 1099])
    ref = oracle.hybrid_mlp(x, (wg, bmg, idg), (wu, bmu, idu), rows=rows)
    status = tsg.new_status()
    h = tsg.patch_gemm_mlp(to_dev_bf16(x), pack_on_gpu(wg, bmg, idg), pack_on_gpu(wu, bmu, idu), status=status)
    code, bits = tsg.patch_read_status(status)
    assert code == 0, (code, bits)
    hb = bits_of(h)
    check_gemm(hb if rows is None else hb[rows], ref, f"gated MLP M={M}")


def test_gated_mlp_rejects_mismatched_weights():
    a = pack_on_gpu(si.gen_w(256, 256, 1, 0), np.zeros((2, 2), np.uint8), si.patterns_top2(si.gen_w(256, 256, 1, 0)))
    b = pack_on_gpu(si.gen_w(384, 256, 1, 1), np.zeros((3, 2), np.uint8), si.patterns_top2(si.gen_w(384, 256, 1, 1)))
    x = to_dev_bf16(si.gen_x(4, 256, 1, 0))
    with pytest.raises(ValueError):
        tsg.patch_gemm_mlp(x, a, b)
    import ctypes
    h = torch.empty((4, 256), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    status = tsg.new_status()
    sa, sb = a.struct(), b.struct()
    rc = tsg.lib().patch_gemm_mlp(ctypes.c_void_p(x.data_ptr()), 4, ctypes.byref(sa), ctypes.byref(sb),
                                  ctypes.c_void_p(h.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                  ctypes.c_void_p(status.data_ptr()),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 2  # PATCH_ERR_SHAPE, before any launch


def test_prefill_long_k_reads_descriptors_from_global():
    """More K-tiles per row than the kernel stages in shared memory (K > 16384),
    odd tile-row count (the last row pair has one row)."""
    N, K, M = 384, 128 * 130, 40
    x, w, bm, ids = _layer(N, K, M, "exact", 0.5, cfg=10)
    ref = oracle.hybrid_gemm(x, w, bm, ids)
    y = gemm_on_gpu(x, pack_on_gpu(w, bm, ids), tsg.PATH_PREFILL)
    check_gemm(y, ref, "prefill long K")


def test_gemm_all_sparse_equals_24_and_all_dense_equals_dense():
    N, K, M = 256, 256, 64
    x = si.gen_x(M, K, 9, 0)
    w = si.gen_w(N, K, 9, 0)
    ids = si.patterns_top2(w)
    for frac in (0.0, 1.0):
        bm = np.full((N // TILE, K // TILE), int(frac), np.uint8)
        pw = pack_on_gpu(w, bm, ids)
        xd = to_dev_bf16(x).float()
        w_eff = torch.from_numpy(oracle.apply_mask(w, bm, ids).view(np.int16)).view(torch.bfloat16).cuda().float()
        torch_ref = (xd @ w_eff.T).double().cpu().numpy()   # plain fp32 reference of the same op
        for path in (tsg.PATH_PREFILL, tsg.PATH_DECODE, tsg.PATH_DECODE_SIMT):
            if path != tsg.PATH_PREFILL:
                y = gemm_on_gpu(x[:16], pw, path)
                check_gemm(y, torch_ref[:16], f"decode f={frac}")
            else:
                y = gemm_on_gpu(x, pw, path)
                check_gemm(y, torch_ref, f"prefill f={frac}")


def test_decode_workspace_reused_across_calls():
    """The decode path leaves its workspace zero-filled, so back-to-back calls on
    one workspace keep finishing the rows cut between CTAs."""
    x, w, bm, ids = _layer(4864, 896, 16, "clustered", 0.5, cfg=12, shape_idx=5)
    pw = pack_on_gpu(w, bm, ids)
    ws = torch.zeros(tsg.patch_gemm_workspace_size(16, pw), dtype=torch.uint8, device="cuda")
    ref = oracle.hybrid_gemm(x, w, bm, ids)
    xd = to_dev_bf16(x)
    for it in range(4):
        status = tsg.new_status()
        y = tsg.patch_gemm(xd[: 16 - it], pw, workspace=ws, status=status)
        assert tsg.patch_read_status(status)[0] == 0
        check_gemm(bits_of(y), ref[: 16 - it], f"call {it}")


def test_one_workspace_serves_layers_paths_and_token_counts_in_any_order():
    """One zero-filled workspace of the largest size, shared by layers whose
    grids differ (a layer with fewer panels than CTAs, clustered and even
    ones), both decode paths, the gated MLP and every token count, in an
    interleaved order.  The tensor-core kernel's arrival counters live in a
    fixed region at the start that every call leaves zero; scratch written by
    one call (partial sums of another layout, the other path's split-K
    partials, the MLP's G and U) never lands there."""
    specs = [(128, 896, 0.5, "clustered"), (4864, 896, 0.5, "clustered"), (384, 640, 0.5, "exact")]
    layers = []
    for i, (N, K, frac, kind) in enumerate(specs):
        x, w, bm, ids = _layer(N, K, 16, kind, frac, cfg=14, shape_idx=i)
        layers.append((x, w, bm, ids, pack_on_gpu(w, bm, ids)))
    gate, up = layers[1][4], _layer(4864, 896, 16, "exact", 0.5, cfg=14, shape_idx=7)
    up_pw = pack_on_gpu(up[1], up[2], up[3])
    import ctypes
    b = ctypes.c_size_t()
    sg, su = gate.struct(), up_pw.struct()
    assert tsg.lib().patch_gemm_mlp_workspace_size(16, ctypes.byref(sg), ctypes.byref(su), ctypes.byref(b)) == 0
    need = max([b.value] + [tsg.patch_gemm_workspace_size(M, L[4]) for L in layers for M in (1, 7, 16)])
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    order = [(0, 16, tsg.PATH_AUTO), (1, 1, tsg.PATH_DECODE_SIMT), (2, 7, tsg.PATH_AUTO), ("mlp", 16, None),
             (0, 1, tsg.PATH_AUTO), (1, 16, tsg.PATH_AUTO), (2, 16, tsg.PATH_DECODE_SIMT), (1, 7, tsg.PATH_AUTO),
             (0, 7, tsg.PATH_DECODE_SIMT), (2, 1, tsg.PATH_AUTO)]
    for li, M, path in order:
        status = tsg.new_status()
        if li == "mlp":
            x = layers[1][0][:M]
            h = tsg.patch_gemm_mlp(to_dev_bf16(x), gate, up_pw, workspace=ws, status=status)
            assert tsg.patch_read_status(status)[0] == 0
            ref = oracle.hybrid_mlp(x, (layers[1][1], layers[1][2], layers[1][3]), up[1:4])
            check_gemm(bits_of(h), ref, "gated MLP on the shared workspace")
        else:
            x, w, bm, ids, pw = layers[li]
            y = tsg.patch_gemm_ex(to_dev_bf16(x[:M]), pw, workspace=ws, status=status, path=path)
            assert tsg.patch_read_status(status)[0] == 0
            check_gemm(bits_of(y), oracle.hybrid_gemm(x[:M], w, bm, ids), f"layer {li} M={M} path {path}")
        assert int(torch.count_nonzero(ws[:65536]).item()) == 0, f"counter region not left zero after {li} M={M}"


def test_gemm_zero_tokens_is_noop():
    x, w, bm, ids = _layer(256, 256, 4, "exact", 0.5)
    pw = pack_on_gpu(w, bm, ids)
    y = torch.full((0, 256), 1.0, dtype=torch.bfloat16, device="cuda")
    out = tsg.patch_gemm(torch.empty((0, 256), dtype=torch.bfloat16, device="cuda"), pw, Y=y)
    assert out.shape == (0, 256)


def test_decode_workspace_too_small_is_rejected():
    x, w, bm, ids = _layer(4096, 4096, 4, "exact", 0.5)
    pw = pack_on_gpu(w, bm, ids)
    need = tsg.patch_gemm_workspace_size(4, pw)
    assert need > 65536
    # the counter region alone: no room for the decode kernel's partial rows
    with pytest.raises(tsg.PatchError) as e:
        tsg.patch_gemm(to_dev_bf16(x), pw, workspace=torch.zeros(65536, dtype=torch.uint8, device="cuda"))
    assert e.value.code == 8


# ------------------------------------------- mask tiles finer than the execution tile


@pytest.mark.parametrize("b", [4, 8, 16, 32, 64, 128])
def test_hard_mask_tiles_bit_exact(b):
    N, K = 256, 384  # K/b mask tiles per row: 3 times a power of two (odd at b = 128)
    w = si.gen_w(N, K, 11, b)
    tl = si.gen_tile_logits(N, K, 11, b, tile=b)
    pl = si.gen_pattern_logits(N, K, 11, b)
    pl[::5, ::7, 2] = pl[::5, ::7, 0]  # ties
    pl[::13, ::3, 1] = np.nan
    tl[::3, ::2, 1] = tl[::3, ::2, 0]  # tile ties -> dense
    wm_ref, bm_ref, id_ref = oracle.hard_mask_tiles(w, tl, pl, b)
    wm, bm, ids = tsg.patch_hard_mask_tiles(to_dev_bf16(w), to_dev(tl), to_dev(pl), b)
    assert np.array_equal(bits_of(wm), wm_ref)
    assert np.array_equal(bm.cpu().numpy(), bm_ref)
    assert np.array_equal(ids.cpu().numpy(), id_ref)
    _, bm2, ids2 = tsg.patch_hard_mask_tiles(to_dev_bf16(w), to_dev(tl), to_dev(pl), b, want_masked=False)
    assert np.array_equal(bm2.cpu().numpy(), bm_ref) and np.array_equal(ids2.cpu().numpy(), id_ref)


@pytest.mark.parametrize("b", [4, 16, 64, 128])
@pytest.mark.parametrize("clustered", [False, True])
def test_exec_tiles_bit_exact(b, clustered):
    N, K = 512, 640
    for frac in (0.5, 0.9, 1.0):
        kinds = si.mask_tiles(N, K, b, frac, clustered, 12, b)
        ex_ref, n_ref = oracle.exec_tiles(kinds, N, K, b)
        ex, n = tsg.patch_exec_tiles(to_dev(kinds), N, K, b)
        assert np.array_equal(ex.cpu().numpy(), ex_ref), (b, clustered, frac)
        assert int(n.item()) == n_ref


@pytest.mark.parametrize("b", [4, 32, 64])
@pytest.mark.parametrize("M", [1, 16, 300])
def test_fine_mask_pipeline_packs_and_multiplies_as_the_masked_weight(b, M):
    """hard mask (b x b tiles) -> execution tiles -> pack of W_masked -> GEMM on
    the GPU: blobs bit-exact with the oracle's, Y within tolerance of the oracle
    GEMM on the oracle's W_masked."""
    N, K = 384, 512
    w = si.gen_w(N, K, 13, b)
    kinds = si.mask_tiles(N, K, b, 0.8, True, 13, b)  # one band of 80% of the tile rows: some execution tiles sparse
    tl = si.choice_logits(kinds)
    pl = si.gen_pattern_logits(N, K, 13, b)
    wm_ref, bm_ref, id_ref = oracle.hard_mask_tiles(w, tl, pl, b)
    ex_ref, n_ref = oracle.exec_tiles(bm_ref, N, K, b)
    assert 0 < n_ref < ex_ref.size
    v_ref, m_ref, d_ref = oracle.pack(wm_ref, ex_ref, id_ref)
    wm, bm, ids = tsg.patch_hard_mask_tiles(to_dev_bf16(w), to_dev(tl), to_dev(pl), b)
    ex, n = tsg.patch_exec_tiles(bm, N, K, b)
    status = tsg.new_status()
    pw = tsg.patch_pack(wm, ex, ids, int(n.item()), status=status)
    assert tsg.patch_read_status(status)[0] == 0
    assert np.array_equal(pw.values.cpu().numpy(), v_ref)
    assert np.array_equal(pw.meta.cpu().numpy(), m_ref)
    assert np.array_equal(pw.desc.cpu().numpy(), d_ref)
    x = si.gen_x(M, K, 13, b)
    check_gemm(gemm_on_gpu(x, pw), oracle.gemm(x, wm_ref), f"mask tile {b}, M={M}")


def test_mask_tile_arguments_are_checked():
    import ctypes
    N = K = 256
    dev = torch.device("cuda")
    w = torch.zeros((N, K), dtype=torch.bfloat16, device=dev)
    pl = torch.zeros((N, K // 4, 6), dtype=torch.float32, device=dev)
    tl = torch.zeros((N // 4, K // 4, 2), dtype=torch.float32, device=dev)
    for bad in (0, 2, 3, 48, 256):
        with pytest.raises(tsg.PatchError) as e:
            tsg.patch_hard_mask_tiles(w, tl, pl, bad)
        assert e.value.code == 1  # PATCH_ERR_INVALID_ARG, before any launch
        with pytest.raises(tsg.PatchError) as e:
            tsg.patch_exec_tiles(torch.zeros((N // 4, K // 4), dtype=torch.uint8, device=dev), N, K, bad)
        assert e.value.code == 1
    rc = tsg.lib().patch_exec_tiles(ctypes.c_void_p(tl.data_ptr()), N, K, 4, ctypes.c_void_p(tl.data_ptr()),
                                    ctypes.c_void_p(tl.data_ptr() + 4), None)
    assert rc == 3  # PATCH_ERR_ALIGN: n_sparse not 8-byte aligned
