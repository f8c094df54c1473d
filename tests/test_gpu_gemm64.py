"""GPU parity of the 64 x 64 execution-tile format ("Ablation Studies", tile
size) through the C ABI against the CPU oracle: pack and execution tiles byte
for byte, the GEMM within the layer's tolerance (relative Frobenius error
<= 5e-3, |err| <= 1e-2 (1 + |ref|)).  Shapes with odd tile counts make the
stream-K shares cut tile rows at arbitrary panels; the token counts cover
the 16-token decode blocks, the 256-token blocks and ragged last blocks."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import tile_sparse_gemm_b200 as tsg
from _util import bits_of, check_gemm, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu
T64 = 64


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert torch.cuda.get_device_capability()[0] == 10, "GPU tests need an sm_100 device"
    tsg.lib()


def layer64(N, K, frac, seed, cfg=2):
    """W, a random 64 x 64 bitmap with the given sparse fraction, magnitude top-2 pattern ids."""
    w = si.gen_w(N, K, cfg, seed)
    rng = np.random.default_rng(1000 + seed)
    bm = (rng.random((N // T64, K // T64)) < frac).astype(np.uint8)
    ids = si.patterns_top2(w)
    return w, bm, ids


def pack64_on_gpu(w, bm, ids):
    status = tsg.new_status()
    pw = tsg.patch_pack64(to_dev_bf16(w), to_dev(bm), to_dev(ids), int(bm.sum()), status=status)
    code, bits = tsg.patch_read_status(status)
    assert code == 0, (code, bits)
    return pw


def gemm64_on_gpu(x, pw, workspace=None):
    status = tsg.new_status()
    y = tsg.patch_gemm64(to_dev_bf16(x), pw, workspace=workspace, status=status)
    code, bits = tsg.patch_read_status(status)
    assert code == 0, (code, bits)
    return bits_of(y)


@pytest.mark.parametrize("N,K,frac", [(64, 64, 1.0), (192, 320, 0.5), (1024, 1536, 0.3), (512, 256, 0.0),
                                      (256, 512, 1.0)])
def test_pack64_byte_exact(N, K, frac):
    w, bm, ids = layer64(N, K, frac, 1)
    v, m, d = oracle.pack64(w, bm, ids)
    pw = pack64_on_gpu(w, bm, ids)
    assert np.array_equal(pw.desc.cpu().numpy(), d)
    assert np.array_equal(pw.values.cpu().numpy(), v)
    assert np.array_equal(pw.meta.cpu().numpy(), m)


def test_pack64_flags_bad_patterns_and_counts():
    w, bm, ids = layer64(128, 128, 1.0, 2)
    ids = ids.copy()
    ids[5, 3] = 9
    status = tsg.new_status()
    tsg.patch_pack64(to_dev_bf16(w), to_dev(bm), to_dev(ids), int(bm.sum()), status=status)
    code, bits = tsg.patch_read_status(status)
    assert bits & tsg.DEV_BAD_PATTERN
    status = tsg.new_status()
    n = int(bm.sum())
    pw = tsg.patch_pack64(to_dev_bf16(w), to_dev(bm), to_dev(layer64(128, 128, 1.0, 2)[2]), n - 1, status=status)
    code, bits = tsg.patch_read_status(status)
    assert bits & tsg.DEV_COUNT
    assert pw.values.numel() == tsg.patch_pack64_sizes(128, 128, n - 1)[0]


@pytest.mark.parametrize("b", [4, 8, 16, 32, 64])
def test_exec_tiles64_bit_exact(b):
    N, K = 3 * T64, 5 * T64
    rng = np.random.default_rng(b)
    bm = (rng.random((N // b, K // b)) < (0.97 if b < 16 else 0.6)).astype(np.uint8)
    ex_ref, n_ref = oracle.exec_tiles_e(bm, N, K, b, 64)
    ex, n = tsg.patch_exec_tiles64(to_dev(bm), N, K, b)
    assert np.array_equal(ex.cpu().numpy(), ex_ref) and int(n.item()) == n_ref


GEMM_CASES = [  # N, K, frac, M
    (64, 64, 1.0, 1), (64, 64, 0.0, 16), (192, 320, 0.5, 1), (192, 320, 0.5, 7), (192, 320, 0.5, 16),
    (1024, 1536, 0.3, 4), (1024, 1536, 0.7, 16), (512, 4096, 0.5, 1), (4096, 256, 0.5, 3),
    (192, 320, 0.5, 17), (256, 512, 0.0, 256), (256, 512, 1.0, 257), (1024, 1536, 0.5, 300),
    (640, 1024, 0.5, 1000),
]


@pytest.mark.parametrize("N,K,frac,M", GEMM_CASES)
def test_gemm64_matches_oracle(N, K, frac, M):
    w, bm, ids = layer64(N, K, frac, M)
    x = si.gen_x(M, K, 2, N + M)
    pw = pack64_on_gpu(w, bm, ids)
    ref = oracle.gemm(x, oracle.apply_mask_tiles(w, bm, ids, 64))
    check_gemm(gemm64_on_gpu(x, pw), ref, f"gemm64 {N}x{K} f={frac} M={M}")


def test_gemm64_deterministic_and_leaves_counters_zero():
    """Two calls give the same bits; the counter region is zero after each (one
    zero-filled workspace serves every call)."""
    N, K, M = 1024, 1536, 16
    w, bm, ids = layer64(N, K, 0.5, 3)
    pw = pack64_on_gpu(w, bm, ids)
    x = si.gen_x(M, K, 2, 3)
    ws = torch.zeros(tsg.patch_gemm64_workspace_size(M, pw), dtype=torch.uint8, device="cuda")
    y1 = gemm64_on_gpu(x, pw, ws)
    counters = (N // 64) * 16  # one token block: 4 u32 per tile row
    assert int(torch.count_nonzero(ws[:counters]).item()) == 0
    y2 = gemm64_on_gpu(x, pw, ws)
    assert np.array_equal(y1, y2)
    assert int(torch.count_nonzero(ws[:counters]).item()) == 0
    # the same workspace, now at a prefill token count and back
    x2 = si.gen_x(300, K, 2, 4)
    ws2 = torch.zeros(max(tsg.patch_gemm64_workspace_size(300, pw), ws.numel()), dtype=torch.uint8, device="cuda")
    gemm64_on_gpu(x2, pw, ws2)
    assert np.array_equal(gemm64_on_gpu(x, pw, ws2), y1)


def test_gemm64_equals_the_128_path_on_a_128_granular_mask():
    """A bitmap made of whole 128 x 128 tiles gives the same layer in both
    formats (each within tolerance of the oracle, and close to each other)."""
    N, K, M = 512, 1024, 5
    w = si.gen_w(N, K, 2, 9)
    bm128 = (np.random.default_rng(9).random((N // 128, K // 128)) < 0.5).astype(np.uint8)
    bm64 = np.repeat(np.repeat(bm128, 2, axis=0), 2, axis=1)
    ids = si.patterns_top2(w)
    x = si.gen_x(M, K, 2, 9)
    ref = oracle.gemm(x, oracle.apply_mask(w, bm128, ids))
    pw64 = pack64_on_gpu(w, bm64, ids)
    y64 = gemm64_on_gpu(x, pw64)
    check_gemm(y64, ref, "64 format")
    status = tsg.new_status()
    pw128 = tsg.patch_pack(to_dev_bf16(w), to_dev(bm128), to_dev(ids), int(bm128.sum()), status=status)
    y128 = bits_of(tsg.patch_gemm(to_dev_bf16(x), pw128, status=status))
    assert tsg.patch_read_status(status)[0] == 0
    check_gemm(y128, ref, "128 format")


@pytest.mark.parametrize("b", [4, 32, 64])
def test_fine_mask_runs_as_the_masked_weight(b):
    """The product path of the ablation: patch_hard_mask_tiles -> patch_exec_tiles64
    -> patch_pack64 of W_masked -> patch_gemm64 equals the oracle's masked layer."""
    N, K, M = 512, 768, 9
    w = si.gen_w(N, K, 2, b)
    kinds = si.mask_tiles(N, K, b, 0.5, False, 2, b)
    tl = si.choice_logits(kinds)
    pl = np.zeros((N, K // 4, 6), np.float32)
    np.put_along_axis(pl, si.patterns_top2(w)[..., None].astype(np.int64), 1.0, axis=2)
    status = tsg.new_status()
    wm, bm, pid = tsg.patch_hard_mask_tiles(to_dev_bf16(w), to_dev(tl), to_dev(pl), b, status=status)
    ex, n_dev = tsg.patch_exec_tiles64(bm, N, K, b)
    pw = tsg.patch_pack64(wm, ex, pid, int(n_dev.item()), status=status)
    assert tsg.patch_read_status(status)[0] == 0
    wm_ref, bm_ref, pid_ref = oracle.hard_mask_tiles(w, tl, pl, b)
    ex_ref, n_ref = oracle.exec_tiles_e(bm_ref, N, K, b, 64)
    assert pw.n_sparse == n_ref
    if b == 64:
        assert n_ref == int(kinds.sum())  # every sparse mask tile runs sparse
    x = si.gen_x(M, K, 2, b)
    check_gemm(gemm64_on_gpu(x, pw), oracle.gemm(x, wm_ref), f"fine mask b={b}")


@pytest.mark.parametrize("name,N,K", [(n, N, K) for n, N, K in si.LLAMA2_7B if n in ("q", "down")])
def test_gemm64_full_size_sampled(name, N, K):
    """LLaMA-2-7B shapes with a random half of the 64-tiles sparse, M = 1, 16
    and 2048, on sampled output rows."""
    w, bm, ids = layer64(N, K, 0.5, 5)
    pw = pack64_on_gpu(w, bm, ids)
    wm = oracle.apply_mask_tiles(w, bm, ids, 64)
    for M in (1, 16, 2048):
        x = si.gen_x(M, K, 2, M)
        y = gemm64_on_gpu(x, pw)
        rows = np.unique(np.random.default_rng(M).integers(0, M, 12))
        ref = oracle.gemm(x, wm, rows=rows)
        check_gemm(y[rows], ref, f"{name} M={M}")


def test_gemm64_argument_checks():
    w, bm, ids = layer64(128, 128, 0.5, 1)
    pw = pack64_on_gpu(w, bm, ids)
    x = to_dev_bf16(si.gen_x(4, 128, 2, 1))
    with pytest.raises(tsg.PatchError) as e:
        tsg.patch_gemm64(x, pw, workspace=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert e.value.code == 8  # PATCH_ERR_WORKSPACE
    with pytest.raises(TypeError):
        tsg.patch_gemm64(x, tsg.patch_pack(to_dev_bf16(w), to_dev(np.zeros((1, 1), np.uint8)), to_dev(ids), 0))
    with pytest.raises(tsg.PatchError) as e:
        tsg.patch_pack64_sizes(96, 128, 0)
    assert e.value.code == 2  # PATCH_ERR_SHAPE
    assert tsg.patch_gemm64(x[:0], pw).shape == (0, 128)


def test_gemm64_wait_limit_runs_out_cleanly():
    """A 1 us wait limit makes the bounded waits give up: the call reports
    DEV_TIMEOUT (or finishes in time), and the context stays usable."""
    N, K, M = 1024, 4096, 16
    w, bm, ids = layer64(N, K, 0.5, 6)
    pw = pack64_on_gpu(w, bm, ids)
    x = si.gen_x(M, K, 2, 6)
    status = tsg.new_status()
    tsg.patch_gemm64(to_dev_bf16(x), pw, status=status, wait_limit_us=1)
    code, bits = tsg.patch_read_status(status)
    assert code in (0, 7), (code, bits)  # PATCH_OK or PATCH_ERR_TIMEOUT
    ref = oracle.gemm(x, oracle.apply_mask_tiles(w, bm, ids, 64))
    check_gemm(gemm64_on_gpu(x, pw), ref, "after a timed-out call")
