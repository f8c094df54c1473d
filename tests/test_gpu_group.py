"""GPU parity of patch_gemm_group (independent GEMMs of any token count in one
launch of the prefill kernel) through the C ABI against the CPU oracle.

"PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", section 2
"Inference & Deployment": each GEMM of the group is the hybrid layer (dense
tiles on dense tensor-core MMA, 2:4 tiles on the sparse one), so each Y_j is
checked against the oracle's fp64 product within the layer's tolerance
(relative Frobenius error <= 5e-3, |err| <= 1e-2 (1 + |ref|)).  The groups mix
shapes, token counts (1 ... 1000, ragged token blocks) and sparse fractions,
so the CTAs' waves interleave units of different GEMMs."""
import functools

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import tile_sparse_gemm_b200 as tsg
from _util import bits_of, check_gemm, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available() and torch.cuda.get_device_capability()[0] == 10
    tsg.lib()


def layer(N, K, frac, seed):
    w = si.gen_w(N, K, 5, seed)
    bm = si.tiles_exact(N, K, frac, 5, seed)
    ids = si.patterns_top2(w)
    status = tsg.new_status()
    pw = tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids), int(bm.sum()), status=status)
    assert tsg.patch_read_status(status)[0] == 0
    return w, bm, ids, pw


def run_group(specs, seed0=0):
    """specs: list of (N, K, frac, M); returns [(y bits, oracle masked W, x)]."""
    calls, keep = [], []
    for j, (N, K, frac, M) in enumerate(specs):
        w, bm, ids, pw = layer(N, K, frac, seed0 + j)
        x = si.gen_x(M, K, 5, seed0 + 100 + j)
        calls.append((to_dev_bf16(x), pw, None))
        keep.append((x, oracle.apply_mask(w, bm, ids)))
    status = tsg.new_status()
    ys = tsg.patch_gemm_group(calls, status=status)
    code, bits = tsg.patch_read_status(status)
    assert code == 0, (code, bits)
    return [(bits_of(y), wm, x) for y, (x, wm) in zip(ys, keep)]


GROUPS = {
    # a small model's projections at one token count (one short wave each alone)
    "qwen_like": [(896, 896, 0.5, 300), (128, 896, 0.5, 300), (128, 896, 0.5, 300), (896, 896, 0.5, 300),
                  (1024, 896, 0.5, 300), (896, 1024, 0.5, 300)],
    # mixed shapes, token counts and fractions; odd tile-row counts (a pair with one row)
    "mixed": [(384, 640, 0.0, 17), (1024, 512, 1.0, 257), (128, 128, 0.5, 1), (640, 384, 0.3, 1000),
              (256, 2048, 0.7, 16), (1152, 256, 0.5, 241)],
}


@pytest.mark.parametrize("name", list(GROUPS))
def test_group_matches_oracle(name):
    for j, (y, wm, x) in enumerate(run_group(GROUPS[name])):
        check_gemm(y, oracle.gemm(x, wm), f"{name} call {j}")


def test_group_of_more_than_32_calls_takes_several_launches():
    specs = [(128 * (1 + j % 3), 256, (j % 5) / 4, 20 + 7 * j) for j in range(35)]
    for j, (y, wm, x) in enumerate(run_group(specs, 40)):
        check_gemm(y, oracle.gemm(x, wm), f"call {j}")


def test_group_is_deterministic_and_agrees_with_separate_calls():
    specs = [(1024, 1536, 0.5, 300), (256, 1536, 0.5, 300), (512, 640, 0.25, 33)]
    calls = []
    for j, (N, K, frac, M) in enumerate(specs):
        w, bm, ids, pw = layer(N, K, frac, 60 + j)
        calls.append((to_dev_bf16(si.gen_x(M, K, 5, 160 + j)), pw, None, oracle.apply_mask(w, bm, ids)))
    g = tsg.Group([(x, pw, y) for x, pw, y, _ in calls])
    y1 = [bits_of(y) for y in g.run()]
    y2 = [bits_of(y) for y in g.run()]
    for a, b in zip(y1, y2):
        assert np.array_equal(a, b)
    for (x, pw, _, wm), y in zip(calls, y1):
        xs = bits_of(x)
        ref = oracle.gemm(xs, wm)
        check_gemm(y, ref, "group")
        check_gemm(bits_of(tsg.patch_gemm(x, pw)), ref, "separate")


def test_group_full_size_llama3_qwen_m512_sampled():
    """LLaMA-3-8B and Qwen-2.5-0.5B linears, clustered half-sparse tiles, M = 512
    (the mid-size prefill workload), as one group; sampled token rows."""
    calls, refs = [], []
    for j, (name, N, K) in enumerate(si.LLAMA3_8B + si.QWEN25_05B):
        w = si.gen_w(N, K, 5, j)
        bm = si.tiles_clustered(N, K, 0.5, 5, j)
        ids = si.patterns_top2(w)
        status = tsg.new_status()
        pw = tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids), int(bm.sum()), status=status)
        x = si.gen_x(512, K, 5, j)
        calls.append((to_dev_bf16(x), pw, None))
        refs.append((name, x, w, bm, ids))
    ys = tsg.patch_gemm_group(calls)
    rows = np.array([0, 175, 176, 351, 352, 511])  # both sides of each 176-token block boundary
    for y, (name, x, w, bm, ids) in zip(ys, refs):
        ref = oracle.gemm(x, oracle.apply_mask(w, bm, ids), rows=rows)
        check_gemm(bits_of(y)[rows], ref, f"{name} M=512")


@functools.lru_cache(maxsize=8)
def llama2_weight(idx):
    name, N, K = si.LLAMA2_7B[idx]
    w = si.gen_w(N, K, 3, idx)
    return w, si.patterns_top2(w)


@pytest.mark.parametrize("frac", [0.0, 1.0])
def test_group_full_size_llama2_prefill_sampled(frac):
    """The 7 LLaMA-2-7B linears at M = 2048 and one sparse-tile fraction as one
    group (the bench's grouped prefill launch), on sampled token rows at the
    240-token block edges."""
    calls, refs = [], []
    status = tsg.new_status()
    for idx, (name, N, K) in enumerate(si.LLAMA2_7B):
        w, ids = llama2_weight(idx)
        bm = si.tiles_exact(N, K, frac, 3, idx)
        pw = tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids), int(bm.sum()), status=status)
        x = si.gen_x(2048, K, 3, idx)
        calls.append((to_dev_bf16(x), pw, None))
        refs.append((name, x, w, bm, ids))
    ys = tsg.patch_gemm_group(calls, status=status)
    code, bits = tsg.patch_read_status(status)
    assert code == 0, (code, bits)
    rows = np.array([0, 1, 239, 240, 1023, 1500, 2046, 2047])
    for y, (name, x, w, bm, ids) in zip(ys, refs):
        ref = oracle.hybrid_gemm(x, w, bm, ids, rows=rows)
        check_gemm(bits_of(y)[rows], ref, f"{name} f={frac}")


def test_group_skips_empty_calls_and_checks_arguments():
    w, bm, ids, pw = layer(256, 256, 0.5, 70)
    x = to_dev_bf16(si.gen_x(40, 256, 5, 70))
    empty = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    ys = tsg.patch_gemm_group([(empty, pw, None), (x, pw, None)])
    assert ys[0].shape == (0, 256)
    check_gemm(bits_of(ys[1]), oracle.gemm(bits_of(x), oracle.apply_mask(w, bm, ids)), "after an empty call")
    assert tsg.patch_gemm_group([]) == []
    g = tsg.Group([(x, pw, None)])
    g.calls[0].after_previous = 1  # the group's calls are independent by definition
    with pytest.raises(tsg.PatchError) as e:
        g.run()
    assert e.value.code == 1  # PATCH_ERR_INVALID_ARG
    g = tsg.Group([(x, pw, None)])
    g.calls[0].X = g.calls[0].X + 2  # not 16-byte aligned
    with pytest.raises(tsg.PatchError) as e:
        g.run()
    assert e.value.code == 3  # PATCH_ERR_ALIGN


def test_group_wait_limit_runs_out_cleanly():
    """A 1 us wait limit makes the bounded waits give up: the call reports
    DEV_TIMEOUT (or finishes in time), and the context stays usable."""
    specs = [(2048, 4096, 0.5, 512), (1024, 4096, 0.5, 512)]
    calls = []
    for j, (N, K, frac, M) in enumerate(specs):
        w, bm, ids, pw = layer(N, K, frac, 80 + j)
        calls.append((to_dev_bf16(si.gen_x(M, K, 5, 180 + j)), pw, None))
    status = tsg.new_status()
    tsg.patch_gemm_group(calls, status=status, wait_limit_us=1)
    code, bits = tsg.patch_read_status(status)
    assert code in (0, 7), (code, bits)  # PATCH_OK or PATCH_ERR_TIMEOUT
    for y, (x, pw, _) in zip(tsg.patch_gemm_group(calls), calls):
        assert torch.isfinite(y.float()).all()
