"""GPU parity at the full workload sizes, in the launch configuration bench.py times.

Each workload's layers are packed on the GPU (byte for byte against the
oracle's pack) and multiplied through patch_gemm exactly as the benchmark
calls it.  The oracle checks every
output of the decode GEMMs (M <= 16) and a sample of token rows of the
prefill GEMMs (the fp64 triple loop over 2048 x 11008 x 4096 is too slow to
run whole); the tolerance is the layer's (relative Frobenius <= 5e-3,
|err| <= 1e-2 * (1 + |ref|)).

Workloads:
  * LLaMA-2-7B decode: 7 shapes, M in {1, 4, 16}, 50% sparse tiles (exact count)
  * LLaMA-2-7B prefill: 7 shapes, M = 2048, sparse-tile fraction 0 .. 1
  * 32-layer LLaMA-2-7B stack, M in {1, 8}, non-uniform fractions 0.1 / 0.2 / 0.7 / 0.8
  * LLaMA-3-8B and Qwen-2.5-0.5B shapes, M in {1, 512}, clustered 50% sparse tiles
"""
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


@functools.lru_cache(maxsize=16)
def weight(N, K, cfg, idx):
    w = si.gen_w(N, K, cfg, idx)
    return w, si.patterns_top2(w)


def run_layer(x, w, bm, ids, rows=None):
    """Pack on the GPU (compared byte for byte with the oracle's pack), then patch_gemm."""
    status = tsg.new_status()
    pw = tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids), int(bm.sum()), status=status)
    y = tsg.patch_gemm(to_dev_bf16(x), pw, status=status)
    code, bits = tsg.patch_read_status(status)
    assert code == 0, (code, bits)
    v_ref, m_ref, d_ref = oracle.pack(w, bm, ids)
    assert np.array_equal(pw.desc.cpu().numpy(), d_ref)
    assert np.array_equal(pw.values.cpu().numpy(), v_ref)
    assert np.array_equal(pw.meta.cpu().numpy(), m_ref)
    yb = bits_of(y)
    ref = oracle.hybrid_gemm(x, w, bm, ids, rows=rows)
    return (yb if rows is None else yb[rows]), ref


@pytest.mark.parametrize("idx", range(7))
def test_llama2_decode(idx):
    name, N, K = si.LLAMA2_7B[idx]
    w, ids = weight(N, K, 2, idx)
    bm = si.tiles_exact(N, K, 0.5, 2, idx)
    for M in (1, 4, 16):
        x = si.gen_x(M, K, 2, idx)
        y, ref = run_layer(x, w, bm, ids)
        check_gemm(y, ref, f"decode {name} M={M}")


@pytest.mark.parametrize("idx", range(7))
def test_llama2_prefill(idx):
    name, N, K = si.LLAMA2_7B[idx]
    w, ids = weight(N, K, 3, idx)
    x = si.gen_x(2048, K, 3, idx)
    rows = np.array([0, 1, 255, 256, 1023, 1500, 2046, 2047])
    for f in (0.0, 0.25, 0.5, 0.75, 1.0):
        bm = si.tiles_exact(N, K, f, 3, idx)
        y, ref = run_layer(x, w, bm, ids, rows=rows)
        check_gemm(y, ref, f"prefill {name} f={f}")


@pytest.mark.parametrize("group", ["edge", "middle"])
@pytest.mark.parametrize("M", [1, 8])
def test_llama2_stack_sampled_layers(group, M):
    """One layer of each (projection, fraction) class of the 32-layer stack."""
    layer = 0 if group == "edge" else 16
    for idx, (name, N, K) in enumerate(si.LLAMA2_7B):
        f = si.stack_fraction(layer, name)
        w, ids = weight(N, K, 4, idx)
        bm = si.tiles_exact(N, K, f, 4, 7 * layer + idx)
        x = si.gen_x(M, K, 4, 7 * layer + idx)
        y, ref = run_layer(x, w, bm, ids)
        check_gemm(y, ref, f"stack L{layer} {name} f={f} M={M}")


@pytest.mark.parametrize("family", ["llama3", "qwen", "gemma3"])
def test_llama3_qwen_clustered(family):
    shapes = {"llama3": si.LLAMA3_8B, "qwen": si.QWEN25_05B, "gemma3": si.GEMMA3_1B}[family]
    base = {"llama3": 0, "qwen": 7, "gemma3": 14}[family]
    for j, (name, N, K) in enumerate(shapes):
        idx = base + j
        w, ids = weight(N, K, 5, idx)
        bm = si.tiles_clustered(N, K, 0.5, 5, idx)
        x1 = si.gen_x(1, K, 5, idx)
        y, ref = run_layer(x1, w, bm, ids)
        check_gemm(y, ref, f"{family} {name} M=1")
        x = si.gen_x(512, K, 5, idx)
        rows = np.array([0, 127, 128, 300, 511])
        y, ref = run_layer(x, w, bm, ids, rows=rows)
        check_gemm(y, ref, f"{family} {name} M=512")
