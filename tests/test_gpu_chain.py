"""patch_gemm_chain on the GPU, called through the C ABI: a sequence of decode
GEMMs in one persistent launch, each output within the layer's tolerance of
the oracle (relative Frobenius <= 5e-3, |err| <= 1e-2 (1 + |ref|)).

Covers independent and dependent calls (a call reading the previous call's
output, which starts as NaN so that a read before it is written fails),
tiny layers with fewer panels than CTAs, chains long enough to need several
launches (more calls than one launch takes, more tile rows than the counter
region holds), a workspace shared with patch_gemm, skipped M = 0 calls,
determinism across runs, the argument checks, the full LLaMA-2-7B decode
step as one chain, and a bounded wait that runs out (the kernel reports
PATCH_ERR_TIMEOUT and the context stays usable)."""
import ctypes
import functools

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import tile_sparse_gemm_b200 as tsg
from _util import bits_of, bf16_to_f64, check_gemm, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu
CFG = 17


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available() and torch.cuda.get_device_capability()[0] == 10
    tsg.lib()


@functools.lru_cache(maxsize=64)
def layer(N, K, frac, idx, clustered=False):
    w = si.gen_w(N, K, CFG, idx)
    bm = (si.tiles_clustered if clustered else si.tiles_exact)(N, K, frac, CFG, idx)
    ids = si.patterns_top2(w)
    return w, bm, ids, tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids))


def test_independent_calls_mixed_shapes_and_tokens():
    specs = [(4096, 4096, 0.5, 1, 1), (1024, 2048, 0.0, 5, 0), (128, 896, 0.5, 16, 1), (2048, 1024, 1.0, 3, 1),
             (896, 896, 0.5, 2, 0), (4096, 4096, 0.25, 16, 1), (256, 128, 0.5, 7, 1)]
    calls, refs = [], []
    for idx, (N, K, f, M, after) in enumerate(specs):
        w, bm, ids, pw = layer(N, K, f, idx, clustered=(idx % 2 == 1))
        x = si.gen_x(M, K, CFG, 100 + idx)
        calls.append((to_dev_bf16(x), pw, None, bool(after)))
        refs.append(oracle.hybrid_gemm(x, w, bm, ids))
    ch = tsg.Chain(calls)
    ys = ch.run()
    assert tsg.patch_read_status(ch.status)[0] == 0
    first = [bits_of(y) for y in ys]
    for (N, K, f, M, _), y, ref in zip(specs, first, refs):
        check_gemm(y, ref, f"chain {N}x{K} f={f} M={M}")
    # a second run on the same workspace (counters left zero) gives the same bits
    ys = ch.run()
    assert tsg.patch_read_status(ch.status)[0] == 0
    for a, b in zip(first, ys):
        assert np.array_equal(a, bits_of(b))


def test_calls_that_wait_for_none_split_the_whole_launch():
    """With no call waiting for another the CTAs split the launch's whole panel
    sequence (runs cross call boundaries; small calls fall inside one CTA's run;
    only the rows at the ends of each run are cut)."""
    specs = [(128, 896, 0.5, 3), (4096, 4096, 0.5, 16), (256, 128, 1.0, 1), (11008, 512, 0.5, 5),
             (128, 128, 0.0, 2), (1024, 2048, 0.75, 8), (896, 4864, 0.5, 16), (128, 256, 0.5, 1)]
    calls, refs = [], []
    for idx, (N, K, f, M) in enumerate(specs):
        w, bm, ids, pw = layer(N, K, f, 80 + idx, clustered=(idx % 3 == 0))
        x = si.gen_x(M, K, CFG, 800 + idx)
        calls.append((to_dev_bf16(x), pw, None, False))
        refs.append(oracle.hybrid_gemm(x, w, bm, ids))
    ch = tsg.Chain(calls)
    first = None
    for _ in range(2):
        ys = ch.run()
        assert tsg.patch_read_status(ch.status)[0] == 0
        got = [bits_of(y) for y in ys]
        for (N, K, f, M), y, ref in zip(specs, got, refs):
            check_gemm(y, ref, f"global split {N}x{K} f={f} M={M}")
        if first is not None:
            for a_, b_ in zip(first, got):
                assert np.array_equal(a_, b_)
        first = got


def test_dependent_calls_read_the_previous_output():
    # x0 -> L0 (4096 x 2048) -> L1 (1024 x 4096) -> L2 (4096 x 1024) -> L3 (2048 x 4096)
    shapes = [(4096, 2048, 0.5), (1024, 4096, 0.25), (4096, 1024, 0.75), (2048, 4096, 0.5)]
    M = 4
    x0 = si.gen_x(M, 2048, CFG, 200)
    lays = [layer(N, K, f, 20 + i) for i, (N, K, f) in enumerate(shapes)]
    ys = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") for N, _, _ in shapes]
    calls = [(to_dev_bf16(x0), lays[0][3], ys[0], True)]
    for i in range(1, len(shapes)):
        calls.append((ys[i - 1], lays[i][3], ys[i], True))
    ch = tsg.Chain(calls)
    ch.run()
    assert tsg.patch_read_status(ch.status)[0] == 0
    refs = oracle.chain(x0, [(w, bm, ids) for w, bm, ids, _ in lays])
    for i, (y, ref) in enumerate(zip(ys, refs)):
        # each layer against the oracle on the GPU's own (bf16) input, and the chain against the oracle's chain
        x_in = x0 if i == 0 else bits_of(ys[i - 1])
        w, bm, ids, _ = lays[i]
        check_gemm(bits_of(y), oracle.hybrid_gemm(x_in, w, bm, ids), f"dependent layer {i}")
        check_gemm(bits_of(y), ref, f"dependent chain after layer {i}")


def test_long_chain_takes_several_launches():
    # 70 calls (more than one launch holds) of a layer with 86 tile rows (the
    # counter region holds ~47 such calls per launch), alternating with small ones
    w1, bm1, ids1, pw1 = layer(11008, 128, 0.5, 40)
    w2, bm2, ids2, pw2 = layer(256, 384, 0.5, 41)
    calls, refs = [], []
    for j in range(70):
        M = 1 + j % 16
        if j % 2 == 0:
            x = si.gen_x(M, 128, CFG, 300 + j)
            calls.append((to_dev_bf16(x), pw1, None, j % 3 != 0))
            refs.append((x, w1, bm1, ids1))
        else:
            x = si.gen_x(M, 384, CFG, 300 + j)
            calls.append((to_dev_bf16(x), pw2, None, j % 3 != 0))
            refs.append((x, w2, bm2, ids2))
    ch = tsg.Chain(calls)
    ys = ch.run()
    assert tsg.patch_read_status(ch.status)[0] == 0
    for j, (y, (x, w, bm, ids)) in enumerate(zip(ys, refs)):
        check_gemm(bits_of(y), oracle.hybrid_gemm(x, w, bm, ids), f"long chain call {j}")


def test_workspace_shared_with_patch_gemm_and_zero_token_calls():
    w, bm, ids, pw = layer(4096, 4096, 0.5, 50)
    w2, bm2, ids2, pw2 = layer(2048, 4096, 0.5, 51)
    x = si.gen_x(8, 4096, CFG, 500)
    xd = to_dev_bf16(x)
    y_skip = torch.full((0, 2048), 0.0, dtype=torch.bfloat16, device="cuda")
    calls = [(xd, pw, None, True), (xd[:0], pw2, y_skip, True), (xd, pw2, None, True)]
    probe = tsg.Chain(calls)
    size = max(probe.workspace_bytes, tsg.patch_gemm_workspace_size(8, pw), tsg.patch_gemm_workspace_size(300, pw))
    ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
    status = tsg.new_status()
    ch = tsg.Chain(calls, workspace=ws, status=status)
    ref1, ref2 = oracle.hybrid_gemm(x, w, bm, ids), oracle.hybrid_gemm(x, w2, bm2, ids2)
    x300 = si.gen_x(300, 4096, CFG, 501)
    ref300 = oracle.hybrid_gemm(x300, w, bm, ids, rows=np.array([0, 150, 299]))
    for _ in range(2):  # chain, decode GEMM, split-K prefill GEMM, chain again, on one workspace
        ys = ch.run()
        check_gemm(bits_of(ys[0]), ref1, "chain call 0")
        check_gemm(bits_of(ys[2]), ref2, "chain call 2")
        y = tsg.patch_gemm(xd, pw, workspace=ws, status=status)
        check_gemm(bits_of(y), ref1, "patch_gemm decode on the shared workspace")
        y = tsg.patch_gemm(to_dev_bf16(x300), pw, workspace=ws, status=status)
        check_gemm(bits_of(y)[[0, 150, 299]], ref300, "patch_gemm prefill on the shared workspace")
    assert tsg.patch_read_status(status)[0] == 0


@pytest.mark.parametrize("after", [True, False])
def test_llama2_decode_step_as_one_chain(after):
    """The benchmark's decode step: 7 LLaMA-2-7B layers x M = 1, 4, 16 as one chain,
    each call waiting for the previous one, or none waiting (the split of the
    whole step's panel sequence the benchmark's headline runs); every output checked."""
    calls, refs = [], []
    packs = {}
    for idx, (name, N, K) in enumerate(si.LLAMA2_7B):
        w = si.gen_w(N, K, 2, idx)
        bm = si.tiles_exact(N, K, 0.5, 2, idx)
        ids = si.patterns_top2(w)
        packs[idx] = (w, bm, ids, tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids)))
    for M in (1, 4, 16):
        for idx, (name, N, K) in enumerate(si.LLAMA2_7B):
            w, bm, ids, pw = packs[idx]
            x = si.gen_x(M, K, 2, idx)
            calls.append((to_dev_bf16(x), pw, None, after))
            refs.append((f"{name}@M={M}", x, w, bm, ids))
    ch = tsg.Chain(calls)
    ys = ch.run()
    assert tsg.patch_read_status(ch.status)[0] == 0
    for y, (what, x, w, bm, ids) in zip(ys, refs):
        check_gemm(bits_of(y), oracle.hybrid_gemm(x, w, bm, ids), f"chain {what}")


def _raw_chain(calls_arr, n, ws, status, limit=0):
    L = tsg.lib()
    return L.patch_gemm_chain(ctypes.cast(calls_arr, ctypes.c_void_p), n,
                              ctypes.c_void_p(ws.data_ptr()) if ws is not None else None,
                              ws.numel() if ws is not None else 0, ctypes.c_void_p(status.data_ptr()),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), limit)


def test_argument_checks():
    w, bm, ids, pw = layer(256, 256, 0.5, 60)
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    status = tsg.new_status()
    ws = torch.zeros(tsg.Chain([(x, pw, y, False)]).workspace_bytes, dtype=torch.uint8, device="cuda")

    def arr(*calls):
        a = (tsg._ChainCall * len(calls))()
        for j, c in enumerate(calls):
            a[j] = c
        return a

    good = tsg._ChainCall(x.data_ptr(), y.data_ptr(), pw.struct(), 4, 1, 0)
    assert _raw_chain(arr(good), 1, ws, status) == 0
    assert _raw_chain(arr(tsg._ChainCall(x.data_ptr(), y.data_ptr(), pw.struct(), 17, 1, 0)), 1, ws, status) == 1
    assert _raw_chain(arr(tsg._ChainCall(x.data_ptr() + 2, y.data_ptr(), pw.struct(), 4, 1, 0)), 1, ws, status) == 3
    assert _raw_chain(arr(good), 1, ws[:1024], status) == 8  # workspace too small
    assert _raw_chain(arr(good), 1, None, status) == 8
    assert _raw_chain(arr(good), -1, ws, status) == 1
    assert _raw_chain(arr(good), 0, ws, status) == 0  # nothing to do
    wide = pw.struct()
    wide.N = 4096 * 128  # 4096 tile rows: more than the counter region holds for one call
    assert _raw_chain(arr(tsg._ChainCall(x.data_ptr(), y.data_ptr(), wide, 4, 1, 0)), 1, ws, status) == 2
    assert tsg.patch_read_status(status)[0] == 0


def test_wait_that_runs_out_reports_timeout_and_leaves_the_context_usable():
    # the second call waits for the first (~5 us on every CTA); a 1 us limit runs out
    w, bm, ids, pw = layer(4096, 4096, 0.5, 70)
    x = si.gen_x(16, 4096, CFG, 700)
    xd = to_dev_bf16(x)
    status = tsg.new_status()
    ch = tsg.Chain([(xd, pw, None, True), (xd, pw, None, True), (xd, pw, None, True)], status=status)
    ch.run(wait_limit_us=1)
    code, bits = tsg.patch_read_status(status)
    assert code == 7 and bits & tsg.DEV_TIMEOUT, (code, bits)
    # after an error: zero the workspace and the status word, then the same chain runs normally
    ch.workspace.zero_()
    status.zero_()
    ys = ch.run()
    assert tsg.patch_read_status(status)[0] == 0
    ref = oracle.hybrid_gemm(x, w, bm, ids)
    for y in ys:
        check_gemm(bits_of(y), ref, "after the timeout")
    assert np.isfinite(bf16_to_f64(bits_of(ys[0]))).all()
