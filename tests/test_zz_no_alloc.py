"""patch_gemm_decode_noalloc: the decode GEMM for callers that cannot allocate.

Some callers cannot get device scratch memory (a plugin whose host framework
owns the memory pool and passes it only its inputs and outputs, or a
latency-critical loop where cudaMalloc's possible device-wide synchronisation
is unacceptable).  For them the library keeps the split-K partial sums in a
buffer compiled into libpatch.so.  These tests call that entry point through
the C ABI and check it against patch_gemm (caller-provided workspace) within
the layer's tolerance, on two different problems in a row, so that the
second call also shows that what the first left in the shared buffer does
not leak into its result.  The entry point runs the CUDA-core split-K decode
path (patch_gemm_ex with PATH_DECODE_SIMT), so agreement is within the GEMM
tolerance, not bitwise.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import tile_sparse_gemm_b200 as tsg
from _util import bits_of, check_gemm, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


def noalloc(x, pw, y, status):
    L = tsg.lib()
    f = L.patch_gemm_decode_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(tsg._Weight), ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    st = pw.struct()
    return f(ctypes.c_void_p(x.data_ptr()) if x.numel() else None, x.shape[0], ctypes.byref(st),
             ctypes.c_void_p(y.data_ptr()) if y.numel() else None, ctypes.c_void_p(status.data_ptr()) if status is not None else None,
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def problem(N, K, M, frac, idx):
    w = si.gen_w(N, K, 11, idx)
    bm = si.tiles_exact(N, K, frac, 11, idx)
    ids = si.patterns_top2(w)
    x = si.gen_x(M, K, 11, idx)
    pw = tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids))
    return x, w, bm, ids, pw


COUNTER_REGION = 65536  # fixed counter region at the start of a patch_gemm workspace


def simt_needs_partials(xd, pw):
    """True when the CUDA-core decode path splits K for this problem: it then
    rejects a workspace that holds only the counter region (no room for the
    fp32 partials) and accepts one of patch_gemm_workspace_size bytes."""
    M = xd.shape[0]
    small = torch.zeros(COUNTER_REGION, dtype=torch.uint8, device="cuda")
    try:
        tsg.patch_gemm_ex(xd, pw, workspace=small, path=tsg.PATH_DECODE_SIMT)
    except tsg.PatchError as e:
        assert e.code == 8, e  # PATCH_ERR_WORKSPACE, before any launch
        full = torch.zeros(tsg.patch_gemm_workspace_size(M, pw), dtype=torch.uint8, device="cuda")
        tsg.patch_gemm_ex(xd, pw, workspace=full, path=tsg.PATH_DECODE_SIMT)
        return True
    return False


def test_noalloc_matches_patch_gemm_on_two_calls_in_a_row():
    assert torch.cuda.is_available() and torch.cuda.get_device_capability()[0] == 10
    # first a problem with many K splits (large partial-sum footprint), then a smaller one
    cases = [(4096, 4096, 16, 0.5, 0), (1024, 2048, 5, 0.75, 1)]
    for N, K, M, frac, idx in cases:
        x, w, bm, ids, pw = problem(N, K, M, frac, idx)
        xd = to_dev_bf16(x)
        # the CUDA-core plan splits K here, so the built-in buffer really carries partial sums
        assert simt_needs_partials(xd, pw)
        status = tsg.new_status()
        y_ref = tsg.patch_gemm(xd, pw, status=status)   # existing entry point, caller workspace
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert noalloc(xd, pw, y, status) == 0
        code, bits = tsg.patch_read_status(status)
        assert code == 0, (code, bits)
        ref_bits = bits_of(y_ref)
        check_gemm(bits_of(y), (ref_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64),
                   f"noalloc vs patch_gemm N={N} K={K} M={M}")
        # and both against the oracle
        check_gemm(bits_of(y), oracle.hybrid_gemm(x, w, bm, ids), "noalloc vs oracle")


def test_noalloc_rejects_partials_beyond_the_buffer():
    # N = 34816 (544 row slabs of 64 < 4 per SM on 148 SMs) splits K in two:
    # 2 x 16 x 34816 x 4 B = 4.46 MB of partials > the 4 MiB buffer
    N, K, M = 34816, 256, 16
    x, w, bm, ids, pw = problem(N, K, M, 0.5, 3)
    xd = to_dev_bf16(x)
    assert simt_needs_partials(xd, pw)
    y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    assert noalloc(xd, pw, y, tsg.new_status()) == 8  # PATCH_ERR_WORKSPACE, nothing launched
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(y.view(torch.int16))) == 0
    # one token fewer fits: 2 x 15 x 34816 x 4 B = 4,177,920 B <= 4,194,304 B
    y15 = torch.empty((15, N), dtype=torch.bfloat16, device="cuda")
    assert noalloc(xd[:15], pw, y15, None) == 0  # dev_status may be NULL on this path
    check_gemm(bits_of(y15), oracle.hybrid_gemm(x[:15], w, bm, ids), "noalloc M=15 at the buffer's limit")


def test_noalloc_argument_checks():
    x, w, bm, ids, pw = problem(256, 256, 4, 0.5, 2)
    status = tsg.new_status()
    empty = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    assert noalloc(empty, pw, torch.empty((0, 256), dtype=torch.bfloat16, device="cuda"), status) == 0
    big = torch.zeros((17, 256), dtype=torch.bfloat16, device="cuda")
    assert noalloc(big, pw, torch.empty((17, 256), dtype=torch.bfloat16, device="cuda"), status) == 1
    assert tsg.patch_read_status(status)[0] == 0
