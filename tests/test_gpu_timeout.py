"""Bounded waits: a prefill kernel whose producer stops early reports a timeout
and leaves the CUDA context usable.

PATCH_PATH_TEST_STALL makes the TMA producer stop after its first K-tile, so
the MMA thread's next mbarrier wait can never complete.  Every wait in the
kernel is bounded in time (here 0.2 s): the kernel must set
PATCH_DEV_TIMEOUT, wait for its own copies and MMAs, free tensor memory and
return, after which a normal call on the same context gives correct results.
No fault, trap or unbounded spin is involved.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import tile_sparse_gemm_b200 as tsg
from _util import bits_of, check_gemm, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


def test_prefill_stall_times_out_and_context_survives():
    assert torch.cuda.is_available() and torch.cuda.get_device_capability()[0] == 10
    N, K, M = 512, 1024, 300  # several K-tiles and output tiles
    w = si.gen_w(N, K, 13, 0)
    bm = si.tiles_exact(N, K, 0.5, 13, 0)
    ids = si.patterns_top2(w)
    x = si.gen_x(M, K, 13, 0)
    pw = tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids))
    xd = to_dev_bf16(x)

    status = tsg.new_status()
    t0 = time.monotonic()
    tsg.patch_gemm_ex(xd, pw, status=status, path=tsg.PATH_PREFILL | tsg.PATH_TEST_STALL, wait_limit_us=200_000)
    code, bits = tsg.patch_read_status(status)
    elapsed = time.monotonic() - t0
    assert code == 7 and bits & tsg.DEV_TIMEOUT, (code, bits)
    assert elapsed < 20.0, elapsed

    status = tsg.new_status()
    y = tsg.patch_gemm_ex(xd, pw, status=status, path=tsg.PATH_PREFILL)
    assert tsg.patch_read_status(status)[0] == 0
    check_gemm(bits_of(y), oracle.hybrid_gemm(x, w, bm, ids), "after timeout")
