"""The packed-weight check on the GPU: patch_check_weight flags a descriptor
table that breaks the packed format, and the debug build (libpatch_debug.so,
every GEMM entry point checks its weights first) refuses such a weight with
PATCH_ERR_BOUNDS before any GEMM kernel runs, while valid weights multiply as
in the release build.  The corrupted tables are only ever read by the check
kernel, which reads nothing but the descriptors themselves."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import synth_inputs as si
import tile_sparse_gemm_b200 as tsg
from _util import to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def corruptions(pw):
    """Copies of a packed weight whose descriptor tables break one rule each."""
    d = pw.desc.view(torch.int64).view(-1, 2).clone()  # [kind | ordinal << 32, val_offset]
    out = {}
    sparse = (d[:, 0] & 0xFFFFFFFF) == 1
    t_sp = int(torch.nonzero(sparse)[0])
    t_dn = int(torch.nonzero(~sparse)[0])
    bad = d.clone()
    bad[t_sp, 0] = 1 | (int(pw.n_sparse) << 32)  # sparse ordinal past the metadata blob
    out["ordinal"] = bad
    bad = d.clone()
    bad[t_dn, 1] += 16384 * 1000  # values offset past the values blob
    out["offset"] = bad
    bad = d.clone()
    bad[t_dn, 0] = 7  # not a tile kind
    out["kind"] = bad
    bad = d.clone()
    bad[t_sp, 0] = -(1 << 32)  # kind 0, ordinal 0xFFFFFFFF: a sparse tile relabelled dense (count, offsets off)
    out["count"] = bad
    return {k: tsg.PackedWeight(pw.N, pw.K, pw.n_sparse, pw.values, pw.meta, v.view(torch.uint8).view(-1))
            for k, v in out.items()}


def test_check_weight_release_build():
    N, K = 512, 768
    w = si.gen_w(N, K, 19, 0)
    bm = si.tiles_exact(N, K, 0.5, 19, 0)
    pw = tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(si.patterns_top2(w)))
    assert tsg.patch_read_status(tsg.patch_check_weight(pw)) == (0, 0)
    for name, bad in corruptions(pw).items():
        code, bits = tsg.patch_read_status(tsg.patch_check_weight(bad))
        assert code == 10 and bits == tsg.DEV_BOUNDS, (name, code, bits)


DEBUG_SCRIPT = r"""
import sys, torch, numpy as np
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
import tile_sparse_gemm_b200 as tsg, synth_inputs as si, oracle
from _util import to_dev, to_dev_bf16, bits_of, check_gemm
from test_gpu_debug_build import corruptions
assert "debug" in tsg.version(), tsg.version()
N, K = 512, 768
w = si.gen_w(N, K, 19, 1); bm = si.tiles_exact(N, K, 0.5, 19, 1); ids = si.patterns_top2(w)
pw = tsg.patch_pack(to_dev_bf16(w), to_dev(bm), to_dev(ids))
for M in (4, 300):  # a valid weight: decode and prefill as in the release build
    x = si.gen_x(M, K, 19, M)
    check_gemm(bits_of(tsg.patch_gemm(to_dev_bf16(x), pw)), oracle.hybrid_gemm(x, w, bm, ids), f"debug M={M}")
x4 = to_dev_bf16(si.gen_x(4, K, 19, 4))
for name, bad in corruptions(pw).items():
    for what, fn in (("decode", lambda s: tsg.patch_gemm(x4, bad, Y=y, status=s)),
                     ("simt", lambda s: tsg.patch_gemm_ex(x4, bad, Y=y, status=s, path=tsg.PATH_DECODE_SIMT)),
                     ("prefill", lambda s: tsg.patch_gemm_ex(x4, bad, Y=y, status=s, path=tsg.PATH_PREFILL)),
                     ("chain", lambda s: tsg.Chain([(x4, bad, y, True)], status=s).run()),
                     ("mlp", lambda s: tsg.patch_gemm_mlp(x4, pw, bad, H=y, status=s))):
        y = torch.zeros((4, N), dtype=torch.bfloat16, device="cuda")
        s = tsg.new_status()
        try:
            fn(s)
            raise AssertionError(f"{name}/{what}: accepted")
        except tsg.PatchError as e:
            assert e.code == 10, (name, what, e)
        torch.cuda.synchronize()
        assert int(torch.count_nonzero(y.view(torch.int16))) == 0, (name, what)  # no GEMM ran
print("debug build ok")
"""


def test_debug_build_refuses_broken_weights():
    from tile_sparse_gemm_b200 import build as tsg_build
    tsg_build.build(debug=True)
    env = dict(os.environ, TSG_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + DEBUG_SCRIPT], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "debug build ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
