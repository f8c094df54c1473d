"""The C-ABI library loads and exports every entry point include/patch.h declares
(no GPU needed: only host-side calls that launch nothing)."""
import ctypes
import re
from pathlib import Path

import pytest

import tile_sparse_gemm_b200 as tsg
from tile_sparse_gemm_b200 import build as tsg_build

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def lib():
    tsg_build.build()
    return tsg.lib()


def declared_symbols():
    text = (ROOT / "include" / "patch.h").read_text()
    return sorted(set(re.findall(r"PATCH_API\s+[\w\s\*]+?\b(patch_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 9, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in patch.h but not exported"


def test_debug_build_exports_the_same_symbols():
    path = tsg_build.build(debug=True)
    dbg = ctypes.CDLL(str(path))
    for n in declared_symbols():
        assert hasattr(dbg, n), f"{n} declared in patch.h but not exported by the debug build"
    dbg.patch_version.restype = ctypes.c_char_p
    assert b"debug" in dbg.patch_version()


def test_version_and_strerror(lib):
    assert b"sm_100a" in lib.patch_version()
    for code in range(11):
        assert lib.patch_strerror(code)
    assert lib.patch_strerror(99) == b"unknown status"


def test_pack_sizes_host_only(lib):
    assert tsg.patch_pack_sizes(512, 512, 8) == (8 * 32768 + 8 * 16384, 8 * 2048, 16 * 16)
    with pytest.raises(tsg.PatchError) as e:
        tsg.patch_pack_sizes(500, 512, 0)
    assert e.value.code == 2  # PATCH_ERR_SHAPE
    with pytest.raises(tsg.PatchError) as e:
        tsg.patch_pack_sizes(128, 128, 2)
    assert e.value.code == 1  # n_sparse > T


def test_host_checks_reject_before_any_launch(lib):
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: every call below fails its host checks first
    # bad shape
    assert lib.patch_hard_mask(fake, 100, 128, fake, fake, None, fake, fake, fake, None) == 2
    # null required pointer
    assert lib.patch_hard_mask(fake, 128, 128, None, fake, None, fake, fake, fake, None) == 1
    # misaligned pointer
    assert lib.patch_pack(P(0x10001), 128, 128, fake, fake, 0, fake, None, fake, fake, None) == 3
    # n_sparse out of range
    assert lib.patch_pack(fake, 128, 128, fake, fake, 5, fake, fake, fake, fake, None) == 1
    # gemm: bad path selector, decode path with M > 16, negative M
    w = tsg._Weight(128, 128, 0, 0x10000, None, 0x10000)
    assert lib.patch_gemm_ex(fake, 4, ctypes.byref(w), fake, None, 0, fake, None, 7, 0) == 1
    assert lib.patch_gemm_ex(fake, 17, ctypes.byref(w), fake, None, 0, fake, None, 1, 0) == 1
    assert lib.patch_gemm_ex(fake, -1, ctypes.byref(w), fake, None, 0, fake, None, 0, 0) == 1
    # the tensor-core decode path holds arrival counters for at most 4096 tile rows (N <= 524288)
    wide = tsg._Weight(128 * 4097, 128, 0, 0x10000, None, 0x10000)
    assert lib.patch_gemm_ex(fake, 4, ctypes.byref(wide), fake, None, 0, fake, None, 1, 0) == 2
    # the stall test hook is refused outside the prefill path
    assert lib.patch_gemm_ex(fake, 4, ctypes.byref(w), fake, None, 0, fake, None, 0x101, 0) == 1
    # M == 0 is a no-op that needs no device
    assert lib.patch_gemm_ex(None, 0, ctypes.byref(w), None, None, 0, fake, None, 0, 0) == 0
    # weight with a bad shape
    wbad = tsg._Weight(128, 130, 0, 0x10000, None, 0x10000)
    assert lib.patch_gemm(fake, 4, ctypes.byref(wbad), fake, None, 0, fake, None) == 2


def test_64_tile_format_host_checks(lib):
    """The 64 x 64 execution-tile calls: closed-form sizes, and host checks that
    refuse before any device query or launch."""
    assert tsg.patch_pack64_sizes(192, 320, 7) == ((15 - 7) * 8192 + 7 * 4096, 7 * 512, 16 * 15)
    assert tsg.patch_pack64_sizes(64, 64, 0) == (8192, 0, 16)
    with pytest.raises(tsg.PatchError) as e:
        tsg.patch_pack64_sizes(96, 64, 0)
    assert e.value.code == 2
    with pytest.raises(tsg.PatchError) as e:
        tsg.patch_pack64_sizes(64, 64, 2)
    assert e.value.code == 1
    P = ctypes.c_void_p
    fake = P(0x10000)
    SZ = ctypes.c_size_t
    w = tsg._Weight(192, 320, 0, 0x10000, None, 0x10000)
    # M == 0: no-op, zero workspace, no device needed
    b = SZ(123)
    assert lib.patch_gemm64_workspace_size(0, ctypes.byref(w), ctypes.byref(b)) == 0 and b.value == 0
    assert lib.patch_gemm64(None, 0, ctypes.byref(w), None, None, 0, fake, None, 0) == 0
    # bad shape, n_sparse out of range, missing metadata, misaligned blob, negative M, NULL status
    assert lib.patch_gemm64(fake, 4, ctypes.byref(tsg._Weight(192, 96 + 1, 0, 0x10000, None, 0x10000)),
                            fake, None, 0, fake, None, 0) == 2
    assert lib.patch_gemm64(fake, 4, ctypes.byref(tsg._Weight(64, 64, 2, 0x10000, 0x10000, 0x10000)),
                            fake, None, 0, fake, None, 0) == 1
    assert lib.patch_gemm64(fake, 4, ctypes.byref(tsg._Weight(64, 64, 1, 0x10000, None, 0x10000)),
                            fake, None, 0, fake, None, 0) == 1
    assert lib.patch_gemm64(fake, 4, ctypes.byref(tsg._Weight(64, 64, 0, 0x10008, None, 0x10000)),
                            fake, None, 0, fake, None, 0) == 3
    assert lib.patch_gemm64(fake, -1, ctypes.byref(w), fake, None, 0, fake, None, 0) == 1
    assert lib.patch_gemm64(fake, 4, ctypes.byref(w), fake, None, 0, None, None, 0) == 1
    # pack64: shape, n_sparse range, alignment; exec tiles: mask tile above 64
    assert lib.patch_pack64(fake, 96, 64, fake, fake, 0, fake, None, fake, fake, None) == 2
    assert lib.patch_pack64(fake, 64, 64, fake, fake, 2, fake, fake, fake, fake, None) == 1
    assert lib.patch_pack64(P(0x10002), 64, 64, fake, fake, 0, fake, None, fake, fake, None) == 3
    assert lib.patch_exec_tiles64(fake, 128, 128, 128, fake, fake, None) == 1
    assert lib.patch_exec_tiles64(fake, 96, 128, 32, fake, fake, None) == 2
    # the MMA probe takes M = 64 or 128 only
    assert lib.patch_mma_probe_m(96, 0, 10, fake, None) == 1


def test_group_host_checks(lib):
    """patch_gemm_group refuses bad calls before any device query or launch, and
    a group of empty calls is a no-op."""
    P = ctypes.c_void_p
    fake = 0x10000
    w = tsg._Weight(256, 256, 0, fake, None, fake)

    def group(*calls, status=P(fake)):
        arr = (tsg._ChainCall * len(calls))(*calls)
        return lib.patch_gemm_group(ctypes.cast(arr, P), len(calls), status, None, 0)

    assert group(tsg._ChainCall(None, None, w, 0, 0, 0)) == 0                         # empty call: no-op
    assert lib.patch_gemm_group(None, 0, P(fake), None, 0) == 0                       # no calls
    assert lib.patch_gemm_group(None, 1, P(fake), None, 0) == 1                       # NULL calls
    assert group(tsg._ChainCall(fake, fake, w, 4, 0, 0), status=None) == 1            # NULL status
    assert group(tsg._ChainCall(fake, fake, w, -1, 0, 0)) == 1                        # negative M
    assert group(tsg._ChainCall(fake, fake, w, 4, 1, 0)) == 1                         # after_previous set
    assert group(tsg._ChainCall(fake, None, w, 4, 0, 0)) == 1                         # NULL Y
    assert group(tsg._ChainCall(fake + 2, fake, w, 4, 0, 0)) == 3                     # misaligned X
    assert group(tsg._ChainCall(fake, fake, tsg._Weight(256, 200, 0, fake, None, fake), 4, 0, 0)) == 2
    # the first bad call decides, even after good ones
    assert group(tsg._ChainCall(None, None, w, 0, 0, 0), tsg._ChainCall(fake, fake, w, 4, 1, 0)) == 1


def test_shard_rows_by_refuses_an_unknown_balance(lib):
    import numpy as np
    bm = np.zeros((4, 2), np.uint8)
    out = np.zeros(3, np.int64)
    P = ctypes.c_void_p
    args = (bm.ctypes.data_as(P), 4, 2, 2)
    assert lib.patch_shard_rows_by(*args, 0, out.ctypes.data_as(P)) == 0 and list(out) == [0, 2, 4]
    assert lib.patch_shard_rows_by(*args, 1, out.ctypes.data_as(P)) == 0 and list(out) == [0, 2, 4]
    assert lib.patch_shard_rows_by(*args, 2, out.ctypes.data_as(P)) == 1
    assert lib.patch_shard_rows_by(*args, -1, out.ctypes.data_as(P)) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(tsg, "_lib", None)
    monkeypatch.setattr(tsg, "_LIB_PATH", tmp_path / "libpatch.so")
    with pytest.raises(ImportError):
        tsg.lib()


def test_packed_weight_save_load_round_trip(tmp_path):
    """save_packed / load_packed keep a packed weight's blobs bit for bit (CPU
    tensors here; the blobs are the oracle's packing of a mixed layer) and
    refuse a file whose blob sizes do not fit its shape."""
    import numpy as np
    import torch

    import oracle
    import synth_inputs as si
    N, K = 256, 384
    w = si.gen_w(N, K, 18, 0)
    bm = si.tiles_exact(N, K, 0.5, 18, 0)
    ids = si.patterns_top2(w)
    v, m, d = oracle.pack(w, bm, ids)
    pw = tsg.PackedWeight(N, K, int(bm.sum()), torch.from_numpy(v), torch.from_numpy(m), torch.from_numpy(d))
    path = tmp_path / "layer.npz"
    tsg.save_packed(pw, path)
    back = tsg.load_packed(path, device="cpu")
    assert (back.N, back.K, back.n_sparse) == (N, K, int(bm.sum()))
    for a, b in ((back.values, v), (back.meta, m), (back.desc, d)):
        assert np.array_equal(a.numpy(), b)
    bad = tsg.PackedWeight(N, K, int(bm.sum()) + 1, pw.values, pw.meta, pw.desc)
    tsg.save_packed(bad, tmp_path / "bad.npz")
    with pytest.raises(ValueError):
        tsg.load_packed(tmp_path / "bad.npz", device="cpu")
