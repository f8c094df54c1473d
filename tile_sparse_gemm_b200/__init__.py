"""B200-native PATCH hybrid tile-sparse linear layer (Y = X * W_eff^T).

Thin Python binding over the C ABI of ``libpatch.so`` (declared in
include/patch.h).  It only marshals arguments: torch supplies device memory
and the current CUDA stream, every step of the hot path runs in the
library's sm_100a kernels.  There is no CPU fallback: importing the binding
works anywhere, but every call fails loudly unless the in-tree library has
been built (``python -m tile_sparse_gemm_b200.build``) and a B200 is present.

Entry points (same names as the C ABI):
    patch_pack_sizes(N, K, n_sparse)          -> (values_bytes, meta_bytes, desc_bytes)
    patch_hard_mask(W, tile_logits, pattern_logits) -> (W_masked, bitmap, pat_id)
    patch_pack(W, bitmap, pat_id, n_sparse)   -> PackedWeight
    patch_gemm_workspace_size(M, weight)      -> bytes
    patch_gemm(X, weight)                     -> Y
    patch_gemm_ex(X, weight, path=..., wait_limit_us=...) -> Y
    patch_read_status(status)                 -> (status code, device bits)
    patch_gemm_mlp, patch_tile_kinds, patch_pack_from_logits, patch_soft_mask,
    patch_hard_mask_tiles, patch_exec_tiles, shard_rows / shard_of,
    patch_gemm_chain / Chain (a sequence of decode GEMMs in one launch; see each docstring)
    patch_gemm_group / Group (independent GEMMs of any token count in one prefill launch)
    64 x 64 execution tiles: patch_pack64_sizes, patch_exec_tiles64, patch_pack64 -> PackedWeight64,
    patch_gemm64_workspace_size, patch_gemm64; patch_mma_probe_m (M = 64 or 128 MMA rate)
Helpers of this binding: save_packed(weight, path) / load_packed(path) keep a
packed weight in one .npz file (shape, sparse-tile count, the three blobs).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from pathlib import Path

import torch

# TSG_DEBUG=1 loads the debug build (every GEMM entry point checks its weights first)
_LIB_PATH = Path(__file__).resolve().parent / ("libpatch_debug.so" if os.environ.get("TSG_DEBUG") == "1"
                                               else "libpatch.so")

TILE = 128
PANEL_BYTES = 16384
DECODE_MAX_M = 16
MASK_TILES = (4, 8, 16, 32, 64, 128)  # mask tile sizes patch_hard_mask_tiles takes

PATCH_OK = 0
STATUS_NAMES = {0: "PATCH_OK", 1: "PATCH_ERR_INVALID_ARG", 2: "PATCH_ERR_SHAPE", 3: "PATCH_ERR_ALIGN",
                4: "PATCH_ERR_DEVICE", 5: "PATCH_ERR_CUDA", 6: "PATCH_ERR_BAD_PATTERN",
                7: "PATCH_ERR_TIMEOUT", 8: "PATCH_ERR_WORKSPACE", 9: "PATCH_ERR_COUNT", 10: "PATCH_ERR_BOUNDS"}
DEV_BAD_PATTERN, DEV_TIMEOUT, DEV_COUNT, DEV_BOUNDS = 0x1, 0x2, 0x4, 0x8
PATH_AUTO, PATH_DECODE, PATH_PREFILL, PATH_DECODE_SIMT, PATH_TEST_STALL = 0, 1, 2, 3, 0x100


class PatchError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)} ({_strerror(code)})")


class _Weight(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64), ("n_sparse", ctypes.c_int64),
                ("values", ctypes.c_void_p), ("meta", ctypes.c_void_p), ("desc", ctypes.c_void_p)]


class _ChainCall(ctypes.Structure):
    _fields_ = [("X", ctypes.c_void_p), ("Y", ctypes.c_void_p), ("W", _Weight), ("M", ctypes.c_int64),
                ("after_previous", ctypes.c_int32), ("reserved", ctypes.c_int32)]


CHAIN_MAX_CALLS = 64  # calls per launch of patch_gemm_chain (longer chains take several launches)
GROUP_MAX_CALLS = 32  # calls per launch of patch_gemm_group


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libpatch.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not _LIB_PATH.exists():
            raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m tile_sparse_gemm_b200.build`")
        L = ctypes.CDLL(str(_LIB_PATH))
        P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        WP = ctypes.POINTER(_Weight)
        sigs = {
            "patch_pack_sizes": [I64, I64, I64, ctypes.POINTER(SZ), ctypes.POINTER(SZ), ctypes.POINTER(SZ)],
            "patch_hard_mask": [P, I64, I64, P, P, P, P, P, P, P],
            "patch_pack": [P, I64, I64, P, P, I64, P, P, P, P, P],
            "patch_tile_kinds": [P, I64, I64, P, P, P],
            "patch_hard_mask_tiles": [P, I64, I64, I64, P, P, P, P, P, P, P],
            "patch_exec_tiles": [P, I64, I64, I64, P, P, P],
            "patch_soft_mask": [P, I64, I64, P, P, P, P, ctypes.c_float, P, P, P],
            "patch_shard_rows": [P, I64, I64, I64, P],
            "patch_shard_rows_by": [P, I64, I64, I64, I64, P],
            "patch_pack_from_logits": [P, I64, I64, P, P, I64, P, P, P, P, P],
            "patch_gemm_workspace_size": [I64, WP, ctypes.POINTER(SZ)],
            "patch_gemm": [P, I64, WP, P, P, SZ, P, P],
            "patch_gemm_ex": [P, I64, WP, P, P, SZ, P, P, I32, ctypes.c_uint64],
            "patch_read_status": [P, P, ctypes.POINTER(ctypes.c_int32)],
            "patch_gemm_mlp_workspace_size": [I64, WP, WP, ctypes.POINTER(SZ)],
            "patch_gemm_mlp": [P, I64, WP, WP, P, P, SZ, P, P],
            "patch_gemm_chain_workspace_size": [P, I64, ctypes.POINTER(SZ)],
            "patch_gemm_chain": [P, I64, P, SZ, P, P, ctypes.c_uint64],
            "patch_gemm_group": [P, I64, P, P, ctypes.c_uint64],
            "patch_mma_probe": [I32, I64, P, P],
            "patch_mma_probe_m": [I32, I32, I64, P, P],
            "patch_pack64_sizes": [I64, I64, I64, ctypes.POINTER(SZ), ctypes.POINTER(SZ), ctypes.POINTER(SZ)],
            "patch_exec_tiles64": [P, I64, I64, I64, P, P, P],
            "patch_pack64": [P, I64, I64, P, P, I64, P, P, P, P, P],
            "patch_gemm64_workspace_size": [I64, WP, ctypes.POINTER(SZ)],
            "patch_gemm64": [P, I64, WP, P, P, SZ, P, P, ctypes.c_uint64],
            "patch_check_weight": [WP, P, P],
        }
        for name, args in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = I32
        L.patch_strerror.argtypes = [I32]
        L.patch_strerror.restype = ctypes.c_char_p
        L.patch_version.argtypes = []
        L.patch_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _strerror(code: int) -> str:
    try:
        return lib().patch_strerror(code).decode()
    except Exception:  # the library itself may be what is missing
        return "?"


def _check(code: int, what: str):
    if code != PATCH_OK:
        raise PatchError(code, what)


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor | None, name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def new_status(device=None) -> torch.Tensor:
    """A zeroed device status word for the kernels to OR error bits into."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


@dataclass
class PackedWeight:
    """A packed hybrid weight: three device blobs plus its shape."""
    N: int
    K: int
    n_sparse: int
    values: torch.Tensor  # uint8, patch_pack_sizes bytes
    meta: torch.Tensor    # uint8 (may be empty)
    desc: torch.Tensor    # uint8, 16 bytes per tile

    def struct(self) -> _Weight:
        return _Weight(self.N, self.K, self.n_sparse, self.values.data_ptr(),
                       self.meta.data_ptr() if self.meta.numel() else None, self.desc.data_ptr())

    @property
    def stored_bytes(self) -> int:
        return self.values.numel() + self.meta.numel() + self.desc.numel()


def patch_pack_sizes(N: int, K: int, n_sparse: int) -> tuple[int, int, int]:
    v, m, d = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().patch_pack_sizes(N, K, n_sparse, ctypes.byref(v), ctypes.byref(m), ctypes.byref(d)),
           "patch_pack_sizes")
    return v.value, m.value, d.value


_PACKED_FORMAT = 1  # version of the saved layout below


def save_packed(weight: PackedWeight, path) -> None:
    """Write a packed weight to one .npz file: its shape, sparse-tile count and
    the three blobs as bytes (pack once offline, load at serving time)."""
    import numpy as np
    np.savez(path, format=_PACKED_FORMAT, N=weight.N, K=weight.K, n_sparse=weight.n_sparse,
             values=weight.values.cpu().numpy(), meta=weight.meta.cpu().numpy(), desc=weight.desc.cpu().numpy())


def load_packed(path, device="cuda", check: bool = True) -> PackedWeight:
    """Read a packed weight written by save_packed onto `device`, checking the
    blob sizes against patch_pack_sizes for its shape and sparse-tile count and,
    with `check` on a CUDA device, its descriptor table (patch_check_weight)."""
    import numpy as np
    with np.load(path) as f:
        if int(f["format"]) != _PACKED_FORMAT:
            raise ValueError(f"{path}: packed-weight format {int(f['format'])}, expected {_PACKED_FORMAT}")
        N, K, n_sparse = int(f["N"]), int(f["K"]), int(f["n_sparse"])
        blobs = {k: np.ascontiguousarray(f[k], dtype=np.uint8) for k in ("values", "meta", "desc")}
    sizes = dict(zip(("values", "meta", "desc"), patch_pack_sizes(N, K, n_sparse)))
    for k, b in blobs.items():
        if b.size != sizes[k]:
            raise ValueError(f"{path}: {k} blob has {b.size} bytes, a packed {N}x{K} weight with "
                             f"{n_sparse} sparse tiles has {sizes[k]}")
    t = {k: torch.from_numpy(b).to(device) for k, b in blobs.items()}
    w = PackedWeight(N, K, n_sparse, t["values"], t["meta"], t["desc"])
    if check and torch.device(device).type == "cuda":
        code, bits = patch_read_status(patch_check_weight(w))
        if code != PATCH_OK:
            raise PatchError(code, f"{path}: descriptor table")
    return w


def patch_hard_mask(W: torch.Tensor | None, tile_logits: torch.Tensor, pattern_logits: torch.Tensor,
                    status: torch.Tensor | None = None, want_masked: bool = True, stream=None):
    """Argmax hard mask.  Returns (W_masked or None, bitmap u8 [Tn][Tk], pat_id u8 [N][K/4])."""
    N, K4, _ = pattern_logits.shape
    K = 4 * K4
    dev = pattern_logits.device
    status = new_status(dev) if status is None else status
    wm = torch.empty((N, K), dtype=torch.bfloat16, device=dev) if want_masked else None
    bitmap = torch.empty((N // TILE, K // TILE), dtype=torch.uint8, device=dev)
    pid = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
    _check(lib().patch_hard_mask(_dev(W, "W"), N, K, _dev(tile_logits, "tile_logits"),
                                 _dev(pattern_logits, "pattern_logits"), _dev(wm, "W_masked"),
                                 _dev(bitmap, "bitmap"), _dev(pid, "pat_id"), _dev(status, "status"),
                                 _stream(stream)), "patch_hard_mask")
    return wm, bitmap, pid


def patch_hard_mask_tiles(W: torch.Tensor | None, tile_logits: torch.Tensor, pattern_logits: torch.Tensor,
                          mask_tile: int, status: torch.Tensor | None = None, want_masked: bool = True,
                          stream=None):
    """Argmax hard mask with b x b mask tiles (b = mask_tile, 4..128): tile_logits
    fp32 [N/b][K/b][2].  Returns (W_masked or None, bitmap u8 [N/b][K/b], pat_id u8 [N][K/4])."""
    N, K4, _ = pattern_logits.shape
    K = 4 * K4
    b = int(mask_tile)
    dev = pattern_logits.device
    status = new_status(dev) if status is None else status
    wm = torch.empty((N, K), dtype=torch.bfloat16, device=dev) if want_masked else None
    shape = (N // b, K // b) if b in MASK_TILES else (1,)  # the library rejects other sizes
    bitmap = torch.empty(shape, dtype=torch.uint8, device=dev)
    pid = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
    _check(lib().patch_hard_mask_tiles(_dev(W, "W"), N, K, b, _dev(tile_logits, "tile_logits"),
                                       _dev(pattern_logits, "pattern_logits"), _dev(wm, "W_masked"),
                                       _dev(bitmap, "bitmap"), _dev(pid, "pat_id"), _dev(status, "status"),
                                       _stream(stream)), "patch_hard_mask_tiles")
    return wm, bitmap, pid


def patch_exec_tiles(bitmap: torch.Tensor, N: int, K: int, mask_tile: int,
                     stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """128 x 128 execution tiles of a b x b mask bitmap (sparse only where every
    mask tile inside is sparse): (exec u8 [N/128][K/128], n_sparse int64 [1]), on the device."""
    dev = bitmap.device
    ex = torch.empty((N // TILE, K // TILE), dtype=torch.uint8, device=dev)
    n_sparse = torch.empty(1, dtype=torch.int64, device=dev)
    _check(lib().patch_exec_tiles(_dev(bitmap, "bitmap"), N, K, int(mask_tile), _dev(ex, "exec"),
                                  _dev(n_sparse, "n_sparse"), _stream(stream)), "patch_exec_tiles")
    return ex, n_sparse


def patch_pack(W: torch.Tensor, bitmap: torch.Tensor, pat_id: torch.Tensor, n_sparse: int | None = None,
               status: torch.Tensor | None = None, stream=None) -> PackedWeight:
    """Pack W (bf16 [N][K]) under a tile bitmap and pattern ids into the mixed layout."""
    N, K = W.shape
    if n_sparse is None:
        n_sparse = int(torch.count_nonzero(bitmap).item())
    vb, mb, db = patch_pack_sizes(N, K, n_sparse)
    dev = W.device
    status = new_status(dev) if status is None else status
    values = torch.empty(vb, dtype=torch.uint8, device=dev)
    meta = torch.empty(mb, dtype=torch.uint8, device=dev)
    desc = torch.empty(db, dtype=torch.uint8, device=dev)
    _check(lib().patch_pack(_dev(W, "W"), N, K, _dev(bitmap, "bitmap"), _dev(pat_id, "pat_id"), n_sparse,
                            _dev(values, "values"), _dev(meta, "meta") if mb else None, _dev(desc, "desc"),
                            _dev(status, "status"), _stream(stream)), "patch_pack")
    return PackedWeight(N, K, n_sparse, values, meta, desc)


def patch_soft_mask(W: torch.Tensor, tile_logits: torch.Tensor, pattern_logits: torch.Tensor, tau: float,
                    tile_noise: torch.Tensor | None = None, pattern_noise: torch.Tensor | None = None,
                    want_mask: bool = True, stream=None):
    """Training-time hybrid mask: (W_soft bf16 [N][K], M fp32 [N][K] or None)."""
    N, K = W.shape
    dev = W.device
    w_soft = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    mask = torch.empty((N, K), dtype=torch.float32, device=dev) if want_mask else None
    _check(lib().patch_soft_mask(_dev(W, "W"), N, K, _dev(tile_logits, "tile_logits"),
                                 _dev(tile_noise, "tile_noise"), _dev(pattern_logits, "pattern_logits"),
                                 _dev(pattern_noise, "pattern_noise"), float(tau), _dev(w_soft, "W_soft"),
                                 _dev(mask, "mask"), _stream(stream)), "patch_soft_mask")
    return w_soft, mask


def patch_tile_kinds(tile_logits: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Tile kinds (argmax of the 2 tile logits, ties -> dense) of fp32
    tile_logits [Tn][Tk][2]: (bitmap u8 [Tn][Tk], n_sparse int64 [1]), both on
    the device."""
    Tn, Tk, two = tile_logits.shape
    if two != 2:
        raise ValueError("tile_logits must be [Tn][Tk][2]")
    dev = tile_logits.device
    bitmap = torch.empty((Tn, Tk), dtype=torch.uint8, device=dev)
    n_sparse = torch.empty(1, dtype=torch.int64, device=dev)
    _check(lib().patch_tile_kinds(_dev(tile_logits, "tile_logits"), Tn * 128, Tk * 128, _dev(bitmap, "bitmap"),
                                  _dev(n_sparse, "n_sparse"), _stream(stream)), "patch_tile_kinds")
    return bitmap, n_sparse


def patch_pack_from_logits(W: torch.Tensor, bitmap: torch.Tensor, pattern_logits: torch.Tensor,
                           n_sparse: int | None = None, status: torch.Tensor | None = None,
                           stream=None) -> PackedWeight:
    """Hard mask and pack in one pass: like patch_pack, with each sparse tile's
    pattern ids the argmax of its pattern logits (fp32 [N][K/4][6])."""
    N, K = W.shape
    if n_sparse is None:
        n_sparse = int(torch.count_nonzero(bitmap).item())
    vb, mb, db = patch_pack_sizes(N, K, n_sparse)
    dev = W.device
    status = new_status(dev) if status is None else status
    values = torch.empty(vb, dtype=torch.uint8, device=dev)
    meta = torch.empty(mb, dtype=torch.uint8, device=dev)
    desc = torch.empty(db, dtype=torch.uint8, device=dev)
    _check(lib().patch_pack_from_logits(_dev(W, "W"), N, K, _dev(bitmap, "bitmap"),
                                        _dev(pattern_logits, "pattern_logits"), n_sparse, _dev(values, "values"),
                                        _dev(meta, "meta") if mb else None, _dev(desc, "desc"),
                                        _dev(status, "status"), _stream(stream)), "patch_pack_from_logits")
    return PackedWeight(N, K, n_sparse, values, meta, desc)


def patch_gemm_workspace_size(M: int, weight: PackedWeight) -> int:
    b = ctypes.c_size_t()
    st = weight.struct()
    _check(lib().patch_gemm_workspace_size(M, ctypes.byref(st), ctypes.byref(b)), "patch_gemm_workspace_size")
    return b.value


def patch_gemm_ex(X: torch.Tensor, weight: PackedWeight, Y: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                  path: int = PATH_AUTO, wait_limit_us: int = 0, stream=None) -> torch.Tensor:
    M, K = X.shape
    if K != weight.K:
        raise ValueError(f"X has K={K}, weight has K={weight.K}")
    dev = X.device
    if Y is None:
        Y = torch.empty((M, weight.N), dtype=torch.bfloat16, device=dev)
    status = new_status(dev) if status is None else status
    st = weight.struct()
    if workspace is None:
        need = patch_gemm_workspace_size(M, weight)  # covers every path M can take
        workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)  # must start zero-filled
    _check(lib().patch_gemm_ex(_dev(X, "X"), M, ctypes.byref(st), _dev(Y, "Y"), _dev(workspace, "workspace"),
                               workspace.numel(), _dev(status, "status"), _stream(stream), path, wait_limit_us),
           "patch_gemm")
    return Y


def patch_gemm(X: torch.Tensor, weight: PackedWeight, Y: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """Y = X * W_eff^T (bf16 out, fp32 accumulate); M <= 16 decode path, else prefill.

    Every call runs on the current stream and launches only libpatch kernels, so a
    sequence of calls can be captured in a CUDA graph (after one eager call)."""
    return patch_gemm_ex(X, weight, Y, workspace, status, PATH_AUTO, 0, stream)


class Chain:
    """A fixed sequence of decode GEMMs (M <= 16 each) for patch_gemm_chain.

    calls: list of (X, weight, Y, after_previous) with X bf16 [M][K], Y bf16
    [M][N] (device tensors; Y None allocates it) and after_previous True when
    X is written by an earlier call of the chain (the call then reads X only
    after every earlier call has completed).  The ctypes array of calls and a
    zero-filled workspace are built once; run() launches the chain on the
    current stream (capturable in a CUDA graph after one eager run)."""

    def __init__(self, calls, workspace: torch.Tensor | None = None, status: torch.Tensor | None = None):
        self.Y = []
        arr = (_ChainCall * len(calls))()
        self._keep = []
        for j, (X, weight, Y, after) in enumerate(calls):
            M, K = X.shape
            if K != weight.K:
                raise ValueError(f"call {j}: X has K={K}, weight has K={weight.K}")
            if Y is None:
                Y = torch.empty((M, weight.N), dtype=torch.bfloat16, device=X.device)
            arr[j] = _ChainCall(_dev(X, "X") if M else None, _dev(Y, "Y") if M else None, weight.struct(), M,
                                1 if after else 0, 0)
            self.Y.append(Y)
            self._keep += [X, Y, weight]
        self.calls = arr
        self.n = len(calls)
        b = ctypes.c_size_t()
        _check(lib().patch_gemm_chain_workspace_size(ctypes.cast(arr, ctypes.c_void_p), self.n, ctypes.byref(b)),
               "patch_gemm_chain_workspace_size")
        dev = calls[0][0].device if calls else None
        if workspace is None:
            workspace = torch.zeros(max(b.value, 16), dtype=torch.uint8, device=dev)  # must start zero-filled
        elif workspace.numel() < b.value:
            raise ValueError(f"workspace of {workspace.numel()} bytes < {b.value} needed")
        self.workspace = workspace
        self.status = new_status(dev) if status is None else status

    @property
    def workspace_bytes(self) -> int:
        return self.workspace.numel()

    def run(self, wait_limit_us: int = 0, stream=None):
        _check(lib().patch_gemm_chain(ctypes.cast(self.calls, ctypes.c_void_p), self.n, _dev(self.workspace, "workspace"),
                                      self.workspace.numel(), _dev(self.status, "status"), _stream(stream),
                                      wait_limit_us), "patch_gemm_chain")
        return self.Y


def patch_gemm_chain(calls, workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                     wait_limit_us: int = 0, stream=None) -> list[torch.Tensor]:
    """One launch (per 64 calls) of a sequence of decode GEMMs: see Chain."""
    return Chain(calls, workspace, status).run(wait_limit_us, stream)


class Group:
    """A fixed set of independent GEMMs (any token counts) for patch_gemm_group.

    calls: list of (X, weight, Y) with X bf16 [M][K] and Y bf16 [M][N] device
    tensors (Y None allocates it); no call may write memory another call reads
    or writes.  The ctypes array of calls is built once; run() launches the
    group on the current stream (capturable in a CUDA graph after one eager run)."""

    def __init__(self, calls, status: torch.Tensor | None = None):
        self.Y = []
        arr = (_ChainCall * len(calls))()
        self._keep = []
        for j, (X, weight, Y) in enumerate(calls):
            M, K = X.shape
            if K != weight.K:
                raise ValueError(f"call {j}: X has K={K}, weight has K={weight.K}")
            if Y is None:
                Y = torch.empty((M, weight.N), dtype=torch.bfloat16, device=X.device)
            arr[j] = _ChainCall(_dev(X, "X") if M else None, _dev(Y, "Y") if M else None, weight.struct(), M, 0, 0)
            self.Y.append(Y)
            self._keep += [X, Y, weight]
        self.calls = arr
        self.n = len(calls)
        dev = calls[0][0].device if calls else None
        self.status = new_status(dev) if status is None else status

    def run(self, wait_limit_us: int = 0, stream=None):
        _check(lib().patch_gemm_group(ctypes.cast(self.calls, ctypes.c_void_p), self.n, _dev(self.status, "status"),
                                      _stream(stream), wait_limit_us), "patch_gemm_group")
        return self.Y


def patch_gemm_group(calls, status: torch.Tensor | None = None, wait_limit_us: int = 0,
                     stream=None) -> list[torch.Tensor]:
    """One prefill launch (per 32 calls) of independent GEMMs: see Group."""
    return Group(calls, status).run(wait_limit_us, stream)


def patch_gemm_mlp(X: torch.Tensor, gate: PackedWeight, up: PackedWeight, H: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """H = silu(X W_gate^T) * (X W_up^T) (bf16 [M][N]) on two packed weights of one shape."""
    M, K = X.shape
    if K != gate.K or (gate.N, gate.K) != (up.N, up.K):
        raise ValueError("X, gate and up shapes disagree")
    dev = X.device
    if H is None:
        H = torch.empty((M, gate.N), dtype=torch.bfloat16, device=dev)
    status = new_status(dev) if status is None else status
    sg, su = gate.struct(), up.struct()
    if workspace is None:
        b = ctypes.c_size_t()
        _check(lib().patch_gemm_mlp_workspace_size(M, ctypes.byref(sg), ctypes.byref(su), ctypes.byref(b)),
               "patch_gemm_mlp_workspace_size")
        workspace = torch.zeros(max(b.value, 16), dtype=torch.uint8, device=dev)  # must start zero-filled
    _check(lib().patch_gemm_mlp(_dev(X, "X"), M, ctypes.byref(sg), ctypes.byref(su), _dev(H, "H"),
                                _dev(workspace, "workspace"), workspace.numel(), _dev(status, "status"),
                                _stream(stream)), "patch_gemm_mlp")
    return H


SHARD_BY = {"bytes": 0, "flops": 1}  # PATCH_SHARD_BY_BYTES / PATCH_SHARD_BY_FLOPS


def shard_rows(bitmap, n_shards: int, by: str = "bytes") -> list[tuple[int, int]]:
    """Column-parallel split of a layer into n_shards contiguous tile-row ranges
    (host computation): [(row_begin, row_end), ...], balanced by stored bytes
    (by="bytes": decode) or by the tensor cores' work (by="flops": prefill, a
    dense tile counting twice a sparse one)."""
    import numpy as np
    bm = np.ascontiguousarray(bitmap.cpu().numpy() if isinstance(bitmap, torch.Tensor) else bitmap, dtype=np.uint8)
    Tn, Tk = bm.shape
    out = np.zeros(n_shards + 1, dtype=np.int64)
    _check(lib().patch_shard_rows_by(bm.ctypes.data_as(ctypes.c_void_p), Tn, Tk, n_shards, SHARD_BY[by],
                                     out.ctypes.data_as(ctypes.c_void_p)), "patch_shard_rows_by")
    return [(int(out[i]), int(out[i + 1])) for i in range(n_shards)]


def shard_of(W: torch.Tensor, bitmap: torch.Tensor, pat_id: torch.Tensor, rows: tuple[int, int]):
    """Views of one shard's W rows, bitmap rows and pattern-id rows (no copy)."""
    b, e = rows
    return W[b * 128:e * 128], bitmap[b:e], pat_id[b * 128:e * 128]


def patch_mma_probe(sparse: bool, iters: int, status: torch.Tensor | None = None, stream=None) -> None:
    """Launch the tensor-core MMA rate probe (dense or 2:4 sparse rounds of four
    M = 128, N = 240 MMAs per SM on shared-memory operands); time it with CUDA
    events on the stream.  FLOPs per launch: SMs x iters x 4 x 2 x 128 x 240 x
    (32 if sparse else 16), dense-equivalent."""
    status = new_status() if status is None else status
    _check(lib().patch_mma_probe(1 if sparse else 0, iters, _dev(status, "status"), _stream(stream)),
           "patch_mma_probe")


def patch_check_weight(weight: PackedWeight, status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Check a packed weight's descriptor table on the device (tile kinds, sparse
    ordinals, values offsets, sparse-tile count); a violation sets DEV_BOUNDS in
    the returned status word (read it with patch_read_status)."""
    status = new_status(weight.desc.device) if status is None else status
    st = weight.struct()
    _check(lib().patch_check_weight(ctypes.byref(st), _dev(status, "status"), _stream(stream)), "patch_check_weight")
    return status


def patch_read_status(status: torch.Tensor, stream=None) -> tuple[int, int]:
    """Synchronise the stream and decode the status word: (status code, raw bits)."""
    bits = ctypes.c_int32()
    code = lib().patch_read_status(_dev(status, "status"), _stream(stream), ctypes.byref(bits))
    return code, bits.value


def version() -> str:
    return lib().patch_version().decode()


# ---- 64 x 64 execution tiles ("Ablation Studies", tile size)

TILE64 = 64


@dataclass
class PackedWeight64:
    """A weight packed in the 64 x 64 execution-tile format (patch_pack64)."""
    N: int
    K: int
    n_sparse: int
    values: torch.Tensor  # uint8, patch_pack64_sizes bytes
    meta: torch.Tensor    # uint8 (may be empty)
    desc: torch.Tensor    # uint8, 16 bytes per 64 x 64 tile

    def struct(self) -> _Weight:  # patch_weight64 has patch_weight's layout
        return _Weight(self.N, self.K, self.n_sparse, self.values.data_ptr(),
                       self.meta.data_ptr() if self.meta.numel() else None, self.desc.data_ptr())

    @property
    def stored_bytes(self) -> int:
        return self.values.numel() + self.meta.numel() + self.desc.numel()


def patch_pack64_sizes(N: int, K: int, n_sparse: int) -> tuple[int, int, int]:
    v, m, d = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().patch_pack64_sizes(N, K, n_sparse, ctypes.byref(v), ctypes.byref(m), ctypes.byref(d)),
           "patch_pack64_sizes")
    return v.value, m.value, d.value


def patch_exec_tiles64(bitmap: torch.Tensor, N: int, K: int, mask_tile: int,
                       stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """64 x 64 execution tiles of a b x b mask bitmap (b <= 64): (exec u8 [N/64][K/64],
    n_sparse int64 [1]), on the device."""
    dev = bitmap.device
    ex = torch.empty((N // TILE64, K // TILE64), dtype=torch.uint8, device=dev)
    n_sparse = torch.empty(1, dtype=torch.int64, device=dev)
    _check(lib().patch_exec_tiles64(_dev(bitmap, "bitmap"), N, K, int(mask_tile), _dev(ex, "exec"),
                                    _dev(n_sparse, "n_sparse"), _stream(stream)), "patch_exec_tiles64")
    return ex, n_sparse


def patch_pack64(W: torch.Tensor, bitmap: torch.Tensor, pat_id: torch.Tensor, n_sparse: int | None = None,
                 status: torch.Tensor | None = None, stream=None) -> PackedWeight64:
    """Pack W (bf16 [N][K]) under a 64 x 64 execution bitmap and pattern ids."""
    N, K = W.shape
    if n_sparse is None:
        n_sparse = int(torch.count_nonzero(bitmap).item())
    vb, mb, db = patch_pack64_sizes(N, K, n_sparse)
    dev = W.device
    status = new_status(dev) if status is None else status
    values = torch.empty(vb, dtype=torch.uint8, device=dev)
    meta = torch.empty(mb, dtype=torch.uint8, device=dev)
    desc = torch.empty(db, dtype=torch.uint8, device=dev)
    _check(lib().patch_pack64(_dev(W, "W"), N, K, _dev(bitmap, "bitmap"), _dev(pat_id, "pat_id"), n_sparse,
                              _dev(values, "values"), _dev(meta, "meta") if mb else None, _dev(desc, "desc"),
                              _dev(status, "status"), _stream(stream)), "patch_pack64")
    return PackedWeight64(N, K, n_sparse, values, meta, desc)


def patch_gemm64_workspace_size(M: int, weight: PackedWeight64) -> int:
    b = ctypes.c_size_t()
    st = weight.struct()
    _check(lib().patch_gemm64_workspace_size(M, ctypes.byref(st), ctypes.byref(b)), "patch_gemm64_workspace_size")
    return b.value


def patch_gemm64(X: torch.Tensor, weight: PackedWeight64, Y: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                 wait_limit_us: int = 0, stream=None) -> torch.Tensor:
    """Y = X * W_eff^T for a 64 x 64 packed weight (bf16 out, fp32 accumulate), any M."""
    if not isinstance(weight, PackedWeight64):
        raise TypeError("patch_gemm64 takes a PackedWeight64 (patch_pack64)")
    M, K = X.shape
    if K != weight.K:
        raise ValueError(f"X has K={K}, weight has K={weight.K}")
    dev = X.device
    if Y is None:
        Y = torch.empty((M, weight.N), dtype=torch.bfloat16, device=dev)
    status = new_status(dev) if status is None else status
    st = weight.struct()
    if workspace is None:
        workspace = torch.zeros(max(patch_gemm64_workspace_size(M, weight), 16), dtype=torch.uint8, device=dev)
    _check(lib().patch_gemm64(_dev(X, "X"), M, ctypes.byref(st), _dev(Y, "Y"), _dev(workspace, "workspace"),
                              workspace.numel(), _dev(status, "status"), _stream(stream), wait_limit_us),
           "patch_gemm64")
    return Y


def patch_mma_probe_m(m: int, sparse: bool, iters: int, status: torch.Tensor | None = None, stream=None) -> None:
    """patch_mma_probe for MMA shape M = 64 or 128: FLOPs per launch SMs x iters x 4 x 2 x m x 240 x
    (32 if sparse else 16), dense-equivalent."""
    status = new_status() if status is None else status
    _check(lib().patch_mma_probe_m(int(m), 1 if sparse else 0, iters, _dev(status, "status"), _stream(stream)),
           "patch_mma_probe_m")
