"""Build libpatch.so in-tree with nvcc for sm_100a (B200).

    python -m tile_sparse_gemm_b200.build          # compile if sources changed
    python -m tile_sparse_gemm_b200.build --force  # always recompile
    python -m tile_sparse_gemm_b200.build --debug  # libpatch_debug.so: every GEMM entry point
                                                   # first checks its weights on the device
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIB = PKG / "libpatch.so"
LIB_DEBUG = PKG / "libpatch_debug.so"
SOURCES = ["capi.cu", "hard_mask.cu", "pack.cu", "gemm_decode.cu", "gemm_decode_tc.cu", "gemm_prefill.cu",
           "gemm_decode_noalloc.cu", "gated_mlp.cu", "gemm_decode_chain.cu", "mma_probe.cu", "validate.cu",
           "gemm64.cu"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(lib: Path) -> bool:
    if not lib.exists():
        return True
    t = lib.stat().st_mtime
    deps = [CSRC / s for s in SOURCES] + list(CSRC.glob("*.cuh")) + [INCLUDE / "patch.h"]
    return any(d.stat().st_mtime > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> Path:
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    build_dir = PKG / ("_build_debug" if debug else "_build")
    build_dir.mkdir(exist_ok=True)
    extra = ["-DPATCH_DEBUG"] if debug else []

    def compile_one(src):
        obj = build_dir / (src + ".o")
        cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-I", str(INCLUDE), "-c", str(CSRC / src), "-o", str(obj)]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        return str(obj)

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    tmp = lib.with_suffix(f".so.{os.getpid()}.tmp")
    subprocess.run([_nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", str(tmp), *objs,
                    "-lcudart"], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
