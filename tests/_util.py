"""Helpers shared by the GPU tests: numpy bf16 bits <-> torch tensors, tolerance."""
import numpy as np
import torch

# GEMM tolerance (bf16 output, fp32 accumulation) against the fp64 oracle
REL_FRO = 5e-3
ELEM_ABS = 1e-2


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_gemm(y_bits: np.ndarray, ref: np.ndarray, what: str = ""):
    """|Y - ref|_F / |ref|_F <= 5e-3 and |Y - ref| <= 1e-2 * (1 + |ref|) elementwise."""
    y = bf16_to_f64(y_bits)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = np.abs(y - ref)
    denom = np.linalg.norm(ref)
    rel = np.linalg.norm(y - ref) / denom if denom > 0 else np.linalg.norm(y - ref)
    worst = float(np.max(err / (1.0 + np.abs(ref)))) if err.size else 0.0
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert worst <= ELEM_ABS, f"{what}: elementwise error {worst:.3e} > {ELEM_ABS} (1+|ref|)"
    return rel, worst
