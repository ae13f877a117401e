"""Shared helpers of the GPU parity tests (comparison metrics, transfers)."""
import numpy as np
import torch

REL_FRO_TOL = 1e-3      # GEMM: relative Frobenius error vs bf16(fp64 oracle)
ATTN_ABS_TOL = 2e-3     # attention: max abs error on bf16 outputs


def cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().to("cuda")


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp64 -> nearest bf16 (via fp32 then bf16 RNE), back as fp64."""
    return torch.from_numpy(np.asarray(x, np.float64)).to(torch.float32).to(torch.bfloat16).double().numpy()


def rel_fro(got: np.ndarray, want: np.ndarray) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()
