"""Helpers shared by the GPU tests (marshalling only)."""
import numpy as np
import torch


def to_dev(a: np.ndarray) -> torch.Tensor:
    """uint16 BF16 patterns -> int16 CUDA tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).cuda()


def from_dev_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def blob_to_host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def blob_to_dev(b: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b, dtype=np.uint8)).cuda()


def new_flag() -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def assert_within_tolerance(y_gpu: np.ndarray, y_ref: np.ndarray, s_ref: np.ndarray, rel: float = 1e-3):
    """|y - y_ref| <= rel * sum_j |W_ij x_j| elementwise (the pass rule)."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    err = np.abs(y_gpu - y_ref)
    bound = rel * s_ref
    bad = err > bound
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} outputs outside tolerance; "
                           f"worst ratio {float((err / np.maximum(bound, 1e-300)).max()):.3g}")
    return float((err / np.maximum(s_ref, 1e-300)).max())
