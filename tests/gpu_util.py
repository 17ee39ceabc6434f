"""Helpers shared by the GPU parity tests (marshalling only)."""
import numpy as np
import torch


def cuda_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def cuda_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def cuda_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def rel_fro(y: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(y.astype(np.float64) - ref) / max(np.linalg.norm(ref), 1e-300))


def assert_close_1e3(y: np.ndarray, ref: np.ndarray):
    """The W4A4/W4A16 output bar: relative Frobenius error <= 1e-3, and every
    element within 1e-3 * (|ref| + rms(ref))."""
    y = y.astype(np.float64)
    assert rel_fro(y, ref) <= 1e-3, rel_fro(y, ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bad = np.abs(y - ref) > 1e-3 * (np.abs(ref) + rms)
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:5])
