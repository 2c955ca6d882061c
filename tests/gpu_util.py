"""Helpers for the GPU parity tests (moving seeded inputs to the device and back)."""
import numpy as np
import torch


def dev():
    if not torch.cuda.is_available():
        raise RuntimeError("GPU tests need a CUDA device (B200)")
    return torch.device("cuda", 0)


def to_dev(a: np.ndarray):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(dev())


def bf16_dev(bits: np.ndarray):
    """uint16 bf16 bit patterns -> torch.bfloat16 CUDA tensor."""
    return to_dev(bits.astype(np.uint16)).view(torch.bfloat16)


def to_np(t):
    torch.cuda.synchronize()
    if t.dtype == torch.bfloat16:
        return t.view(torch.uint16).cpu().numpy()
    return t.cpu().numpy()


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))
