"""bf16 helpers for tests, built on torch's own conversions (not the oracle's)."""
import numpy as np
import torch


def to_u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> its uint16 storage as numpy."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def dec(u: np.ndarray) -> np.ndarray:
    """uint16 bf16 storage -> float64 (torch decode)."""
    u = np.ascontiguousarray(u).view(np.int16)
    return torch.from_numpy(u.copy()).view(torch.bfloat16).to(torch.float64).numpy()


def enc(v) -> np.ndarray:
    """float64 -> bf16 storage by torch (through fp32: may double-round, rarely)."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float64))
    return to_u16(t.to(torch.float32).to(torch.bfloat16))


def ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 units in the last place between two uint16 arrays."""
    def key(u):
        s = u.astype(np.int32)
        mag = s & 0x7FFF
        return np.where(s & 0x8000, -mag, mag)
    return np.abs(key(np.asarray(a)) - key(np.asarray(b)))
