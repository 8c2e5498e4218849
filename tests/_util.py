"""Small helpers shared by the tests (no method arithmetic)."""
import numpy as np
import torch


def f32(t: torch.Tensor) -> np.ndarray:
    """Exact decode of a bf16 (or fp32) torch tensor into a float32 numpy array."""
    return t.detach().cpu().float().numpy()


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest even) and decode back to float64."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
