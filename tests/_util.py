"""Small helpers shared by the tests (conversions only, no method arithmetic)."""
import numpy as np
import torch


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device, any strides) -> numpy uint16 bit patterns (contiguous copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    """uint8 / float8_e4m3fn tensor -> numpy uint8 codes (contiguous copy)."""
    assert t.dtype in (torch.uint8, torch.float8_e4m3fn)
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().to(torch.float32).numpy()


def from_u16(a: np.ndarray) -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))
