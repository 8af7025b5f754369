"""Helpers shared by the GPU parity tests (marshalling and comparison only)."""
import numpy as np
import torch


def ws_tensor(nbytes: int, device) -> torch.Tensor:
    """Zero-filled workspace of at least nbytes (int32 storage, 256-byte aligned by the allocator)."""
    return torch.zeros(max(1, (nbytes + 3) // 4), dtype=torch.int32, device=device)


def status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def assert_ok(st: torch.Tensor) -> None:
    torch.cuda.synchronize()
    assert int(st.item()) == 0, f"device status {int(st.item())}"


def f64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))))
