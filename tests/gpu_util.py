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


def bf16_ulp(x) -> np.ndarray:
    """Spacing of bf16 values at |x| (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def assert_bf16_close(got, want, tol=2e-2, what="", ulps=1):
    """Max abs error `tol`, plus one bf16 storage ulp of the reference: both
    sides round a nearly equal real to bf16, and where that real sits next to
    a rounding boundary the two roundings differ by one ulp (0.03125 for
    |x| in [4, 8)).  How many elements may use that allowance: a flip needs
    the two reals (which differ by delta, the fp32-against-fp64 arithmetic
    difference, at most about 3e-3 here) to straddle a boundary, probability
    delta / ulp, so at most 10% of the elements whose ulp exceeds tol (the
    only ones a flip can take past tol), or 0.1% of all elements where that
    is more.  ulps=2 for a decoder layer's output rows: the residual stream
    is stored twice per layer (after the O-projection add and after the down
    add), and a flip at the first store is carried into the second sum, whose
    rounding can flip again."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    # the larger of the two values' spacings: across a power of two the steps
    # of a flip are those of the upper binade
    ulp = bf16_ulp(np.maximum(np.abs(got), np.abs(want)))
    bad = np.argwhere(err > tol + ulps * ulp)
    detail = [(tuple(int(v) for v in i), float(got[tuple(i)]), float(want[tuple(i)]), float(err[tuple(i)]))
              for i in bad[:8]]
    assert len(bad) == 0, (what, float(err.max()), detail)
    n_allow = int(np.sum(err > tol))
    budget = max(1e-3 * err.size, 0.1 * int(np.sum(ulp > tol)))
    assert n_allow <= budget, (what, n_allow, budget, err.size)
