"""Block-masked attention (N2N / N2C / C2C): CUDA path vs the oracle.

Bar: max abs error 2e-2 on bf16 outputs (the oracle is fp64 on the same bf16
inputs), 1e-4 on the fp32 path."""
import math

import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import dvlm_gen as gen
import oracle as O
from gpu_util import assert_ok, f64, max_abs, status

pytestmark = pytest.mark.gpu
TOL_BF16 = 2e-2


def run_attn(q, k, v, n_rows, n_clean, L, dev, dtype=dv.DVLM_BF16, Hq=16, Hkv=2, D=128):
    """q [nb, n, Hq, D]; k [nb, Hkv, Lmax, D]; v [nb, Hkv, Lmax, D] (transposed here)."""
    nb, Lmax = k.shape[0], k.shape[2]
    qd = q.to(dev).contiguous()
    kd = k.to(dev).contiguous()
    vt = v.transpose(-1, -2).contiguous().to(dev)
    out = torch.full_like(qd, float("nan"))
    st = status(dev)
    dv.block_attn(qd, out, kd, vt, n_batch=nb, n_rows=n_rows, n_clean=n_clean, L=L, Lmax=Lmax, Hq=Hq, Hkv=Hkv,
                  D=D, scale=1.0 / math.sqrt(D), dtype=dtype, status=st)
    assert_ok(st)
    return out


def oracle_attn(q, k, v, n_clean, L):
    q64, k64, v64 = f64(q), f64(k), f64(v)
    D = q64.shape[-1]
    return np.stack([O.block_attention(q64[b], k64[b], v64[b], L, n_clean, 1.0 / math.sqrt(D))
                     for b in range(q64.shape[0])])


def _pad8(n):
    return (n + 7) // 8 * 8


@pytest.mark.parametrize("B", [4, 8, 16, 32])
@pytest.mark.parametrize("L", [256, 1024, 4096])
def test_noisy_block_sweep(cuda, B, L):
    """Block-attention configuration: 16 query / 2 KV heads, head_dim 128,
    K/V/Q N(0,1), noisy block of B rows over a cache of L slots."""
    q, k, v = (t for t, _ in gen.attn_case(1, B, L, Lmax=_pad8(L + B)))
    out = run_attn(q, k, v, B, 0, L, cuda)
    err = max_abs(f64(out), oracle_attn(q, k, v, 0, L))
    assert err < TOL_BF16, err


@pytest.mark.parametrize("n_rows,n_clean,L", [(16, 16, 1280), (12, 5, 1000), (16, 16, 0), (3, 3, 37),
                                              (1, 1, 1343), (16, 8, 64), (20, 20, 100)])
def test_clean_and_mixed_rows(cuda, n_rows, n_clean, L):
    q, k, v = (t for t, _ in gen.attn_case(2, n_rows, L, Lmax=_pad8(L + n_rows) + 8))
    out = run_attn(q, k, v, n_rows, n_clean, L, cuda)
    err = max_abs(f64(out), oracle_attn(q, k, v, n_clean, L))
    assert err < TOL_BF16, err


def test_batched_problems(cuda):
    q, k, v = (t for t, _ in gen.attn_case(3, 16, 700, Lmax=720, n_batch=3))
    out = run_attn(q, k, v, 16, 4, 700, cuda)
    err = max_abs(f64(out), oracle_attn(q, k, v, 4, 700))
    assert err < TOL_BF16, err


@pytest.mark.parametrize("n_vis,L,n_rows,n_clean,nb", [(1280, 1344, 16, 0, 1), (64, 300, 16, 0, 2),
                                                       (8, 100, 4, 0, 1), (64, 64, 16, 0, 1), (128, 500, 12, 5, 1)])
def test_text_only_pass_through_offset_cache_views(cuda, n_vis, L, n_rows, n_clean, nb):
    """TEXT-ONLY pass of certificate-guided routing: cache slots 0..n_vis-1
    (the vision rows) hidden from every row, positions unchanged.  Attention
    reads no positions, so the public entry point computes it over the cache
    seen from slot n_vis: K and V^T base pointers advanced by n_vis slots
    (n_vis a multiple of 8 keeps both 16-byte aligned) and length L - n_vis.
    Lmax keeps 64 spare slots, so the last 64-key chunk of every head stays
    inside that head's rows."""
    Lmax = _pad8(L + n_rows) + 64
    q, k, v = (t for t, _ in gen.attn_case(8, n_rows, L, Lmax=Lmax, n_batch=nb))
    qd, kd = q.to(cuda).contiguous(), k.to(cuda).contiguous()
    vt = v.transpose(-1, -2).contiguous().to(cuda)
    out = torch.full_like(qd, float("nan"))
    st = status(cuda)
    D = q.shape[-1]
    dv.block_attn(qd, out, kd[:, :, n_vis:, :], vt[:, :, :, n_vis:], n_batch=nb, n_rows=n_rows, n_clean=n_clean,
                  L=L - n_vis, Lmax=Lmax, Hq=16, Hkv=2, D=D, scale=1.0 / math.sqrt(D), dtype=dv.DVLM_BF16, status=st)
    assert_ok(st)
    q64, k64, v64 = f64(q), f64(k), f64(v)
    want = np.stack([O.block_attention(q64[b], k64[b], v64[b], L, n_clean, 1.0 / math.sqrt(D), hide=n_vis)
                     for b in range(nb)])
    err = max_abs(f64(out), want)
    assert err < TOL_BF16, err


def test_slots_past_the_step_are_never_read(cuda):
    """Stale slots at or beyond L+n_rows (here NaN poison, as the speculative
    truncation leaves them) do not change any output."""
    L, n = 300, 16
    q, k, v = (t for t, _ in gen.attn_case(4, n, L, Lmax=512))
    ref = run_attn(q, k, v, n, 0, L, cuda)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, L + n:] = float("nan")
    v2[:, :, L + n:] = float("nan")
    out = run_attn(q, k2, v2, n, 0, L, cuda)
    assert torch.isfinite(out).all()
    assert torch.equal(out, ref)


def test_deterministic(cuda):
    q, k, v = (t for t, _ in gen.attn_case(5, 16, 1024, Lmax=1040))
    a = run_attn(q, k, v, 16, 0, 1024, cuda)
    b = run_attn(q, k, v, 16, 0, 1024, cuda)
    assert torch.equal(a, b)


def test_fp32_path(cuda):
    """Tiny fp32 shapes: 2 query heads, 1 KV head, head_dim 16."""
    q, k, v = (t for t, _ in gen.attn_case(6, 4, 60, Hq=2, Hkv=1, D=16, Lmax=64, dtype="f32"))
    out = run_attn(q, k, v, 4, 0, 60, cuda, dtype=dv.DVLM_FP32, Hq=2, Hkv=1, D=16)
    err = max_abs(f64(out), oracle_attn(q, k, v, 0, 60))
    assert err < 1e-4, err
    out = run_attn(q, k, v, 4, 4, 60, cuda, dtype=dv.DVLM_FP32, Hq=2, Hkv=1, D=16)
    assert max_abs(f64(out), oracle_attn(q, k, v, 4, 60)) < 1e-4


# ---------------------------------------------------------------- split form
def run_attn_split(q, k, v, n_rows, n_clean, L, dev, splits, Hq=16, Hkv=2, D=128):
    nb, Lmax = k.shape[0], k.shape[2]
    qd = q.to(dev).contiguous()
    kd = k.to(dev).contiguous()
    vt = v.transpose(-1, -2).contiguous().to(dev)
    out = torch.full_like(qd, float("nan"))
    ws = torch.zeros((dv.block_attn_split_workspace_size(nb, n_rows, Hkv, splits) + 3) // 4, dtype=torch.int32,
                     device=dev)
    st = status(dev)
    dv.block_attn_split(qd, out, kd, vt, n_batch=nb, n_rows=n_rows, n_clean=n_clean, L=L, Lmax=Lmax, Hq=Hq, Hkv=Hkv,
                        D=D, scale=1.0 / math.sqrt(D), splits=splits, workspace=ws, status=st)
    assert_ok(st)
    return out


@pytest.mark.parametrize("B,L,splits", [(16, 1344, 8), (16, 4096, 2), (4, 256, 3), (32, 1024, 5), (8, 4096, 16),
                                        (16, 0, 4)])
def test_split_attention_matches_oracle(cuda, B, L, splits):
    q, k, v = (t for t, _ in gen.attn_case(7, B, L, Lmax=_pad8(L + B)))
    out = run_attn_split(q, k, v, B, 0, L, cuda, splits)
    err = max_abs(f64(out), oracle_attn(q, k, v, 0, L))
    assert err < TOL_BF16, err


@pytest.mark.parametrize("n_rows,n_clean,L", [(16, 16, 1280), (12, 5, 1000), (3, 3, 37), (20, 20, 100)])
def test_split_attention_clean_and_mixed_rows_with_poisoned_stale_slots(cuda, n_rows, n_clean, L):
    Lmax = _pad8(L + n_rows) + 136
    q, k, v = (t for t, _ in gen.attn_case(8, n_rows, L, Lmax=Lmax))
    k[:, :, L + n_rows:] = float("nan")
    v[:, :, L + n_rows:] = float("nan")
    out = run_attn_split(q, k, v, n_rows, n_clean, L, cuda, 6)
    err = max_abs(f64(out), oracle_attn(q, k, v, n_clean, L))
    assert err < TOL_BF16, err


def test_split_attention_causal_row_independent_of_rows_in_step(cuda):
    """A causal row gives bitwise the same output in a 16-row pass (verify)
    as in a 1-row pass at its own slot (AR): chunks go to splits by absolute
    key position, so the split sums do not depend on the step's rows."""
    L, n = 1300, 16
    q, k, v = (t for t, _ in gen.attn_case(9, n, L, Lmax=_pad8(L + n)))
    full = run_attn_split(q, k, v, n, n, L, cuda, 8)
    for t in (0, 5, 15):
        one = run_attn_split(q[:, t:t + 1].contiguous(), k, v, 1, 1, L + t, cuda, 8)
        assert torch.equal(one[0, 0], full[0, t]), t


def test_split_attention_batch_of_caches(cuda):
    """36 distinct caches in one launch (one per decoder layer)."""
    B, L, nb = 16, 1024, 36
    q, k, v = (t for t, _ in gen.attn_case(10, B, L, Lmax=_pad8(L + B), n_batch=nb))
    out = run_attn_split(q, k, v, B, 0, L, cuda, 2)
    err = max_abs(f64(out), oracle_attn(q, k, v, 0, L))
    assert err < TOL_BF16, err
