"""Speculative verify + longest-prefix accept + in-place KV truncation: CUDA
path vs the oracle (bit-exact: integer work)."""
import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import dvlm_gen as gen
import oracle as O
from gpu_util import assert_ok, f64, status, ws_tensor

pytestmark = pytest.mark.gpu
B = 16


def run_spec(cuda, b, V, draft, logits=None, vids=None, cache_len=None, poison=0, kc=None, vc=None, n_layers=0,
             Hkv=0, D=0, Lmax=0):
    acc = torch.full((b,), -1, dtype=torch.int32, device=cuda)
    ws = ws_tensor(dv.spec_workspace_size(b, B, V), cuda)
    st = status(cuda)
    dv.spec_verify_accept(draft_ids=draft, b=b, B=B, V=V, accept_len=acc, verify_logits=logits, verify_ids=vids,
                          cache_len=cache_len, poison_tail=poison, k_cache=kc, v_cache=vc, n_layers=n_layers,
                          Hkv=Hkv, D=D, Lmax=Lmax, workspace=ws, status=st)
    assert_ok(st)
    return acc.cpu().numpy()


def oracle_accept(logit_vals, draft):
    b = logit_vals.shape[0]
    out = []
    for i in range(b):
        top = O.confidence_from_logits(logit_vals[i].astype(np.float64)).top1
        out.append(O.prefix_accept(top, draft[i]))
    return np.array(out)


@pytest.mark.parametrize("b", [1, 8])
def test_planted_prefix_and_truncation(cuda, b):
    """Speculative configuration: B=16, verify logits [b, 16, 151936] bf16, the
    causal argmax agrees with the draft on positions < k, k ~ U{0..16}."""
    V = 151936
    logits_t, vals, top, draft, k = gen.spec_case(4, b, B, V)
    want = oracle_accept(vals, draft)
    np.testing.assert_array_equal(want, k)           # the construction plants k
    L0 = 1280
    cl = torch.full((b,), L0 + B, dtype=torch.int32, device=cuda)
    got = run_spec(cuda, b, V, torch.from_numpy(draft).to(cuda), logits=logits_t.to(cuda), cache_len=cl)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(cl.cpu().numpy(), L0 + want)


def test_ids_path_and_ties(cuda):
    b, V = 4, 1000
    rng = np.random.default_rng(1)
    vals = rng.standard_normal((b, B, V)).astype(np.float32)
    # exact ties between two ids: the lower id is the argmax
    for i in range(b):
        for j in range(B):
            a1, a2 = sorted(rng.choice(V, 2, replace=False))
            vals[i, j, a1] = vals[i, j, a2] = 9.0
    lt = torch.from_numpy(vals).to(torch.bfloat16)
    vb = f64(lt)
    top = np.stack([O.confidence_from_logits(vb[i]).top1 for i in range(b)]).astype(np.int32)
    draft = top.copy()
    ks = [0, 5, 16, 1]
    for i, kk in enumerate(ks):
        draft[i, kk:] = (top[i, kk:] + 1) % V
    got = run_spec(cuda, b, V, torch.from_numpy(draft).to(cuda), logits=lt.to(cuda))
    np.testing.assert_array_equal(got, ks)
    got = run_spec(cuda, b, V, torch.from_numpy(draft).to(cuda), vids=torch.from_numpy(top).to(cuda))
    np.testing.assert_array_equal(got, ks)


def test_poison_tail_truncates_every_layer(cuda):
    """Truncation of a 36-layer cache (2 KV heads, head_dim 128, 1280 + block
    slots): dropped slots become NaN in K and V, every other slot is intact."""
    b, V, nl, Hkv, D = 2, 4096, 36, 2, 128
    L0 = 1280
    Lmax = L0 + B
    logits_t, vals, top, draft, k = gen.spec_case(5, b, B, V)
    kc = torch.randn((nl, b, Hkv, Lmax, D), device=cuda).to(torch.bfloat16)
    vc = torch.randn((nl, b, Hkv, D, Lmax), device=cuda).to(torch.bfloat16)
    k0, v0 = kc.clone(), vc.clone()
    cl = torch.full((b,), L0 + B, dtype=torch.int32, device=cuda)
    got = run_spec(cuda, b, V, torch.from_numpy(draft).to(cuda), logits=logits_t.to(cuda), cache_len=cl, poison=1,
                   kc=kc, vc=vc, n_layers=nl, Hkv=Hkv, D=D, Lmax=Lmax)
    np.testing.assert_array_equal(got, k)
    for i in range(b):
        lo = L0 + int(k[i])
        assert torch.isnan(kc[:, i, :, lo:L0 + B].float()).all()
        assert torch.isnan(vc[:, i, :, :, lo:L0 + B].float()).all()
        assert torch.equal(kc[:, i, :, :lo], k0[:, i, :, :lo])
        assert torch.equal(vc[:, i, :, :, :lo], v0[:, i, :, :, :lo])


def test_accept_on_lm_head_logits(cuda):
    """Verify logits produced by the LM head of the fused-LM-head configuration
    (hidden [16, 2048] N(0,1), W [151936, 2048] N(0, 0.02) x 25, bf16 logits):
    the draft follows the argmax for positions < k and the runner-up after."""
    B_, V = 16, 151936
    (h_t, h), (w_t, w) = gen.lmhead_case(2, B_, 2048, V, second_set=False)
    lg = O.bf16_round(h.astype(np.float64) @ w.astype(np.float64).T)
    conf = O.confidence_from_logits(lg)
    order = np.argsort(-lg, axis=-1, kind="stable")
    k = 9
    draft = conf.top1.astype(np.int32).copy()
    draft[k:] = order[k:, 1]                      # runner-up: a different id
    logits_t = torch.from_numpy(lg.astype(np.float32)).to(torch.bfloat16).reshape(1, B_, V)
    # the bf16 cast is exact: the oracle already rounded the logits to bf16
    assert np.array_equal(logits_t.float().numpy().reshape(B_, V), lg)
    want = O.prefix_accept(conf.top1, draft)
    assert want == k
    got = run_spec(cuda, 1, V, torch.from_numpy(draft.reshape(1, B_)).to(cuda), logits=logits_t.to(cuda))
    np.testing.assert_array_equal(got, [k])
