"""Top-k commit kernel vs the oracle's rule on the same inputs: the commit
set, the updated tokens and mask and the commit count are bit-exact (both
sides compare the same fp32 probabilities; ties are drawn on purpose)."""
import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import oracle as O
from gpu_util import assert_ok, status

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("R", [1, 5, 16, 128])
@pytest.mark.parametrize("k", [0, 1, 3, 16, 200])
def test_topk_commit_matches_oracle(cuda, R, k):
    rng = np.random.default_rng(17 * R + k)
    p1 = rng.choice(np.array([0.05, 0.3, 0.5, 0.9, 0.91, 1.0], dtype=np.float32), R)
    masked = (rng.random(R) < 0.7).astype(np.uint8)
    ids = rng.integers(0, 151936, R).astype(np.int32)
    tokens0 = (np.arange(R) + 1000).astype(np.int32)
    m_t, tok_t = torch.from_numpy(masked).to(cuda), torch.from_numpy(tokens0).to(cuda)
    commit = torch.full((R,), 7, dtype=torch.uint8, device=cuda)
    n = torch.full((1,), -1, dtype=torch.int32, device=cuda)
    st = status(cuda)
    dv.topk_commit(torch.from_numpy(p1).to(cuda), torch.from_numpy(ids).to(cuda), m_t, tok_t, R=R, k=k,
                   commit=commit, n_commit=n, status=st)
    assert_ok(st)
    want = O.topk_commit(p1.astype(np.float64), masked.astype(bool), k)
    got = [r for r in range(R) if commit.cpu().numpy()[r]]
    assert got == want
    assert set(commit.cpu().numpy().tolist()) <= {0, 1}
    assert int(n.item()) == min(k, int(masked.sum()))
    m_after, tok_after = m_t.cpu().numpy(), tok_t.cpu().numpy()
    for r in range(R):
        if r in want:
            assert m_after[r] == 0 and tok_after[r] == ids[r]
        else:
            assert m_after[r] == masked[r] and tok_after[r] == tokens0[r]


def test_topk_commit_on_the_lm_head_outputs(cuda):
    """Composed with the fused LM head: its top-1 ids and probabilities feed
    the top-k commit in device memory, as a decode step would."""
    import dvlm_gen as gen
    from gpu_util import ws_tensor
    R, H, V, k = 16, 256, 2048, 4
    (h_t, h), (w_t, w) = gen.lmhead_case(9, R, H, V, second_set=False)
    top = torch.zeros(R, dtype=torch.int32, device=cuda)
    p1 = torch.zeros(R, dtype=torch.float32, device=cuda)
    st = status(cuda)
    dv.lmhead_conf_commit(h_t.to(cuda), w_t.to(cuda), R=R, H=H, V=V, dtype=dv.DVLM_BF16, threshold=-1.0,
                          top1_id=top, top1_prob=p1, workspace=ws_tensor(dv.lmhead_workspace_size(R, V, H, 0), cuda),
                          status=st)
    masked = torch.ones(R, dtype=torch.uint8, device=cuda)
    tokens = torch.zeros(R, dtype=torch.int32, device=cuda)
    dv.topk_commit(p1, top, masked, tokens, R=R, k=k, status=st)
    assert_ok(st)
    p1h = p1.cpu().numpy()
    want = O.topk_commit(p1h.astype(np.float64), [True] * R, k)      # the rule on the kernel's own p1
    assert [r for r in range(R) if masked.cpu().numpy()[r] == 0] == want
    conf = O.lm_head_conf(h.astype(np.float64), w.astype(np.float64))
    sure = [r for r in want if conf.p1[r] - conf.p2[r] >= 1e-3]
    assert all(int(tokens[r].item()) == int(conf.top1[r]) for r in sure)


@pytest.mark.parametrize("R", [1, 7, 16, 128])
@pytest.mark.parametrize("k", [0, 2, 5, 200])
def test_divergence_first_commit_matches_oracle(cuda, R, k):
    """FULL branch of certificate-guided routing: divergent rows first, each
    group by FULL confidence; committed rows take the FULL ids."""
    rng = np.random.default_rng(31 * R + k)
    p1 = rng.choice(np.array([0.05, 0.3, 0.5, 0.9, 0.91, 1.0], dtype=np.float32), R)
    masked = (rng.random(R) < 0.7).astype(np.uint8)
    full = rng.integers(0, 4, R).astype(np.int32)
    text = rng.integers(0, 4, R).astype(np.int32)
    tokens0 = (np.arange(R) + 1000).astype(np.int32)
    m_t, tok_t = torch.from_numpy(masked).to(cuda), torch.from_numpy(tokens0).to(cuda)
    commit = torch.full((R,), 7, dtype=torch.uint8, device=cuda)
    n = torch.full((1,), -1, dtype=torch.int32, device=cuda)
    st = status(cuda)
    dv.divergence_first_commit(torch.from_numpy(p1).to(cuda), torch.from_numpy(full).to(cuda),
                               torch.from_numpy(text).to(cuda), m_t, tok_t, R=R, k=k, commit=commit, n_commit=n,
                               status=st)
    assert_ok(st)
    want = sorted(O.divergence_first_order(full, p1.astype(np.float64), text, masked.astype(bool))[:k])
    assert [r for r in range(R) if commit.cpu().numpy()[r]] == want
    assert int(n.item()) == min(k, int(masked.sum()))
    m_after, tok_after = m_t.cpu().numpy(), tok_t.cpu().numpy()
    for r in range(R):
        if r in want:
            assert m_after[r] == 0 and tok_after[r] == full[r]
        else:
            assert m_after[r] == masked[r] and tok_after[r] == tokens0[r]


def test_routing_step_decisions_on_the_lm_head_outputs(cuda):
    """One step of certificate-guided routing on device-resident outputs:
    the FULL rows' LM head gives the anchors, the TEXT-ONLY rows' LM head
    (with those anchors and the mask) gives the certified length; the accept
    branch (top-k over the anchors with k = that length) and the FULL branch
    (divergent-first, k = 3) are then applied, each to its own copy of the
    state.  Every decision equals the oracle's routing functions applied to
    the same kernel outputs (the LM head's own parity is tested elsewhere)."""
    import dvlm_gen as gen
    from gpu_util import ws_tensor
    R, H, V, k = 16, 256, 2048, 3
    (h1_t, _), (w_t, _), (h2_t, _) = gen.lmhead_case(11, R, H, V)
    wd = w_t.to(cuda)
    ws = ws_tensor(dv.lmhead_workspace_size(R, V, H, dv.DVLM_BF16), cuda)
    st = status(cuda)
    masked_h = (np.random.default_rng(12).random(R) < 0.75).astype(np.uint8)
    masked = torch.from_numpy(masked_h).to(cuda)

    def head(h, anchors=None):
        top = torch.zeros(R, dtype=torch.int32, device=cuda)
        p1 = torch.zeros(R, dtype=torch.float32, device=cuda)
        kw = {}
        if anchors is not None:
            kw = dict(masked=masked, anchor_id=anchors[0], anchor_conf=anchors[1],
                      cert_len=torch.full((1,), -1, dtype=torch.int32, device=cuda))
        dv.lmhead_conf_commit(h.to(cuda), wd, R=R, H=H, V=V, dtype=dv.DVLM_BF16, threshold=0.9, top1_id=top,
                              top1_prob=p1, workspace=ws, status=st, **kw)
        return top, p1, kw.get("cert_len")

    a_id, a_p, _ = head(h1_t)
    t_id, t_p, cert = head(h2_t, anchors=(a_id, a_p))
    assert_ok(st)
    assert np.array_equal(masked.cpu().numpy(), masked_h)          # the TEXT-ONLY pass commits nothing
    aid, ap, tid = a_id.cpu().numpy(), a_p.cpu().numpy().astype(np.float64), t_id.cpu().numpy()
    n = int(cert.item())
    assert n == O.certificate_scan(aid, ap, tid, masked_h.astype(bool))
    tokens0 = torch.arange(R, dtype=torch.int32, device=cuda) + 1000

    m1, tok1 = masked.clone(), tokens0.clone()
    dv.topk_commit(a_p, a_id, m1, tok1, R=R, k=n, status=st)
    m2, tok2 = masked.clone(), tokens0.clone()
    dv.divergence_first_commit(a_p, a_id, t_id, m2, tok2, R=R, k=k, status=st)
    assert_ok(st)
    accept = sorted(O.certificate_order(ap, masked_h.astype(bool))[:n])
    full = sorted(O.divergence_first_order(aid, ap, tid, masked_h.astype(bool))[:k])
    for m, tok, want in ((m1, tok1, accept), (m2, tok2, full)):
        m, tok = m.cpu().numpy(), tok.cpu().numpy()
        assert [r for r in range(R) if masked_h[r] and not m[r]] == want
        assert all(tok[r] == aid[r] for r in want)
        assert all(tok[r] == 1000 + r for r in range(R) if r not in want)
