"""CPU checks of the trace replay (tests/decode_replay.py) that the GPU decode
tests rely on.

A stand-in engine drives threshold, speculative and AR decoding of the tiny
fp32 model with the oracle's own forward and emits trace records in the
engine's layout.  The replay must accept its trace, and must reject the trace
of a stand-in with a planted fault: position j scored from its own row instead
of row j-1, a commit below the threshold, a forced commit of the wrong
position, an accepted prefix one too long, a wrong seed, or hidden rows off by
more than the fp32 bar.  The layer-major oracle forward used at full size must
equal the plain forward-by-forward one bit for bit."""
import copy

import numpy as np
import pytest

import dvlm_gen as gen
import oracle as O
from decode_replay import (APPEND, AR, DRAFT, NOISY, QUAD_CAND, QUAD_VERIFY, ROUTE_FULL, ROUTE_TEXT, VERIFY, Rec,
                           Replay, layer_major_hidden, parse_trace)

DIMS = gen.TINY
SEED = 4


def _model(Lmax=256):
    w = O.weights_from_generator(gen, DIMS, SEED)
    return O.OracleModel(O.dims_from(DIMS), weights=w, bf16=False, Lmax=Lmax)


def _prefilled():
    _, vis, ids = gen.decode_context(DIMS, SEED, 32, 16, 16)
    m = _model()
    s = O.prefill(m, vis.astype(np.float64), ids)
    return m, s


def _rec(kind, L, toks, msk, n_clean, R, c, tok_out, msk_out, seed_out, len_out, x):
    n = len(toks)
    top1 = np.full(16, -1, dtype=np.int32)
    p1 = np.zeros(16)
    top1[:R] = c.top1[:R]
    p1[:R] = np.float32(c.p1[:R])
    return Rec(kind=kind, L=L, n_rows=n, n_clean=n_clean, R=R, tok_in=np.array(toks, dtype=np.int32),
               msk_in=np.array(msk, dtype=bool), top1=top1, p1=p1, tok_out=np.array(tok_out, dtype=np.int32),
               msk_out=np.array(msk_out, dtype=bool), seed_out=seed_out, len_out=len_out, x=x.copy())


def standin_threshold(B=4, tau=0.9, n_new=12, fault=None):
    """Threshold decoding with the oracle's forward, recorded as the engine does."""
    m, seed = _prefilled()
    recs, out = [], []
    while len(out) < n_new:
        L = m.L
        toks = [seed] + [DIMS.mask_id] * (B - 1)
        masked = [False] + [True] * (B - 1)
        while any(masked):
            x = m.forward(m.embed(toks), L, 0)
            if fault == "hidden":
                x = x + 1e-3
            c = m.logits_conf(x)
            sh = 0 if fault == "shift0" else 1
            p1 = np.zeros(B)
            top = np.zeros(B, dtype=np.int64)
            for j in range(1, B):
                r = min(j - sh, B - 2)
                p1[j], top[j] = np.float32(c.p1[r]), c.top1[r]
            C = O.threshold_commit(p1, masked, tau)
            if fault == "extra" and len(C) < sum(masked):
                C = C + [min(j for j in range(B) if masked[j] and j not in C)]
            if fault == "force" and len(C) == 1 and p1[C[0]] < tau and sum(masked) > 1:
                C = [max(j for j in range(B) if masked[j] and j != C[0])]
            nt, nm = list(toks), list(masked)
            for j in C:
                nt[j], nm[j] = int(top[j]), False
            # the engine's LM head rows: row r holds what scores position r + 1
            cc = O.Conf(p1=np.array([p1[j + 1] for j in range(B - 1)]),
                        top1=np.array([top[j + 1] for j in range(B - 1)]), p2=None)
            recs.append(_rec(NOISY, L, toks, masked, 0, B - 1, cc, nt, nm, seed, L, x))
            toks, masked = nt, nm
        x = m.forward(m.embed(toks), L, B)
        m.L = L + B
        c = m.logits_conf(x)
        seed = int(c.top1[B - 1])
        if fault == "seed":
            seed = (seed + 1) % DIMS.vocab
        recs.append(_rec(APPEND, L, toks, [False] * B, B, B, c, toks, [False] * B, seed, m.L, x))
        out.extend(toks)
    return recs, out[:n_new]


def standin_spec(B=4, n_new=12, fault=None):
    m, seed = _prefilled()
    recs, out = [], []
    while len(out) < n_new:
        L = m.L
        toks = [seed] + [DIMS.mask_id] * (B - 1)
        x = m.forward(m.embed(toks), L, 0)
        c = m.logits_conf(x)
        draft = [seed] + [int(c.top1[j - 1]) for j in range(1, B)]
        recs.append(_rec(DRAFT, L, toks, [False] + [True] * (B - 1), 0, B - 1, c, draft, [False] * B, seed, L, x))
        x = m.forward(m.embed(draft), L, B)
        g = m.logits_conf(x)
        recs.append(_rec(VERIFY, L, draft, [False] * B, B, B, g, draft, [False] * B, seed, L + B, x))
        ver = [seed] + [int(g.top1[j - 1]) for j in range(1, B)]
        k = O.prefix_accept(ver, draft)
        if fault == "accept" and k < B:
            k += 1
        m.L = L + k
        seed = int(g.top1[k - 1])
        out.extend(draft[:k])
    return recs, out[:n_new], m.L, seed


def standin_quad(B=4, n_new=12, fault=None):
    """Quadratic self-speculative decoding with the oracle's fused forward,
    recorded as the engine does (draft, then QUAD_VERIFY / QUAD_CAND pairs)."""
    m, seed = _prefilled()
    recs, out = [], []
    L = m.L
    toks = [seed] + [DIMS.mask_id] * (B - 1)
    x = m.forward(m.embed(toks), L, 0)
    c = m.logits_conf(x)
    draft = [seed] + [int(c.top1[j - 1]) for j in range(1, B)]
    recs.append(_rec(DRAFT, L, toks, [False] + [True] * (B - 1), 0, B - 1, c, draft, [False] * B, seed, L, x))
    while len(out) < n_new:
        L = m.L
        xa = O.forward_quadratic(m, draft, L)
        g = m.logits_conf(xa[:B])
        recs.append(_rec(QUAD_VERIFY, L, draft, [False] * B, B, B, g, draft, [False] * B, draft[0], L + B, xa[:B]))
        ver = [draft[0]] + [int(g.top1[j - 1]) for j in range(1, B)]
        k = O.prefix_accept(ver, draft)
        if fault == "accept" and k < B:
            k += 1
        vk = int(g.top1[k - 1])
        blk = k if fault == "block" and k < B else k - 1
        xc = xa[B + blk * B:B + (blk + 1) * B]
        cc = m.logits_conf(xc)
        nd = [vk] + [int(cc.top1[j - 1]) for j in range(1, B)]
        recs.append(_rec(QUAD_CAND, L + k, [vk] + [DIMS.mask_id] * (B - 1), [False] + [True] * (B - 1), 0, B - 1,
                         cc, nd, [False] * B, vk, L + k, xc))
        out.extend(draft[:k])
        m.L = L + k
        draft = nd
    return recs, out[:n_new], m.L, draft[0]


def standin_route(B=4, k=1, n_vis=32, n_new=12, fault=None):
    """Certificate-guided routing with the oracle's forward, recorded as the
    engine does (FULL / TEXT-ONLY passes, then the causal append)."""
    m, seed = _prefilled()
    recs, out = [], []
    while len(out) < n_new:
        L = m.L
        toks = [seed] + [DIMS.mask_id] * (B - 1)
        masked = [False] + [True] * (B - 1)
        anc_id = anc_p1 = text_top = None

        def pass_(hide):
            x = m.forward(m.embed(toks), L, 0, hide=hide)
            c = m.logits_conf(x)
            top = np.array([-1] + [int(c.top1[j - 1]) for j in range(1, B)])
            p1 = np.array([0.0] + [float(np.float32(c.p1[j - 1])) for j in range(1, B)])
            return x, c, top, p1

        while any(masked):
            kk = min(k, sum(masked))
            if anc_id is not None:
                x, c, top, p1 = pass_(0 if fault == "sees_vision" else n_vis)
                recs.append(_rec(ROUTE_TEXT, L, toks, masked, 0, B - 1, c, toks, masked, seed, L, x))
                text_top = top
                n = O.certificate_scan(anc_id, anc_p1, text_top, masked)
                if n >= kk:
                    order = O.certificate_order(anc_p1, masked)
                    if fault == "reverse":
                        order = order[::-1]
                    for j in order[:n]:
                        toks[j], masked[j] = int(anc_id[j]), False
                    continue
            x, c, top, p1 = pass_(0)
            recs.append(_rec(ROUTE_FULL, L, toks, masked, 0, B - 1, c, toks, masked, seed, L, x))
            order = (O.certificate_order(p1, masked) if text_top is None
                     else O.divergence_first_order(top, p1, text_top, masked))
            for j in order[:kk]:
                toks[j], masked[j] = int(top[j]), False
            anc_id, anc_p1 = top, p1
        x = m.forward(m.embed(toks), L, B)
        m.L = L + B
        c = m.logits_conf(x)
        seed = int(c.top1[B - 1])
        recs.append(_rec(APPEND, L, toks, [False] * B, B, B, c, toks, [False] * B, seed, m.L, x))
        out.extend(toks)
    return recs, out[:n_new]


def standin_ar(n_new=6):
    m, seed = _prefilled()
    recs, out = [], []
    for _ in range(n_new):
        L = m.L
        x = m.forward(m.embed([seed]), L, 1)
        m.L = L + 1
        c = m.logits_conf(x)
        recs.append(_rec(AR, L, [seed], [False], 1, 1, c, [int(c.top1[0])], [False], int(c.top1[0]), m.L, x))
        out.append(seed)
        seed = int(c.top1[0])
    return recs, out


def _fp32_check(a, b, what):
    assert float(np.max(np.abs(a - b))) < 1e-4, what


def _replay(B=4, tau=0.9):
    m, s = _prefilled()
    return Replay(m, s, B, tau, decide="oracle", hidden_check=_fp32_check)


def test_replay_accepts_the_oracle_trajectories():
    recs, out = standin_threshold()
    rp = _replay()
    assert rp.threshold(recs, 12) == out and rp._next == len(recs)
    assert rp.t.commits_exact + rp.t.commits_excluded > 0 and rp.t.ids_exact > 0
    recs, out, L, s = standin_spec()
    rp = _replay()
    assert rp.speculative(recs, 12, L, s) == out and rp._next == len(recs)
    recs, out = standin_ar()
    rp = _replay()
    assert rp.autoregressive(recs, 6) == out


@pytest.mark.parametrize("fault", ["shift0", "extra", "force", "seed", "hidden"])
def test_replay_rejects_planted_threshold_faults(fault):
    tau = 1.5 if fault == "force" else 0.9     # tau > 1: every commit is a forced one
    recs, out = standin_threshold(tau=tau, fault=fault)
    sig = lambda rs: [(list(r.tok_out), list(r.top1), r.seed_out) for r in rs]
    assert sig(standin_threshold(tau=tau)[0]) != sig(recs) or fault == "hidden"   # the fault did fire
    with pytest.raises(AssertionError):
        _replay(tau=tau).threshold(recs, 12)


def test_replay_rejects_a_long_accept():
    recs, out, L, s = standin_spec(fault="accept")
    with pytest.raises(AssertionError):
        _replay().speculative(recs, 12, L, s)


def test_replay_with_gpu_rows_scores_the_recorded_rows():
    """decide='gpu': decisions are scored from the records' own rows, so a
    stand-in whose hidden rows drift (within the hidden bar) but whose
    decisions follow its own rows still passes; its decisions are then held
    to the looser secondary bar against the oracle's own rows."""
    recs, out = standin_threshold()
    recs2 = copy.deepcopy(recs)
    for r in recs2:
        r.x = r.x * (1 + 1e-7)
    m, s = _prefilled()
    rp = Replay(m, s, 4, 0.9, decide="gpu", hidden_check=_fp32_check, secondary=0.1)
    assert rp.threshold(recs2, 12) == out
    assert rp.t.secondary_checked > 0


def test_layer_major_forward_equals_sequential():
    m1, _ = _prefilled()
    m2, _ = _prefilled()
    rng = np.random.default_rng(0)
    passes = []
    L = m1.L
    for n_clean in (0, 0, 4):
        toks = rng.integers(0, DIMS.vocab, size=4)
        passes.append((m1.embed(toks), L, n_clean))
    seq = [m1.forward(x, L0, nc) for x, L0, nc in passes]
    lw = lambda l: {k: v for k, v in m2._w.items() if k.startswith(f"{l}.")}
    lm = layer_major_hidden(m2, passes, lw)
    for a, b in zip(seq, lm):
        np.testing.assert_array_equal(a, b)
    for l in range(DIMS.n_layers):
        np.testing.assert_array_equal(m1.K[l], m2.K[l])
        np.testing.assert_array_equal(m1.V[l], m2.V[l])


def test_parse_trace_layout():
    """A record written in the engine's byte layout parses back field by field."""
    H = 32
    rb = ((112 * 4 + 16 * H * 2) + 255) // 256 * 256
    raw = np.zeros(2 * rb, dtype=np.uint8)
    w = raw[rb:rb + 448].view(np.int32)
    w[0:5] = [NOISY, 70, 4, 0, 3]
    w[8:12] = [5, 9, 9, 9]
    w[24:28] = [0, 1, 1, 1]
    w[40:43] = [11, 12, 13]
    w[56:59] = np.array([0.5, 0.95, 0.25], dtype=np.float32).view(np.int32)
    w[72:76] = [5, 9, 12, 9]
    w[88:92] = [0, 1, 0, 1]
    w[104:106] = [7, 70]
    xs = np.arange(16 * H, dtype=np.float32).reshape(16, H) / 64.0   # exact in bf16
    raw[rb + 448:rb + 448 + 16 * H * 2] = (xs.view(np.uint32) >> 16).astype(np.uint16).view(np.uint8).ravel()
    r = parse_trace(raw, 2, rb, H, bf16=True)[1]
    assert (r.kind, r.L, r.n_rows, r.n_clean, r.R) == (NOISY, 70, 4, 0, 3)
    assert list(r.tok_in) == [5, 9, 9, 9] and list(r.msk_in) == [False, True, True, True]
    assert list(r.top1[:3]) == [11, 12, 13] and list(r.p1[:3]) == [0.5, float(np.float32(0.95)), 0.25]
    assert list(r.tok_out) == [5, 9, 12, 9] and list(r.msk_out) == [False, True, False, True]
    assert (r.seed_out, r.len_out) == (7, 70)
    np.testing.assert_array_equal(r.x, xs[:4])


def test_replay_quadratic_accepts_the_oracle_and_rejects_faults():
    recs, out, L, s0 = standin_quad()
    rp = _replay()
    assert rp.quadratic(recs, 12, L, s0) == out and rp._next == len(recs)
    assert rp.t.ids_exact > 0
    for fault in ("accept", "block"):
        recs, out, L, s0 = standin_quad(fault=fault)
        with pytest.raises(AssertionError):
            _replay().quadratic(recs, 12, L, s0)


def test_replay_routing_accepts_the_oracle_and_rejects_faults():
    recs, out = standin_route(B=8, k=1, n_new=24)
    rp = Replay(*_prefilled(), 8, 0.9, decide="oracle", hidden_check=_fp32_check)
    assert rp.routing(recs, 24, 1, 32) == out and rp._next == len(recs)
    kinds = [r.kind for r in recs]
    assert ROUTE_TEXT in kinds and ROUTE_FULL in kinds
    sig = lambda rs: [list(r.tok_in) for r in rs]
    for fault in ("sees_vision", "reverse"):
        bad, _ = standin_route(B=8, k=1, n_new=24, fault=fault)
        assert sig(bad) != sig(recs) or fault == "sees_vision"   # the fault did fire
        with pytest.raises(AssertionError):
            Replay(*_prefilled(), 8, 0.9, decide="oracle", hidden_check=_fp32_check).routing(bad, 24, 1, 32)
