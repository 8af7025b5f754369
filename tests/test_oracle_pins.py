"""Pins of the CPU oracle against facts fixed outside the oracle itself:
the pages' printed mask example, closed forms, library routines (torch's
bf16 cast, scipy's softmax/expit, numpy's sort), brute force on tiny inputs,
and invariants of the decoding method.  Each pin is chosen so that a plausible
slip (dropped term, wrong sign or index, transposed operand, > for >=) fails.
"""
import copy
import inspect
import math
import os

import numpy as np
import pytest
import scipy.special as sps
import torch

import dvlm_gen as gen
import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


# ----------------------------------------------------------------------------
# bf16 rounding
# ----------------------------------------------------------------------------
def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000).astype(np.float32) * 3,
                        rng.standard_normal(1000).astype(np.float32) * 1e-30,
                        rng.standard_normal(1000).astype(np.float32) * 1e30])
    # exact halfway points between neighbouring bf16 values
    base = torch.from_numpy(rng.standard_normal(5000).astype(np.float32)).to(torch.bfloat16).float().numpy()
    bits = base.view(np.uint32) | np.uint32(0x8000)
    x = np.concatenate([x, bits.view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(O.bf16_round(x.astype(np.float64)), ref)


def test_bf16_round_ties_to_even():
    assert O.bf16_round(1.0 + 2.0 ** -8) == 1.0              # halfway, even is 1.0
    assert O.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert O.bf16_round(-(1.0 + 2.0 ** -8 + 2.0 ** -20)) == -(1.0 + 2.0 ** -7)
    assert O.bf16_round(0.0) == 0.0


# ----------------------------------------------------------------------------
# RMSNorm, RoPE, SiLU
# ----------------------------------------------------------------------------
def test_rmsnorm_closed_form():
    for c in (0.5, -3.0, 1e-3):
        x = np.full((2, 64), c)
        np.testing.assert_allclose(O.rmsnorm(x, 1e-6), c / math.sqrt(c * c + 1e-6), rtol=1e-14)
    x = np.random.default_rng(1).standard_normal((3, 128)) * 7
    y = O.rmsnorm(x, 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-12)
    np.testing.assert_array_equal(O.rmsnorm(np.zeros((1, 8))), 0.0)


def test_rope_complex_form_and_invariants():
    rng = np.random.default_rng(2)
    D, base = 16, 10000.0
    x = rng.standard_normal((5, 3, D))
    pos = np.array([0, 1, 7, 100, 1523])
    y = O.rope(x, pos, base)
    half = D // 2
    z = x[..., :half] + 1j * x[..., half:]
    for t, p in enumerate(pos):
        th = p * base ** (-2.0 * np.arange(half) / D)
        w = z[t] * np.exp(1j * th)[None, :]
        np.testing.assert_allclose(y[t, :, :half], w.real, atol=1e-12)
        np.testing.assert_allclose(y[t, :, half:], w.imag, atol=1e-12)
    np.testing.assert_allclose(y[0], x[0], atol=0)                     # position 0
    q, k = rng.standard_normal((1, 1, D)), rng.standard_normal((1, 1, D))
    d1 = np.sum(O.rope(q, [37], base) * O.rope(k, [12], base))
    d2 = np.sum(O.rope(q, [1037], base) * O.rope(k, [1012], base))
    assert abs(d1 - d2) < 1e-9                                          # relative position only


def test_silu_matches_library():
    a = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(O.silu(a), a * sps.expit(a), rtol=1e-13, atol=1e-300)


# ----------------------------------------------------------------------------
# Masks and attention
# ----------------------------------------------------------------------------
def _load_matrix(name):
    rows = []
    with open(os.path.join(HERE, "golden", name)) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(v) for v in line.split()])
    return np.array(rows)


def test_n2n_mask_reproduces_printed_example():
    want = _load_matrix("mask_n2n_block2.txt")
    blocks = [0, 0, 1, 1]
    m = O.mask_from_roles([True] * 4, blocks, [0, 1, 2, 3], [True] * 4, blocks, [0, 1, 2, 3])
    np.testing.assert_array_equal(m, want)


def test_n2c_and_c2c_rules():
    blocks = [0, 0, 1, 1]
    pos = [0, 1, 2, 3]
    n2c = O.mask_from_roles([True] * 4, blocks, pos, [False] * 4, blocks, pos)
    # noisy tokens see clean tokens of preceding blocks only, never the clean
    # copy of their own block (that would leak the answer)
    np.testing.assert_array_equal(n2c, [[0, 0, 0, 0], [0, 0, 0, 0], [1, 1, 0, 0], [1, 1, 0, 0]])
    c2c = O.mask_from_roles([False] * 4, blocks, pos, [False] * 4, blocks, pos)
    np.testing.assert_array_equal(c2c, np.tril(np.ones((4, 4), dtype=int)))
    c2n = O.mask_from_roles([False] * 4, blocks, pos, [True] * 4, blocks, pos)
    assert c2n.sum() == 0


def _roles_case(rng, L, n, n_clean, Hq=4, Hkv=2, D=8):
    """A cache of L clean tokens (blocks of 4) plus n rows at slots L..L+n-1."""
    q = rng.standard_normal((n, Hq, D))
    K = rng.standard_normal((Hkv, L + n, D))
    V = rng.standard_normal((Hkv, L + n, D))
    return q, K, V


@pytest.mark.parametrize("L,n,n_clean", [(12, 4, 0), (9, 5, 0), (8, 4, 4), (0, 3, 3), (7, 1, 1), (5, 6, 2)])
def test_block_attention_equals_dense_masked_bruteforce(L, n, n_clean):
    rng = np.random.default_rng(L * 31 + n * 7 + n_clean)
    q, K, V = _roles_case(rng, L, n, n_clean)
    scale = 1 / math.sqrt(q.shape[-1])
    got = O.block_attention(q, K, V, L, n_clean, scale)
    # dense formulation: keys = cache (clean, blocks < current) then step rows;
    # step rows 0..n_clean-1 are clean (causal), the rest one noisy block
    cur = 10 ** 6
    k_noisy = [False] * (L + n_clean) + [True] * (n - n_clean)
    k_block = [j // 4 for j in range(L)] + [cur - 1] * n_clean + [cur] * (n - n_clean)
    k_pos = list(range(L + n))
    q_noisy, q_block, q_pos = k_noisy[L:], k_block[L:], k_pos[L:]
    m = O.mask_from_roles(q_noisy, q_block, q_pos, k_noisy, k_block, k_pos)
    want = O.dense_masked_attention(q, K.transpose(1, 0, 2), V.transpose(1, 0, 2), m, scale)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(3)
    L, n, D = 10, 4, 8
    q = rng.standard_normal((n, 2, D))
    K = np.tile(rng.standard_normal((1, 1, D)), (1, L + n, 1))     # all keys equal
    V = rng.standard_normal((1, L + n, D))
    out = O.block_attention(q, K, V, L, 0, 0.3)
    np.testing.assert_allclose(out[2, 1], V[0].mean(axis=0), rtol=1e-12)
    out = O.block_attention(q, K, V, L, 2, 0.3)                       # clean row 1 sees L+2 slots
    np.testing.assert_allclose(out[1, 0], V[0, :L + 2].mean(axis=0), rtol=1e-12)
    K2 = rng.standard_normal((1, L + n, D)) * 0.01
    K2[0, 5] = q[3, 0] * 1e4                                           # one dominant key
    out = O.block_attention(q, K2, V, L, 0, 1.0)
    np.testing.assert_allclose(out[3, 0], V[0, 5], rtol=1e-9)
    # single causal row at the end of a cache == textbook softmax attention
    q1 = rng.standard_normal((1, 2, D))
    Kc, Vc = rng.standard_normal((1, 9, D)), rng.standard_normal((1, 9, D))
    out = O.block_attention(q1, Kc, Vc, 8, 1, 0.5)
    for h in range(2):
        p = sps.softmax(0.5 * Kc[0] @ q1[0, h])
        np.testing.assert_allclose(out[0, h], p @ Vc[0], rtol=1e-12)


# ----------------------------------------------------------------------------
# Confidence / argmax
# ----------------------------------------------------------------------------
def test_confidence_matches_full_softmax_and_sort():
    rng = np.random.default_rng(4)
    lg = rng.standard_normal((6, 3000)) * 20
    c = O.confidence_from_logits(lg)
    p = sps.softmax(lg, axis=-1)
    order = np.argsort(-lg, axis=-1, kind="stable")
    ps = np.sort(p, axis=-1)
    np.testing.assert_allclose(c.p1, ps[:, -1], rtol=1e-12)
    np.testing.assert_allclose(c.p2, ps[:, -2], rtol=1e-12)
    np.testing.assert_array_equal(c.top1, order[:, 0])
    np.testing.assert_array_equal(c.top2, order[:, 1])
    np.testing.assert_allclose(c.p2, p[np.arange(6), order[:, 1]], rtol=1e-12)


def test_confidence_closed_forms():
    # one-hot LM-head rows: logits are the hidden entries themselves
    H = 16
    W = np.eye(H)
    h = np.arange(H, dtype=float)[None, :] * 0.1
    c = O.lm_head_conf(h, W)
    assert c.top1[0] == H - 1
    want = 1.0 / np.sum(np.exp(h[0] - h[0].max()))
    assert abs(c.p1[0] - want) < 1e-15
    # two equal maxima: p1 <= 1/2 and the lower id wins
    lg = np.array([[1.0, 5.0, 0.0, 5.0, 2.0]])
    c = O.confidence_from_logits(lg)
    assert c.top1[0] == 1 and c.p1[0] <= 0.5 and abs(c.p1[0] - c.p2[0]) < 1e-15
    assert c.top2[0] == 3   # the other maximum is the runner-up
    # uniform logits: p1 = 1/V
    c = O.confidence_from_logits(np.zeros((1, 256)))
    assert abs(c.p1[0] - 1 / 256) < 1e-15 and c.top1[0] == 0


# ----------------------------------------------------------------------------
# Commit, certificate, accept (hand-worked cases)
# ----------------------------------------------------------------------------
def test_threshold_commit_hand_cases():
    assert O.threshold_commit([.95, .5, .91, .2], [1, 1, 1, 1], 0.9) == [0, 2]
    assert O.threshold_commit([.5, .6, .3], [1, 1, 1], 0.9) == [1]           # force one
    assert O.threshold_commit([.9, .1], [1, 1], 0.9) == [0]                  # >= threshold
    assert O.threshold_commit([.9, .95, .2], [1, 1, 1], 0.9) == [0, 1]
    assert O.threshold_commit([.6, .6, .2], [1, 1, 1], 0.9) == [0]           # tie -> lowest
    assert O.threshold_commit([.99, .6, .2], [0, 1, 1], 0.9) == [1]          # unmasked ignored
    assert O.threshold_commit([.99, .6], [0, 0], 0.9) == []                  # nothing masked
    assert O.threshold_commit([.2, .3, .1], [1, 1, 1], -1.0) == [0, 1, 2]    # draft: commit all


def test_certificate_hand_cases():
    ids, conf = [3, 7, 9, 1], [.2, .9, .5, .8]          # order: 1, 3, 2, 0
    assert O.certificate_scan(ids, conf, [3, 7, 4, 1]) == 2      # disagrees at position 2
    assert O.certificate_scan(ids, conf, ids) == 4               # all agree
    assert O.certificate_scan(ids, conf, [3, 0, 9, 1]) == 0      # first in order disagrees
    assert O.certificate_scan(ids, conf, [0, 7, 9, 1]) == 3      # lowest-confidence one last
    assert O.certificate_scan([1, 2, 3], [.5, .5, .5], [1, 9, 3]) == 1   # ties: lower index first
    assert O.certificate_scan([1, 2, 3], [.5, .5, .5], [1, 2, 9]) == 2
    assert O.certificate_scan(ids, conf, [3, 7, 4, 1], [1, 1, 0, 1]) == 3  # non-participant skipped


def test_prefix_accept_hand_cases():
    assert O.prefix_accept([5, 7, 1, 2], [5, 7, 9, 2]) == 2
    assert O.prefix_accept([5, 7, 9, 2], [5, 7, 9, 2]) == 4
    assert O.prefix_accept([4, 7, 9, 2], [5, 7, 9, 2]) == 0


# ----------------------------------------------------------------------------
# Decode-level invariants on tiny models
# ----------------------------------------------------------------------------
def _tiny(bf16=False, seed=0, layers=1, lm_scale=40.0):
    if bf16:
        gd = gen.ModelDims(n_layers=layers, hidden=64, n_q_heads=4, n_kv_heads=2, head_dim=16,
                           inter=96, vocab=512, lm_scale=lm_scale, dtype="bf16")
    else:
        gd = gen.TINY
    d = O.dims_from(gd)
    w = O.weights_from_generator(gen, gd, seed)
    vis_t, vis, ids = gen.decode_context(gd, seed, 32, 16, 16)
    return gd, d, w, vis.astype(np.float64), ids


def _fresh(d, w, bf16, vis, ids):
    m = O.OracleModel(d, weights=w, bf16=bf16, Lmax=512)
    seed_tok = O.prefill(m, vis, ids)
    return m, seed_tok


@pytest.mark.parametrize("bf16", [False, True])
def test_spec_linear_equals_greedy_ar(bf16):
    gd, d, w, vis, ids = _tiny(bf16)
    m1, s1 = _fresh(d, w, bf16, vis, ids)
    ar = O.decode_ar(m1, s1, 40)
    m2, s2 = _fresh(d, w, bf16, vis, ids)
    sp = O.decode_spec_linear(m2, s2, 8, 40)
    assert sp.tokens == ar.tokens
    assert all(1 <= k <= 8 for k in sp.accept_lens)
    assert m2.L == m1.L + (sum(sp.accept_lens) - 40)  # spec may run past max_new


@pytest.mark.parametrize("bf16", [False, True])
def test_threshold_block1_equals_ar(bf16):
    gd, d, w, vis, ids = _tiny(bf16)
    m1, s1 = _fresh(d, w, bf16, vis, ids)
    ar = O.decode_ar(m1, s1, 12)
    m2, s2 = _fresh(d, w, bf16, vis, ids)
    th = O.decode_threshold(m2, s2, 1, 0.9, 12)
    assert th.tokens == ar.tokens and th.nfe == ar.nfe


def test_threshold_extreme_thresholds():
    gd, d, w, vis, ids = _tiny()
    B = 4
    m, s = _fresh(d, w, False, vis, ids)
    tr = O.decode_threshold(m, s, B, 1.5, 2 * B)       # nothing passes: one commit per iteration
    assert tr.commits_per_iter == [1] * (2 * (B - 1))
    assert tr.nfe == 2 * (B - 1) + 2
    m, s = _fresh(d, w, False, vis, ids)
    tr = O.decode_threshold(m, s, B, 0.0, 2 * B)       # everything passes: one iteration
    assert tr.commits_per_iter == [B - 1, B - 1] and tr.nfe == 4


def test_threshold_observers_do_not_change_the_trajectory():
    """The per-iteration observers used by the teacher-forced GPU checks see
    every iteration (with the scores the commit is decided on) and every block,
    and leave tokens, forwards and commits unchanged."""
    gd, d, w, vis, ids = _tiny()
    B = 4
    m, s = _fresh(d, w, True, vis, ids)
    plain = O.decode_threshold(m, s, B, 0.9, 2 * B)
    seen, blocks = [], []

    def on_iter(L, toks, masked, p1, top, p2):
        seen.append((L, list(toks), list(masked)))
        assert len(p1) == len(top) == len(p2) == B and all(p1 >= p2)

    m, s = _fresh(d, w, True, vis, ids)
    obs = O.decode_threshold(m, s, B, 0.9, 2 * B, on_iter=on_iter, on_block=lambda L, toks: blocks.append((L, toks)))
    assert obs.tokens == plain.tokens and obs.nfe == plain.nfe and obs.commits_per_iter == plain.commits_per_iter
    assert len(seen) == sum(1 for _ in plain.commits_per_iter) and len(blocks) == 2
    assert [b[1] for b in blocks] == [plain.tokens[:B], plain.tokens[B:2 * B]]
    assert blocks[1][0] == blocks[0][0] + B


def test_spec_observer_does_not_change_the_trajectory():
    """The per-round observer of the teacher-forced speculative GPU check sees
    every round: the draft pass's input, both passes' row scores, the draft,
    the accepted length and the next seed, consistent with one another."""
    gd, d, w, vis, ids = _tiny()
    B = 4
    m, s = _fresh(d, w, False, vis, ids)
    plain = O.decode_spec_linear(m, s, B, 12)
    rounds = []

    def on_round(L, toks, c, draft, g, k, nxt):
        assert toks == [draft[0]] + [d.mask_id] * (B - 1)
        assert draft[1:] == [int(t) for t in c.top1[:B - 1]]
        verify = [draft[0]] + [int(t) for t in g.top1[:B - 1]]
        assert k == O.prefix_accept(verify, draft) and nxt == int(g.top1[k - 1])
        rounds.append((L, k))

    m, s = _fresh(d, w, False, vis, ids)
    obs = O.decode_spec_linear(m, s, B, 12, on_round=on_round)
    assert obs.tokens == plain.tokens and obs.accept_lens == plain.accept_lens and obs.nfe == plain.nfe
    assert [k for _, k in rounds] == plain.accept_lens
    assert all(rounds[i + 1][0] == rounds[i][0] + rounds[i][1] for i in range(len(rounds) - 1))


def test_block_first_token_is_ar_token_and_append_kv_equals_prefill():
    gd, d, w, vis, ids = _tiny()
    B = 4
    m, s = _fresh(d, w, False, vis, ids)
    m_ar, s_ar = _fresh(d, w, False, vis, ids)
    tr = O.decode_threshold(m, s, B, 0.9, B)
    ar = O.decode_ar(m_ar, s_ar, 1)
    assert tr.tokens[0] == ar.tokens[0]
    # KV of the causal append pass == KV of a prefill over the same prefix
    m2 = O.OracleModel(d, weights=w, bf16=False, Lmax=512)
    O.prefill(m2, vis, list(ids) + tr.tokens)
    L = m.L
    assert L == len(vis) + len(ids) + B == m2.L
    np.testing.assert_allclose(m.K[0][:, :L], m2.K[0][:, :L], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(m.V[0][:, :L], m2.V[0][:, :L], rtol=1e-12, atol=1e-12)


def test_tiny_threshold_run_completes_block():
    """First configuration: 64-token context, one B=4 block, threshold 0.9."""
    gd, d, w, vis, ids = _tiny()
    m, s = _fresh(d, w, False, vis, ids)
    tr = O.decode_threshold(m, s, 4, 0.9, 4)
    assert len(tr.tokens) == 4 and sum(tr.commits_per_iter) == 3
    assert all(0 <= t < d.vocab for t in tr.tokens)
    # the tiny LM head (x40) spreads top-1 probabilities widely
    c = O.lm_head_conf(np.random.default_rng(0).standard_normal((64, 32)), w["lm_head"])
    assert c.p1.min() < 0.6 and c.p1.max() > 0.95


# ----------------------------------------------------------------------------
# Planted mistakes: each mutant of an oracle function must fail its pin
# ----------------------------------------------------------------------------
def _check_rope(fn):
    x = np.random.default_rng(9).standard_normal((2, 1, 8))
    y = fn(x, [3, 11], 10000.0)
    z = x[..., :4] + 1j * x[..., 4:]
    for t, p in enumerate([3, 11]):
        w = z[t] * np.exp(1j * p * 10000.0 ** (-2.0 * np.arange(4) / 8))[None, :]
        np.testing.assert_allclose(y[t, :, :4], w.real, atol=1e-12)
        np.testing.assert_allclose(y[t, :, 4:], w.imag, atol=1e-12)


def _check_commit(fn):
    assert fn([.95, .5, .91, .2], [1, 1, 1, 1], 0.9) == [0, 2]
    assert fn([.5, .6, .3], [1, 1, 1], 0.9) == [1]
    assert fn([.9, .1], [1, 1], 0.9) == [0]
    assert fn([.9, .95, .2], [1, 1, 1], 0.9) == [0, 1]
    assert fn([.6, .6, .2], [1, 1, 1], 0.9) == [0]


def _check_cert(fn):
    ids, conf = [3, 7, 9, 1], [.2, .9, .5, .8]
    assert fn(ids, conf, [3, 7, 4, 1]) == 2
    assert fn([1, 2, 3], [.5, .5, .5], [1, 9, 3]) == 1
    assert fn([1, 2, 3], [.5, .5, .5], [1, 2, 9]) == 2


def _check_n2c(fn):
    b, p = [0, 0, 1, 1], [0, 1, 2, 3]
    np.testing.assert_array_equal(fn([True] * 4, b, p, [False] * 4, b, p),
                                  [[0, 0, 0, 0], [0, 0, 0, 0], [1, 1, 0, 0], [1, 1, 0, 0]])


def _check_attention(fn):
    rng = np.random.default_rng(5)
    q, K, V = rng.standard_normal((3, 2, 4)), rng.standard_normal((1, 8, 4)), rng.standard_normal((1, 8, 4))
    got = fn(q, K, V, 5, 1, 0.5)
    for t, vis in enumerate([6, 8, 8]):
        for h in range(2):
            np.testing.assert_allclose(got[t, h], sps.softmax(0.5 * K[0, :vis] @ q[t, h]) @ V[0, :vis], rtol=1e-12)


def _check_argmax(fn):
    assert fn(np.array([[1.0, 5.0, 0.0, 5.0, 2.0]])).top1[0] == 1


# ----------------------------------------------------------------------------
# FP8 W8A8 linear layer (next step of the weight stream)
# ----------------------------------------------------------------------------
def _e4m3_grid():
    """Every finite non-negative E4M3 value, from torch's own decoding."""
    codes = torch.arange(0, 128, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    return np.unique(codes[np.isfinite(codes)])


def test_e4m3_round_matches_torch_cast_and_ties():
    g = _e4m3_grid()
    assert g.max() == O.E4M3_MAX and g[1] == 2.0 ** -9 and len(g) == 127
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.standard_normal(20000) * 2.0 ** -7,
                        g, -g, (g[1:] + g[:-1]) / 2, -(g[1:] + g[:-1]) / 2,   # every exact midpoint
                        rng.uniform(448, 463.9, 100)])                       # rounds down to 448
    x = x.astype(np.float32).astype(np.float64)                             # exact inputs for torch's cast
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(O.e4m3_round(x), ref)
    # beyond the finite range the definition saturates (torch's cast gives NaN)
    np.testing.assert_array_equal(O.e4m3_round(np.array([500.0, -1e6])), [448.0, -448.0])


def test_fp8_row_scales_and_power_of_two_invariance():
    rng = np.random.default_rng(4)
    A = rng.standard_normal((6, 96))
    A[2] = 0.0
    q, s = O.fp8_quantize_rows(A)
    for r in range(6):
        if r == 2:
            assert s[r] == 1.0 and not q[r].any()
            continue
        k = np.argmax(np.abs(A[r]))
        assert abs(q[r, k]) == O.E4M3_MAX                      # the row's largest entry maps to +-448
        assert np.all(np.isin(np.abs(q[r]), _e4m3_grid()))      # codes are E4M3 values
    q2, s2 = O.fp8_quantize_rows(A * np.array([1, 2.0 ** 5, 1, 2.0 ** -7, 1, 1])[:, None])
    np.testing.assert_array_equal(q2, q)                        # scaling a row by 2^k moves only its scale
    np.testing.assert_allclose(s2 / s, [1, 2.0 ** 5, 1, 2.0 ** -7, 1, 1], rtol=0, atol=0)


def test_fp8_linear_exact_when_operands_are_representable():
    """Rows made of E4M3 values times 2^j that contain +-448 * 2^j have scale
    2^j and quantise without error: the W8A8 product is then the exact product."""
    rng = np.random.default_rng(5)
    g = _e4m3_grid()
    vals = np.concatenate([g, -g])

    def rows(n, k, jlo, jhi):
        j = rng.integers(jlo, jhi, (n, 1))
        A = rng.choice(vals, (n, k))
        A[:, 0] = O.E4M3_MAX * rng.choice([-1.0, 1.0], n)
        return A * 2.0 ** j

    x, W = rows(8, 64, -3, 4), rows(16, 64, -6, 2)
    assert np.array_equal(O.fp8_quantize_rows(x)[0] * O.fp8_quantize_rows(x)[1][:, None], x)
    np.testing.assert_array_equal(O.fp8_linear(x, W), x @ W.T)


def test_fp8_linear_error_bound():
    """|y_fp8 - x W^T| stays within the bound an E4M3 code error implies:
    per element at most 2^-4 relative (normal codes) or 2^-10 of the row
    scale (subnormal codes), so a dropped scale, a wrong axis or truncation
    would break it by orders of magnitude or on average."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal((16, 2048))
    W = rng.standard_normal((256, 2048)) * 0.02
    y = O.fp8_linear(x, W)
    exact = x @ W.T
    xq, a = O.fp8_quantize_rows(x)
    wq, s = O.fp8_quantize_rows(W)
    dx = np.maximum(np.abs(x) * 2.0 ** -4, a[:, None] * 2.0 ** -10)
    dw = np.maximum(np.abs(W) * 2.0 ** -4, s[:, None] * 2.0 ** -10)
    bound = dx @ np.abs(W).T + np.abs(x) @ dw.T + dx @ dw.T
    assert np.all(np.abs(y - exact) <= bound)
    # round to nearest is unbiased: no systematic shrink or growth of |y|
    # (rounding toward zero would shrink it by about 3%)
    bias = np.mean(np.sign(exact) * (y - exact)) / np.mean(np.abs(exact))
    assert abs(bias) < 0.005


def test_smooth_factors_balance_channels_and_keep_the_product():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((32, 64)) * rng.uniform(0.1, 20, 64)
    W = rng.standard_normal((48, 64)) * rng.uniform(0.001, 0.1, 64)
    xa, wa = np.max(np.abs(x), axis=0), np.max(np.abs(W), axis=0)
    m = O.smooth_factors(xa, wa, 0.5)
    np.testing.assert_allclose(xa / m, wa * m, rtol=1e-12)       # alpha 0.5: equal channel ranges
    np.testing.assert_allclose((x / m) @ (W * m).T, x @ W.T, rtol=1e-12, atol=1e-12)
    m1 = O.smooth_factors(xa, wa, 1.0)
    np.testing.assert_allclose(np.max(np.abs(x / m1), axis=0), 1.0, rtol=1e-12)   # alpha 1: all range to W


def test_fp8_model_differs_from_the_bf16_model_only_in_its_projections(monkeypatch):
    """With the W8A8 product replaced by the exact one, the fp8 model's
    forward equals the bf16 model's bit for bit (norms, RoPE, attention and
    storage points untouched); every layer routes exactly its seven matrices
    through the W8A8 product, each on the activation that feeds it."""
    import oracle.dvlm_oracle as OM
    gd, d, w, vis, ids = _tiny(True, layers=2)
    x0 = np.asarray(vis[:6], dtype=np.float64)
    ref = O.OracleModel(d, weights=w, bf16=True, Lmax=64).forward(x0, 0, n_clean=6)
    seen = []

    def exact(a, W):
        seen.append((a.shape[1], W.shape))
        return a @ W.T

    monkeypatch.setattr(OM, "fp8_linear", exact)
    got = O.OracleModel(d, weights=w, bf16=True, Lmax=64, fp8=True).forward(x0, 0, n_clean=6)
    assert np.array_equal(got, ref)
    H, D, Hq, Hkv, I = d.hidden, d.head_dim, d.n_q_heads, d.n_kv_heads, d.inter
    per_layer = [(H, (Hq * D, H)), (H, (Hkv * D, H)), (H, (Hkv * D, H)), (Hq * D, (H, Hq * D)),
                 (H, (I, H)), (H, (I, H)), (I, (H, I))]
    assert seen == per_layer * d.n_layers


def test_fp8_model_keeps_the_decode_invariants():
    """The fp8 model is a deterministic decoder of its own: speculative
    decoding still reproduces its greedy AR output, and its forward stays
    within the W8A8 error of the exact model."""
    gd, d, w, vis, ids = _tiny(True, layers=2)
    m1 = O.OracleModel(d, weights=w, bf16=True, Lmax=256, fp8=True)
    s1 = O.prefill(m1, vis, ids)
    ar = O.decode_ar(m1, s1, 16)
    m2 = O.OracleModel(d, weights=w, bf16=True, Lmax=256, fp8=True)
    s2 = O.prefill(m2, vis, ids)
    assert O.decode_spec_linear(m2, s2, 4, 16).tokens == ar.tokens
    x0 = np.asarray(vis[:6], dtype=np.float64)
    exact = O.OracleModel(d, weights=w, bf16=False, Lmax=64).forward(x0, 0, n_clean=6)
    q8 = O.OracleModel(d, weights=w, bf16=False, Lmax=64, fp8=True).forward(x0, 0, n_clean=6)
    # each E4M3 operand carries a relative rounding error of at most 2^-4,
    # uniform-like, so a product is off by about sqrt(2) * 2^-4 / sqrt(3) ~ 5%
    # RMS; measured 4.4% of the layers' update here
    rel = np.linalg.norm(q8 - exact) / np.linalg.norm(exact - x0)
    assert 0.01 < rel < 0.1, rel


def test_fp8_model_smoothing_with_unit_factors_is_plain_w8a8():
    gd, d, w, vis, ids = _tiny(True, layers=1)
    x0 = np.asarray(vis[:5], dtype=np.float64)
    plain = O.OracleModel(d, weights=w, bf16=True, Lmax=64, fp8=True).forward(x0, 0, n_clean=5)
    ones = {f"0.{n}": np.ones(w[f"0.{n}"].shape[1]) for n in ("wq", "wk", "wv", "wo", "wg", "wu", "wd")}
    sm = O.OracleModel(d, weights=w, bf16=True, Lmax=64, fp8=True, smooth=ones).forward(x0, 0, n_clean=5)
    assert np.array_equal(plain, sm)
    twos = {k: np.full_like(v, 2.0) for k, v in ones.items()}      # a power of two cancels exactly
    sm2 = O.OracleModel(d, weights=w, bf16=True, Lmax=64, fp8=True, smooth=twos).forward(x0, 0, n_clean=5)
    assert np.array_equal(plain, sm2)


def test_fp8_planted_mistakes_are_caught(monkeypatch):
    """Each plausible slip in the FP8 definitions fails at least one FP8 pin."""
    import oracle.dvlm_oracle as OM
    real_round, real_rows, real_linear = OM.e4m3_round, OM.fp8_quantize_rows, OM.fp8_linear

    def round_toward_zero(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.minimum(np.abs(x), OM.E4M3_MAX)
        _, e = np.frexp(a)
        q = np.ldexp(1.0, np.maximum(e, -5) - 4)
        return np.sign(x) * np.trunc(a / q) * q

    def subnormal_floor_too_low(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.minimum(np.abs(x), OM.E4M3_MAX)
        _, e = np.frexp(a)
        q = np.ldexp(1.0, np.maximum(e, -6) - 4)
        return np.sign(x) * np.minimum(np.round(a / q) * q, OM.E4M3_MAX)

    def scales_per_column(A):
        q, s = real_rows(np.asarray(A).T)
        return q.T, s

    def no_activation_scale(x, W):
        xq, _ = real_rows(x)
        wq, s = real_rows(W)
        return (xq @ wq.T) * s[None, :]

    pins = [test_e4m3_round_matches_torch_cast_and_ties, test_fp8_row_scales_and_power_of_two_invariance,
            test_fp8_linear_exact_when_operands_are_representable, test_fp8_linear_error_bound]
    for name, mutant in [("e4m3_round", round_toward_zero), ("e4m3_round", subnormal_floor_too_low),
                         ("fp8_quantize_rows", scales_per_column), ("fp8_linear", no_activation_scale)]:
        with monkeypatch.context() as mp:
            mp.setattr(OM, name, mutant)
            mp.setattr(O, name, mutant)
            failed = 0
            for pin in pins:
                try:
                    pin()
                except (AssertionError, ValueError, IndexError):   # wrong values or wrong scale shapes
                    failed += 1
            assert failed > 0, name
    assert OM.e4m3_round is real_round and OM.fp8_linear is real_linear


# ----------------------------------------------------------------------------
# Certificate-guided visual routing (LOWN) inside block decoding
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("L,n,n_vis", [(12, 4, 5), (9, 5, 9), (8, 4, 1)])
def test_text_only_attention_equals_dense_without_vision_keys(L, n, n_vis):
    """TEXT-ONLY pass: the dense role mask with the vision keys (the first
    n_vis cache slots) removed, brute force, positions unchanged."""
    rng = np.random.default_rng(L * 13 + n_vis)
    q, K, V = _roles_case(rng, L, n, 0)
    scale = 1 / math.sqrt(q.shape[-1])
    got = O.block_attention(q, K, V, L, 0, scale, hide=n_vis)
    k_noisy = [False] * L + [True] * n
    k_block = [j // 4 for j in range(L)] + [10 ** 6] * n
    k_pos = list(range(L + n))
    m = O.mask_from_roles(k_noisy[L:], k_block[L:], k_pos[L:], k_noisy, k_block, k_pos)
    m[:, :n_vis] = 0
    want = O.dense_masked_attention(q, K.transpose(1, 0, 2), V.transpose(1, 0, 2), m, scale)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    assert not np.allclose(got, O.block_attention(q, K, V, L, 0, scale))


def test_routing_orders_hand_cases():
    conf = [0.3, 0.9, 0.5, 0.9, 0.7]
    part = [False, True, True, True, True]
    assert O.certificate_order(conf, part) == [1, 3, 4, 2]                 # ties: lower position first
    full_top, text_top = [0, 5, 6, 7, 8], [0, 5, 9, 7, 1]
    assert O.divergence_first_order(full_top, conf, text_top, part) == [4, 2, 1, 3]


class _ScriptedModel:
    """Stands in for the decoder: hands out scripted confidences per kind of
    pass (FULL / TEXT-ONLY noisy, causal append) and records the passes."""

    def __init__(self, B, full, text):
        self.d = O.Dims(n_layers=1, hidden=4, n_q_heads=1, n_kv_heads=1, head_dim=2, inter=4, vocab=100)
        self.L, self.B = 40, B
        self.last_conf = O.Conf(p1=np.array([1.0]), top1=np.array([7]), p2=np.array([0.0]))
        self.full, self.text, self.calls = list(full), list(text), []

    def embed(self, toks):
        return np.asarray(toks, dtype=np.float64)[:, None]

    def forward(self, x, L, n_clean, hide=0):
        kind = "causal" if n_clean else ("text" if hide else "full")
        self.calls.append((kind, L, hide, [int(t) for t in x[:, 0]]))
        return kind

    def logits_conf(self, kind):
        if kind == "causal":
            return O.Conf(p1=np.ones(self.B), top1=np.arange(self.B) + 60, p2=np.zeros(self.B))
        script = self.full if kind == "full" else self.text
        assert script, f"one {kind} pass more than scripted"
        p1, top = script.pop(0)
        # row r scores position r + 1
        return O.Conf(p1=np.array(p1[1:] + [0.0]), top1=np.array(top[1:] + [0]), p2=np.zeros(self.B))


def test_lown_routing_on_a_scripted_model():
    B, mk = 5, 99                                   # mask id of the stub's vocabulary
    full1 = ([0, 0.9, 0.5, 0.8, 0.6], [0, 11, 12, 13, 14])
    # 1) TEXT-ONLY disagrees at the first scanned position: FULL refresh, divergent first
    m = _ScriptedModel(B, [full1, ([0, 0, 0.7, 0, 0.95], [0, 0, 22, 0, 44])], [([0] * 5, [0, 0, 12, 0, 98])])
    tr = O.decode_lown(m, 7, B, 2, n_vis=32, max_new=5)
    assert tr.tokens == [7, 11, 22, 13, 44]
    assert (tr.n_full, tr.n_text, tr.n_causal) == (2, 1, 1) and tr.accepted == [2, 2]
    assert tr.text_branch == [False, False]
    assert [c[0] for c in m.calls] == ["full", "text", "full", "causal"]
    assert m.calls[1][2] == 32 and m.calls[1][3] == [7, 11, mk, 13, mk]     # vision hidden, state after step 1
    # 2) TEXT-ONLY agrees along the scan: the prefix is accepted with the anchor ids
    m = _ScriptedModel(B, [full1], [([0] * 5, [0, 0, 12, 0, 14])])
    tr = O.decode_lown(m, 7, B, 2, n_vis=32, max_new=5)
    assert tr.tokens == [7, 11, 12, 13, 14] and (tr.n_full, tr.n_text) == (1, 1)
    assert tr.text_branch == [False, True]
    # 3) a certified prefix longer than k is accepted whole
    m = _ScriptedModel(6, [([0, 0.9, 0.5, 0.8, 0.6, 0.4], [0, 11, 12, 13, 14, 15])],
                       [([0] * 6, [0, 0, 12, 0, 14, 15])])
    tr = O.decode_lown(m, 7, 6, 2, n_vis=32, max_new=6)
    assert tr.accepted == [2, 3] and tr.tokens == [7, 11, 12, 13, 14, 15]
    # 4) the FULL branch unmasks the divergent positions (2, 4) before the more
    # confident agreeing one (5), which the next TEXT-ONLY step certifies
    # against the refreshed anchor
    m = _ScriptedModel(6, [([0, 0.9, 0.5, 0.8, 0.6, 0.4], [0, 11, 12, 13, 14, 15]),
                           ([0, 0, 0.3, 0, 0.2, 0.35], [0, 0, 32, 0, 34, 35])],
                       [([0] * 6, [0, 0, 12, 0, 97, 35]), ([0] * 6, [0, 0, 0, 0, 0, 35])])
    tr = O.decode_lown(m, 7, 6, 2, n_vis=32, max_new=6)
    assert tr.text_branch == [False, False, True] and tr.accepted == [2, 2, 1]
    assert tr.tokens == [7, 11, 32, 13, 34, 35]
    # 5) the certificate stops at the first disagreement (position 4, scanned
    # first) although positions 2 and 5 further down agree, which would reach k
    m = _ScriptedModel(6, [([0, 0.9, 0.5, 0.8, 0.6, 0.4], [0, 11, 12, 13, 14, 15]),
                           ([0, 0, 0.3, 0, 0.2, 0.35], [0, 0, 32, 0, 34, 35])],
                       [([0] * 6, [0, 0, 12, 0, 97, 15]), ([0] * 6, [0, 0, 0, 0, 34, 0])])
    tr = O.decode_lown(m, 7, 6, 2, n_vis=32, max_new=6)
    assert tr.text_branch == [False, False, True] and tr.accepted == [2, 2, 1]
    assert tr.tokens == [7, 11, 32, 13, 34, 35]


def test_lown_observers_do_not_change_the_trajectory():
    """The per-pass observers of the teacher-forced GPU routing check see
    every FULL and TEXT-ONLY pass (tokens before the pass's unmasking) and
    every block, and leave the trajectory unchanged."""
    gd, d, w, vis, ids = _tiny()
    B = 4
    m, s0 = _fresh(d, w, False, vis, ids)
    plain = O.decode_lown(m, s0, B, 1, n_vis=len(vis), max_new=3 * B)
    passes, blocks = [], []
    m, s0 = _fresh(d, w, False, vis, ids)
    obs = O.decode_lown(m, s0, B, 1, n_vis=len(vis), max_new=3 * B,
                        on_pass=lambda kind, L, toks, p1, top: passes.append((kind, L, toks)),
                        on_block=lambda L, toks: blocks.append((L, toks)))
    assert obs.tokens == plain.tokens and obs.accepted == plain.accepted and obs.text_branch == plain.text_branch
    assert [p[0] for p in passes].count("full") == plain.n_full and [p[0] for p in passes].count("text") == plain.n_text
    assert [b[1] for b in blocks] == [plain.tokens[i * B:(i + 1) * B] for i in range(3)]
    assert all(p[2][0] == blocks[[b[0] for b in blocks].index(p[1])][1][0] for p in passes)   # seed row fixed


def test_lown_planted_mistakes_are_caught(monkeypatch):
    import oracle.dvlm_oracle as OM
    real_div = OM.divergence_first_order

    def agreeing_first(full_top, full_conf, text_top, part):
        idx = real_div(full_top, full_conf, text_top, part)
        return [i for i in idx if text_top[i] == full_top[i]] + [i for i in idx if text_top[i] != full_top[i]]

    def count_all_agreeing(anchor_id, anchor_conf, top1, part=None):
        return sum(1 for i in range(len(anchor_id)) if (part is None or part[i]) and top1[i] == anchor_id[i])

    for name, mutant in [("divergence_first_order", agreeing_first), ("certificate_scan", count_all_agreeing)]:
        with monkeypatch.context() as mp:
            mp.setattr(OM, name, mutant)
            with pytest.raises(AssertionError):
                test_lown_routing_on_a_scripted_model()

    # the FULL pass hides the vision rows as well (the routing then never sees them)
    src = inspect.getsource(OM.decode_lown)
    full_call = "model.forward(model.embed(toks), L, n_clean=0)\n"
    assert src.count(full_call) == 1
    ns = dict(vars(OM))
    exec(src.replace(full_call, "model.forward(model.embed(toks), L, n_clean=0, hide=n_vis)\n"), ns)
    with monkeypatch.context() as mp:
        mp.setattr(O, "decode_lown", ns["decode_lown"])
        for check in (test_lown_routing_on_a_scripted_model, test_lown_on_the_tiny_model):
            with pytest.raises(AssertionError):
                check()


def test_lown_on_the_tiny_model():
    """Invariants on a real (tiny) decoder: every step unmasks at least
    min(k, masked) positions; with k covering the block, one FULL step per
    block reproduces threshold decoding with tau 0 (everything commits at
    once)."""
    gd, d, w, vis, ids = _tiny()
    B = 4
    m, s0 = _fresh(d, w, False, vis, ids)
    tr = O.decode_lown(m, s0, B, B - 1, n_vis=len(vis), max_new=3 * B)
    m2, s2 = _fresh(d, w, False, vis, ids)
    th = O.decode_threshold(m2, s2, B, 0.0, 3 * B)
    assert tr.tokens == th.tokens and tr.n_full == 3 and tr.n_text == 0
    for k in (1, 2):
        m, s0 = _fresh(d, w, False, vis, ids)
        tr = O.decode_lown(m, s0, B, k, n_vis=len(vis), max_new=3 * B)
        assert len(tr.tokens) == 3 * B and tr.n_causal == 3 and tr.n_full >= 3
        assert all(a >= 1 for a in tr.accepted) and sum(tr.accepted) == 3 * (B - 1)
        steps_per_block = len(tr.accepted) / 3
        assert steps_per_block <= math.ceil((B - 1) / k)


def test_topk_commit_hand_cases():
    p = [0.95, 0.5, 0.91, 0.2, 0.91]
    assert O.topk_commit(p, [True] * 5, 2) == [0, 2]           # tie at 0.91: lower position
    assert O.topk_commit(p, [True] * 5, 3) == [0, 2, 4]
    assert O.topk_commit(p, [False, True, True, True, True], 1) == [2]
    assert O.topk_commit(p, [False, True, False, True, False], 5) == [1, 3]
    assert O.topk_commit(p, [False] * 5, 2) == []
    assert O.topk_commit(p, [True] * 5, 0) == []
    # k = 1 is the threshold rule's force-commit when nothing passes
    rng = np.random.default_rng(5)
    for _ in range(50):
        q = rng.choice([0.1, 0.3, 0.5, 0.7], 6)
        m = list(rng.random(6) < 0.7)
        assert O.topk_commit(q, m, 1) == O.threshold_commit(q, m, 2.0)
        assert O.topk_commit(q, m, 6) == O.threshold_commit(q, m, 0.0)


def test_topk_planted_mistakes_are_caught(monkeypatch):
    import oracle.dvlm_oracle as OM
    real = OM.topk_commit

    def later_on_ties(p1, masked, k):
        idx = [r for r in range(len(p1)) if masked[r]]
        idx.sort(key=lambda r: (-float(p1[r]), -r))
        return sorted(idx[:k])

    def counts_committed_rows(p1, masked, k):       # k taken over all rows, not the masked ones
        idx = sorted(range(len(p1)), key=lambda r: (-float(p1[r]), r))[:k]
        return sorted(r for r in idx if masked[r])

    for mutant in (later_on_ties, counts_committed_rows, lambda p1, masked, k: real(p1, masked, k + 1)):
        with monkeypatch.context() as mp:
            mp.setattr(OM, "topk_commit", mutant)
            mp.setattr(O, "topk_commit", mutant)
            with pytest.raises(AssertionError):
                test_topk_commit_hand_cases()


@pytest.mark.parametrize("bf16", [False, True])
def test_topk_decoding_limits(bf16):
    """k = 1 equals threshold decoding with nothing passing (tau > 1); k
    covering the block equals tau = 0; in between, ceil((B-1)/k) iterations
    per block, k commits each but the last."""
    gd, d, w, vis, ids = _tiny(bf16)
    B = 5
    runs = {}
    for name, kw in [("k1", dict(tau=0.9, commit_k=1)), ("t2", dict(tau=2.0)),
                     ("kB", dict(tau=0.9, commit_k=B)), ("t0", dict(tau=0.0)), ("k3", dict(tau=0.9, commit_k=3))]:
        m, s0 = _fresh(d, w, bf16, vis, ids)
        runs[name] = O.decode_threshold(m, s0, B, kw.pop("tau"), 3 * B, **kw)
    assert runs["k1"].tokens == runs["t2"].tokens and runs["k1"].commits_per_iter == [1] * (3 * (B - 1))
    assert runs["kB"].tokens == runs["t0"].tokens and runs["kB"].commits_per_iter == [B - 1] * 3
    assert runs["k3"].commits_per_iter == [3, 1] * 3
    assert runs["k3"].nfe == 3 * (math.ceil((B - 1) / 3) + 1)


def test_paged_gather_hand_case():
    pages = np.zeros((4, 1, 2, 1))
    for pg in range(4):
        for r in range(2):
            pages[pg, 0, r, 0] = 10 * pg + r
    # table [3, 0, 2]: slots 0,1 -> page 3; 2,3 -> page 0; 4 -> page 2 row 0
    got = O.paged_gather(pages, [3, 0, 2], 5)[0, :, 0]
    assert list(got) == [30, 31, 0, 1, 20]


def test_paged_planted_mistakes_are_caught(monkeypatch):
    import oracle.dvlm_oracle as OM
    src = inspect.getsource(OM.paged_gather)
    old = "pages[block_table[s // P], :, s % P]"
    assert src.count(old) == 1
    for new in ("pages[block_table[s % P], :, s // P]",          # page and row swapped
                "pages[s // P, :, s % P]",                         # table ignored
                "pages[block_table[s // P], :, (s + 1) % P]"):     # row off by one
        ns = dict(vars(OM))
        exec(src.replace(old, new), ns)
        with monkeypatch.context() as mp:
            mp.setattr(O, "paged_gather", ns["paged_gather"])
            with pytest.raises((AssertionError, IndexError)):
                test_paged_gather_hand_case()


@pytest.mark.parametrize("P,L,n,n_clean", [(1, 7, 3, 0), (3, 10, 4, 2), (16, 37, 5, 5), (16, 64, 16, 0)])
def test_paged_attention_equals_contiguous_cache(P, L, n, n_clean):
    """Scatter a contiguous cache into randomly permuted pages (ragged last
    page), gather it back, and attend: both equal the contiguous results."""
    rng = np.random.default_rng(100 * P + L)
    Hq, Hkv, D = 4, 2, 8
    K, V = rng.standard_normal((2, Hkv, L + n, D))
    q = rng.standard_normal((n, Hq, D))
    n_pages = -(-(L + n) // P)
    table = [int(t) for t in rng.permutation(n_pages + 3)[:n_pages]]      # spare pages stay unused
    Kp = rng.standard_normal((n_pages + 3, Hkv, P, D))                     # garbage outside the table
    Vp = rng.standard_normal((n_pages + 3, Hkv, P, D))
    for s in range(L + n):
        Kp[table[s // P], :, s % P] = K[:, s]
        Vp[table[s // P], :, s % P] = V[:, s]
    np.testing.assert_array_equal(O.paged_gather(Kp, table, L + n), K)
    want = O.block_attention(q, K, V, L, n_clean, 0.3)
    np.testing.assert_array_equal(O.paged_block_attention(q, Kp, Vp, table, L, n_clean, 0.3), want)
    hide = min(3, L)
    np.testing.assert_array_equal(O.paged_block_attention(q, Kp, Vp, table, L, n_clean, 0.3, hide),
                                  O.block_attention(q, K, V, L, n_clean, 0.3, hide))


# ----------------------------------------------------------------------------
# Quadratic self-speculative decoding [FDV §2.3.1]
# ----------------------------------------------------------------------------
def _quad_mask(L, B):
    """The fused forward's visibility from token roles alone: cache slots are
    clean tokens of an earlier block; verify row t is the clean token of a
    block of its own (t) at position L+t; candidate block i holds the noisy
    tokens of block i+1 at positions L+i+1 ... (so it sees verify rows 0..i)."""
    k_noisy = [False] * (L + B) + [True] * (B * B)
    k_block = [-1] * L + list(range(B)) + [i + 1 for i in range(B) for _ in range(B)]
    k_pos = list(range(L + B)) + [L + i + 1 + r for i in range(B) for r in range(B)]
    return O.mask_from_roles(k_noisy[L:], k_block[L:], k_pos[L:], k_noisy, k_block, k_pos)


@pytest.mark.parametrize("L,B", [(5, 1), (7, 3), (4, 4)])
def test_quadratic_attention_equals_dense_masked_bruteforce(L, B):
    rng = np.random.default_rng(10 * L + B)
    Hq, Hkv, D = 4, 2, 8
    K, V = rng.standard_normal((2, Hkv, L + B, D))
    q_ver = rng.standard_normal((B, Hq, D))
    q_cand = rng.standard_normal((B, B, Hq, D))
    k_cand, v_cand = rng.standard_normal((2, B, B, Hkv, D))
    got = O.quadratic_attention(q_ver, q_cand, K, V, L, k_cand, v_cand, 0.3)
    mask = _quad_mask(L, B)
    # a candidate row of block i sees the context, verify rows 0..i and its own B rows
    assert [int(mask[B + i * B].sum()) for i in range(B)] == [L + i + 1 + B for i in range(B)]
    want = O.dense_masked_attention(np.concatenate([q_ver, q_cand.reshape(B * B, Hq, D)]),
                                    np.concatenate([K.transpose(1, 0, 2), k_cand.reshape(B * B, Hkv, D)]),
                                    np.concatenate([V.transpose(1, 0, 2), v_cand.reshape(B * B, Hkv, D)]),
                                    mask, 0.3)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_fused_forward_equals_the_sequential_passes():
    """Verify rows == one causal pass over the draft (same cache writes);
    candidate block k-1 == accepting k draft tokens by a causal pass and then
    running a [MASK] block at L+k as an ordinary noisy pass."""
    gd, d, w, vis, ids = _tiny()
    m, s0 = _fresh(d, w, False, vis, ids)
    B, L = 4, m.L
    rng = np.random.default_rng(3)
    draft = [s0] + [int(t) for t in rng.integers(0, d.vocab - 1, B - 1)]
    mq = copy.deepcopy(m)
    xq = O.forward_quadratic(mq, draft, L)
    assert xq.shape == (B + B * B, d.hidden)
    mv = copy.deepcopy(m)
    xv = mv.forward(mv.embed(draft), L, n_clean=B)
    np.testing.assert_allclose(xq[:B], xv, rtol=0, atol=1e-10)
    for l in range(d.n_layers):
        np.testing.assert_allclose(mq.K[l], mv.K[l], rtol=0, atol=1e-10)
        np.testing.assert_allclose(mq.V[l], mv.V[l], rtol=0, atol=1e-10)
    for k in range(1, B + 1):
        ms = copy.deepcopy(m)
        ms.forward(ms.embed(draft[:k]), L, n_clean=k)
        xs = ms.forward(ms.embed([d.mask_id] * B), L + k, n_clean=0)
        np.testing.assert_allclose(xq[B + (k - 1) * B:B + k * B], xs, rtol=0, atol=1e-10)


@pytest.mark.parametrize("bf16", [False, True])
def test_spec_quadratic_equals_greedy_ar(bf16):
    gd, d, w, vis, ids = _tiny(bf16)
    m1, s1 = _fresh(d, w, bf16, vis, ids)
    ar = O.decode_ar(m1, s1, 24)
    for B in (1, 4):
        m2, s2 = _fresh(d, w, bf16, vis, ids)
        qd = O.decode_spec_quadratic(m2, s2, B, 24)
        assert qd.tokens == ar.tokens
        assert all(1 <= k <= B for k in qd.accept_lens)
        assert qd.nfe == 1 + len(qd.accept_lens)          # one fused forward per round
        assert m2.L == m1.L + sum(qd.accept_lens) - 24
        if B == 1:
            assert qd.accept_lens == [1] * 24


def test_spec_quadratic_drafts_replayed_by_sequential_passes():
    """Every round's draft is [the verifier's token after the accepted
    prefix] + the argmax of an ordinary noisy [MASK] pass placed right after
    that prefix, shifted by one row; replayed with causal and noisy passes."""
    gd, d, w, vis, ids = _tiny()
    B = 4
    m, s0 = _fresh(d, w, False, vis, ids)
    qd = O.decode_spec_quadratic(copy.deepcopy(m), s0, B, 16)
    x = m.forward(m.embed([s0] + [d.mask_id] * (B - 1)), m.L, n_clean=0)
    c = m.logits_conf(x)
    assert qd.drafts[0] == [s0] + [int(c.top1[j - 1]) for j in range(1, B)]
    for r, draft in enumerate(qd.drafts[:-1]):
        L = m.L
        g = m.logits_conf(m.forward(m.embed(draft), L, n_clean=B))
        verify = [draft[0]] + [int(g.top1[j - 1]) for j in range(1, B)]
        k = O.prefix_accept(verify, draft)
        assert k == qd.accept_lens[r]
        m.L = L + k
        probe = copy.deepcopy(m)
        n = probe.logits_conf(probe.forward(probe.embed([d.mask_id] * B), m.L, n_clean=0))
        assert qd.drafts[r + 1] == [int(g.top1[k - 1])] + [int(n.top1[j - 1]) for j in range(1, B)]


class _IdModel:
    """Stub decoder whose rows carry token ids: the LM head's top-1 of a row
    is its first entry.  The first draft's noisy pass predicts 500 + row."""

    def __init__(self):
        self.d = O.Dims(n_layers=1, hidden=1, n_q_heads=1, n_kv_heads=1, head_dim=2, inter=1, vocab=100000)
        self.L = 40

    def embed(self, toks):
        return np.asarray(toks, dtype=np.float64)[:, None]

    def forward(self, x, L, n_clean, hide=0):
        assert n_clean == 0 and L == self.L
        return 500.0 + np.arange(x.shape[0])[:, None]

    def logits_conf(self, x):
        n = x.shape[0]
        return O.Conf(p1=np.ones(n), top1=x[:, 0].astype(np.int64), p2=np.zeros(n))


def test_spec_quadratic_driver_on_a_scripted_model(monkeypatch):
    """Fused forwards scripted: verify row j predicts script[r][j]; row r of
    candidate block i predicts 10000*round + 1000 + 100*i + r.  Accepted
    lengths, seeds, chosen candidate blocks and L worked out by hand."""
    B, script, calls = 4, [[500, 501, 9, 9], [1200, 5, 5, 5], [11100, 11101, 11102, 77]], []

    def fused(model, draft, L):
        r = len(calls)
        assert r < len(script), "one fused forward more than scripted"
        calls.append((list(draft), L))
        cand = [10000 * r + 1000 + 100 * i + q for i in range(B) for q in range(B)]
        return np.asarray(script[r] + cand, dtype=np.float64)[:, None]

    monkeypatch.setitem(O.decode_spec_quadratic.__globals__, "forward_quadratic", fused)
    m = _IdModel()
    tr = O.decode_spec_quadratic(m, 7, B, 9)
    assert tr.drafts == [[7, 500, 501, 502], [9, 1200, 1201, 1202], [5, 11100, 11101, 11102]]
    assert tr.accept_lens == [3, 2, 4] and tr.nfe == 4
    assert tr.tokens == [7, 500, 501, 9, 1200, 5, 11100, 11101, 11102]
    assert [c[1] for c in calls] == [40, 43, 45] and m.L == 49


def test_quadratic_planted_mistakes_are_caught(monkeypatch):
    import oracle.dvlm_oracle as OM

    def mutate(fn_name, old, new, checks, count=1):
        src = inspect.getsource(getattr(OM, fn_name))
        assert src.count(old) == count, old
        ns = dict(vars(OM))
        exec(src.replace(old, new), ns)
        with monkeypatch.context() as mp:
            mp.setattr(OM, fn_name, ns[fn_name])
            mp.setattr(O, fn_name, ns[fn_name])
            for check in checks:
                with pytest.raises(AssertionError):
                    check()

    attn = lambda: test_quadratic_attention_equals_dense_masked_bruteforce(7, 3)
    # candidates see every verify row, not only the accepted prefix
    mutate("quadratic_attention", "[g, :L + i + 1]", "[g, :L + B]", [attn], count=2)
    # candidates see one verify row too few
    mutate("quadratic_attention", "[g, :L + i + 1]", "[g, :L + i]", [attn], count=2)
    # candidate blocks placed one position early (RoPE of the wrong slots)
    mutate("forward_quadratic", "np.arange(L + i + 1, L + i + 1 + B)", "np.arange(L + i, L + i + B)",
           [test_fused_forward_equals_the_sequential_passes])
    scripted = lambda: test_spec_quadratic_driver_on_a_scripted_model(monkeypatch)
    # the next draft taken from the candidate block of one more accepted token
    mutate("decode_spec_quadratic", "rows = B + (k - 1) * B", "rows = B + min(k, B - 1) * B", [scripted])
    # the next draft read without the one-row shift
    mutate("decode_spec_quadratic", "c.top1[rows + j - 1]", "c.top1[rows + j]", [scripted])
    # the next seed taken from the verify row of the last accepted token itself
    mutate("decode_spec_quadratic", "draft = [int(c.top1[k - 1])]", "draft = [int(c.top1[max(k - 2, 0)])]",
           [scripted, lambda: test_spec_quadratic_equals_greedy_ar(False)])


def test_pins_accept_the_oracle():
    _check_rope(O.rope)
    _check_commit(O.threshold_commit)
    _check_cert(O.certificate_scan)
    _check_n2c(O.mask_from_roles)
    _check_attention(O.block_attention)
    _check_argmax(O.confidence_from_logits)


def test_planted_mistakes_are_caught():
    def rope_wrong_sign(x, pos, base=10000.0):
        return O.rope(x, -np.asarray(pos), base)

    def rope_wrong_pairing(x, pos, base=10000.0):      # interleaved pairs instead of halves
        y = O.rope(x.reshape(*x.shape[:-1], -1, 2).swapaxes(-1, -2).reshape(x.shape), pos, base)
        return y.reshape(*x.shape[:-1], 2, -1).swapaxes(-1, -2).reshape(x.shape)

    def commit_strict(p1, masked, tau):
        C = [r for r in range(len(p1)) if masked[r] and p1[r] > tau]
        return C or O.threshold_commit(p1, masked, 2.0)

    def commit_no_force(p1, masked, tau):
        return [r for r in range(len(p1)) if masked[r] and p1[r] >= tau]

    def cert_ascending(a, c, t, part=None):
        return O.certificate_scan(a, [-v for v in c], t, part)

    def cert_tie_high_first(a, c, t, part=None):
        R = len(a)
        idx = sorted(range(R), key=lambda i: (-c[i], -i))
        n = 0
        for i in idx:
            if t[i] != a[i]:
                break
            n += 1
        return n

    def n2c_own_block(qn, qb, qp, kn, kb, kp):
        m = O.mask_from_roles(qn, qb, qp, kn, kb, kp)
        for i in range(len(qn)):
            for j in range(len(kn)):
                if qn[i] and not kn[j] and kb[j] == qb[i]:
                    m[i, j] = 1
        return m

    def attn_clean_sees_block(q, K, V, L, n_clean, scale):
        return O.block_attention(q, K, V, L, 0, scale)

    def attn_no_scale(q, K, V, L, n_clean, scale):
        return O.block_attention(q, K, V, L, n_clean, 1.0)

    def argmax_last(lg):
        c = O.confidence_from_logits(lg)
        c.top1 = lg.shape[-1] - 1 - np.argmax(lg[..., ::-1], axis=-1)
        return c

    for check, mutant in [(_check_rope, rope_wrong_sign), (_check_rope, rope_wrong_pairing),
                          (_check_commit, commit_strict), (_check_commit, commit_no_force),
                          (_check_cert, cert_ascending), (_check_cert, cert_tie_high_first),
                          (_check_n2c, n2c_own_block), (_check_attention, attn_clean_sees_block),
                          (_check_attention, attn_no_scale), (_check_argmax, argmax_last)]:
        with pytest.raises(AssertionError):
            check(mutant)
