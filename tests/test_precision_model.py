"""numpy models of the GPU path's arithmetic (not of its code) against the
fp64 oracle: they show how much of each parity bar the precision choices use.

Attention (bar 2e-2).  A numpy model of the arithmetic of the bf16 attention
path: fp32 scores from bf16 q and k; keys split over 16 cooperating CTAs in
64-key chunks taken round-robin; each CTA's probabilities exp2(s - m_cta)
rounded to fp16 and multiplied by the fp16 copy of V with fp32 accumulation;
each CTA's partial rows divided by its own sum and exchanged in fp16; merged
with weights exp2(m_cta - M) * l_cta; the output stored in bf16.  Measured
against the fp64 oracle on the block-attention configuration's inputs: the
error is the bf16 store's rounding plus well under 1e-3, a small fraction of
the bar."""
import math

import numpy as np
import pytest
import torch

import dvlm_gen as gen
import oracle as O

TOL_BF16 = 2e-2
CHUNK, SPLIT = 64, 16


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def model_attention(q, k, v, L, scale):
    """q [n, Hq, D], k/v [Hkv, >= L+n, D] (bf16 values as float32); noisy rows
    see slots 0..L+n-1."""
    n, Hq, D = q.shape
    G = Hq // k.shape[0]
    nk = L + n
    s2 = scale * math.log2(math.e)
    out = np.zeros((n, Hq, D), dtype=np.float32)
    chunks = [np.arange(c, min(c + CHUNK, nk)) for c in range(0, nk, CHUNK)]
    for h in range(Hq):
        kk, vv = k[h // G, :nk], v[h // G, :nk]
        s = (q[:, h].astype(np.float32) @ kk.T.astype(np.float32)) * np.float32(s2)     # [n, nk] fp32
        parts = []
        for c in range(SPLIT):
            idx = np.concatenate([chunks[j] for j in range(c, len(chunks), SPLIT)] or [np.zeros(0, int)])
            if len(idx) == 0:
                continue
            m = s[:, idx].max(axis=1, keepdims=True)
            p = np.exp2(s[:, idx] - m).astype(np.float32)
            l_ = p.sum(axis=1, keepdims=True, dtype=np.float32)
            o = p.astype(np.float16).astype(np.float32) @ vv[idx].astype(np.float16).astype(np.float32)
            parts.append((m, l_, (o / l_).astype(np.float16).astype(np.float32)))
        M = np.max([m for m, _, _ in parts], axis=0)
        w = [np.exp2(m - M) * l_ for m, l_, _ in parts]
        num = sum(wi * oi for wi, (_, _, oi) in zip(w, parts))
        out[:, h] = num / sum(w)
    return _bf16(out)


@pytest.mark.parametrize("B,L", [(16, 1344), (16, 4096), (32, 4096), (4, 256)])
def test_attention_precision_uses_a_fraction_of_the_bar(B, L):
    q, k, v = (t.float().numpy() for t, _ in gen.attn_case(1, B, L))
    scale = 1.0 / math.sqrt(q.shape[-1])
    got = model_attention(q[0], k[0], v[0], L, scale)
    want = O.block_attention(q[0].astype(np.float64), k[0].astype(np.float64), v[0].astype(np.float64), L, 0,
                             scale)
    err = float(np.abs(got - want).max())
    # the bf16 store alone may cost half an ulp, at most 2^-8 of |out|; the
    # fp16 probabilities and partial rows add at most a few 1e-4 on top
    assert err <= 2.0 ** -8 * float(np.abs(want).max()) + 2e-4, err
    assert err < TOL_BF16 / 4, err


# the reduced bf16 decoder of the GPU decode tests
SMALL_BF16 = gen.ModelDims(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=1, head_dim=128, inter=1024,
                           vocab=4096, lm_scale=25.0, dtype="bf16")
TEACHER_FORCED_DELTA = 0.1


@pytest.mark.parametrize("seed", [1, 3])
def test_bf16_storage_flips_move_p1_by_hundredths(seed):
    """Why bf16 decoding is compared teacher-forced with a 0.1 margin.  Every
    stored activation of a copy of the oracle is perturbed by about 5e-7
    relative before its bf16 rounding (less than fp32 and fp64 sums of 1024
    terms differ by), which flips a few roundings by one ulp; the oracle's
    threshold trajectory is then replayed on that copy over the same block
    tokens.  Top-1 probabilities move by a few 1e-2: a 1e-3 margin cannot
    hold on bf16 storage, 0.1 does (largest move seen over 14 such draws on
    these two seeds: 0.066)."""
    w = O.weights_from_generator(gen, SMALL_BF16, seed)
    od = O.dims_from(SMALL_BF16)
    _, vis, ids = gen.decode_context(SMALL_BF16, seed, 32, 16, 0)
    ref = O.OracleModel(od, weights=w, bf16=True, Lmax=256)
    pert = O.OracleModel(od, weights=w, bf16=True, Lmax=256)
    rng = np.random.default_rng(100)
    pert.rnd = lambda x: O.bf16_round(np.asarray(x) * (1 + 2.0 ** -21 * rng.standard_normal(np.shape(x))))
    s = O.prefill(ref, vis.astype(np.float64), ids)
    assert O.prefill(pert, vis.astype(np.float64), ids) == s
    moves = []

    def on_iter(L, toks, masked, p1o, topo, p2o):
        c = pert.logits_conf(pert.forward(pert.embed(toks), L, n_clean=0))
        moves.extend(abs(c.p1[j - 1] - p1o[j]) for j in range(1, len(toks)) if masked[j])

    def on_block(L, toks):
        pert.forward(pert.embed(toks), L, n_clean=len(toks))
        pert.L = L + len(toks)

    O.decode_threshold(ref, s, 16, 0.9, 32, on_iter=on_iter, on_block=on_block)
    assert 0.01 < max(moves) < TEACHER_FORCED_DELTA, max(moves)


def test_lmhead_p1_precision_within_its_bar():
    """The fused LM head's p1 bar (2e-4 against the fp64 oracle): bf16 hidden
    rows and weights, logits summed in fp32, softmax sum and maximum in fp32.
    On the configuration's distributions (hidden N(0,1), W N(0, 0.02) x 25,
    H = 2048; a 16384-row slice of the vocabulary, the per-logit arithmetic
    being the same) p1 moves by orders of magnitude less than the bar."""
    H, V, R = 2048, 16384, 16
    (_, h), (_, w) = gen.lmhead_case(2, R, H, V, second_set=False)
    lg32 = h.astype(np.float32) @ w.astype(np.float32).T
    m = lg32.max(axis=1, keepdims=True)
    p1_32 = 1.0 / np.exp(lg32 - m).sum(axis=1, dtype=np.float32)
    want = O.lm_head_conf(h.astype(np.float64), w.astype(np.float64))
    err = float(np.abs(p1_32 - want.p1).max())
    assert err < 2e-4 / 20, err
    assert np.array_equal(lg32.argmax(axis=1)[want.p1 - want.p2 >= 1e-3], want.top1[want.p1 - want.p2 >= 1e-3])
