"""The ranking rule of the top-k commit kernel, restated on the CPU: a masked
row commits when fewer than k masked rows precede it in the order
(descending p1, ascending position) -- in the divergence-first variant,
divergent rows (TEXT-ONLY top-1 != FULL top-1) before agreeing ones, each
group in that order.  It selects exactly the oracle's set on random inputs
with many ties."""
import numpy as np

import oracle as O


def _kernel_rule(p1, masked, k, agree=None):
    R = len(p1)
    a = agree if agree is not None else [0] * R
    out = []
    for r in range(R):
        rank = sum(1 for s in range(R) if masked[s] and
                   (a[s] < a[r] or (a[s] == a[r] and (p1[s] > p1[r] or (p1[s] == p1[r] and s < r)))))
        if masked[r] and rank < k:
            out.append(r)
    return out


def test_kernel_rule_equals_oracle_topk():
    rng = np.random.default_rng(3)
    for _ in range(400):
        R = int(rng.integers(1, 129))
        p1 = rng.choice(np.array([0.05, 0.3, 0.5, 0.9, 0.91, 1.0]), R)
        masked = list(rng.random(R) < 0.6)
        k = int(rng.integers(0, R + 3))
        assert _kernel_rule(p1, masked, k) == O.topk_commit(p1, masked, k)


def test_kernel_rule_equals_oracle_divergence_first():
    rng = np.random.default_rng(4)
    for _ in range(400):
        R = int(rng.integers(1, 129))
        p1 = rng.choice(np.array([0.05, 0.3, 0.5, 0.9, 0.91, 1.0]), R)
        masked = list(rng.random(R) < 0.6)
        full = rng.integers(0, 3, R)
        text = rng.integers(0, 3, R)
        k = int(rng.integers(0, R + 3))
        agree = [int(full[r] == text[r]) for r in range(R)]
        want = sorted(O.divergence_first_order(full, p1, text, masked)[:k])
        assert _kernel_rule(p1, masked, k, agree) == want


def test_certified_prefix_is_a_topk_over_anchor_confidence():
    """The certified prefix of certificate-guided routing (its length from
    the scan) is the top-n of the masked rows by anchor confidence, so the
    accept branch is the top-k commit with k = the certificate length."""
    rng = np.random.default_rng(5)
    for _ in range(300):
        R = int(rng.integers(1, 40))
        conf = rng.choice(np.array([0.1, 0.4, 0.6, 0.9, 1.0]), R)
        masked = list(rng.random(R) < 0.7)
        anchor = rng.integers(0, 3, R)
        top1 = np.where(rng.random(R) < 0.8, anchor, rng.integers(0, 3, R))
        n = O.certificate_scan(anchor, conf, top1, masked)
        assert O.topk_commit(conf, masked, n) == sorted(O.certificate_order(conf, masked)[:n])
