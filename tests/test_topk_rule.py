"""The ranking rule of the top-k commit kernel, restated on the CPU: a masked
row commits when fewer than k masked rows precede it in the order
(descending p1, ascending position).  It selects exactly the oracle's set on
random inputs with many ties."""
import numpy as np

import oracle as O


def _kernel_rule(p1, masked, k):
    R = len(p1)
    out = []
    for r in range(R):
        rank = sum(1 for s in range(R) if masked[s] and (p1[s] > p1[r] or (p1[s] == p1[r] and s < r)))
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
