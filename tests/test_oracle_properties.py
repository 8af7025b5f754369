"""Property checks of the oracle's decision rules on random inputs, each
against a second, independent formulation of the same definition (array
primitives instead of the oracle's loops and sorts).  Ties are drawn on
purpose: values come from a small grid."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle as O

GRID = [0.05, 0.3, 0.5, 0.9, 0.91, 1.0]


def rows(min_size=0, max_size=12):
    return st.integers(min_size, max_size).flatmap(
        lambda n: st.tuples(st.lists(st.sampled_from(GRID), min_size=n, max_size=n),
                            st.lists(st.booleans(), min_size=n, max_size=n)))


@settings(max_examples=300, deadline=None)
@given(rows(), st.sampled_from([0.0, 0.5, 0.9, 0.91, 2.0]))
def test_threshold_commit_property(pm, tau):
    """Pages' rule: commit masked rows with p1 >= tau; if none, the first
    masked row attaining the largest p1 (np.argmax keeps the first maximum)."""
    p, m = np.array(pm[0]), np.array(pm[1], dtype=bool)
    want = list(np.nonzero(m & (p >= tau))[0])
    if not want and m.any():
        want = [int(np.argmax(np.where(m, p, -np.inf)))]
    assert O.threshold_commit(p, m, tau) == want


@settings(max_examples=300, deadline=None)
@given(rows(), st.integers(0, 13))
def test_topk_commit_property(pm, k):
    """The k masked rows of highest p1, earlier rows first on ties: a stable
    sort on -p1 over the masked rows, then the first k, reported in order."""
    p, m = np.array(pm[0]), np.array(pm[1], dtype=bool)
    idx = np.nonzero(m)[0]
    order = idx[np.argsort(-p[idx], kind="stable")]
    assert O.topk_commit(p, m, k) == sorted(int(i) for i in order[:k])


@settings(max_examples=300, deadline=None)
@given(rows(), st.data())
def test_certificate_scan_property(pm, data):
    """Certified prefix = the rank (in descending anchor confidence, earlier
    position first) of the first participant that disagrees, or the number of
    participants when none does."""
    conf, part = np.array(pm[0]), np.array(pm[1], dtype=bool)
    n = len(conf)
    anchor = np.array(data.draw(st.lists(st.integers(0, 3), min_size=n, max_size=n)), dtype=np.int64)
    top1 = np.array(data.draw(st.lists(st.integers(0, 3), min_size=n, max_size=n)), dtype=np.int64)
    idx = np.nonzero(part)[0]
    order = idx[np.lexsort((idx, -conf[idx]))]
    bad = np.nonzero(top1[order] != anchor[order])[0]
    want = int(bad[0]) if len(bad) else len(order)
    assert O.certificate_scan(anchor, conf, top1, part) == want
    assert O.certificate_order(conf, part) == [int(i) for i in order]


@settings(max_examples=300, deadline=None)
@given(st.integers(0, 16).flatmap(lambda n: st.tuples(st.lists(st.integers(0, 2), min_size=n, max_size=n),
                                                      st.lists(st.integers(0, 2), min_size=n, max_size=n))))
def test_prefix_accept_property(vd):
    """Longest agreeing prefix = the index of the first mismatch, or the length."""
    v, d = np.array(vd[0], dtype=np.int64), np.array(vd[1], dtype=np.int64)
    mis = np.nonzero(v != d)[0]
    assert O.prefix_accept(v, d) == (int(mis[0]) if len(mis) else len(v))


@settings(max_examples=200, deadline=None)
@given(rows(), st.data())
def test_divergence_first_order_property(pm, data):
    """Divergent positions (TEXT-ONLY top-1 != FULL top-1) first, then the
    agreeing ones; inside each group descending FULL confidence, earlier
    position first: a lexsort on (position, -confidence, agreement)."""
    conf, part = np.array(pm[0]), np.array(pm[1], dtype=bool)
    n = len(conf)
    full = np.array(data.draw(st.lists(st.integers(0, 2), min_size=n, max_size=n)), dtype=np.int64)
    text = np.array(data.draw(st.lists(st.integers(0, 2), min_size=n, max_size=n)), dtype=np.int64)
    idx = np.nonzero(part)[0]
    agree = (full[idx] == text[idx]).astype(int)
    order = idx[np.lexsort((idx, -conf[idx], agree))]
    assert O.divergence_first_order(full, conf, text, part) == [int(i) for i in order]
