"""Teacher-forced replay of the decode engine's forward trace against the oracle.

The engine records every forward its decode driver runs (dvlm_engine_set_trace:
block tokens and masked flags before and after, the LM head's per-row top-1
id and probability, the next AR seed, the cache length, and the final
residual-stream rows).  This module walks such a trace and holds each forward
to the oracle:

* hidden rows: the oracle runs the same forward (same tokens, same cache
  slots) on its own cache and the GPU's rows must agree within the hidden
  bar;
* decisions: top-1 ids, commit sets, accepted lengths and seeds must be
  bit-exact wherever the deciding confidences are at least MARGIN (1e-3)
  away from their boundary (p1 - p2 for an id; |p1 - tau| for a threshold
  decision; the gap between the two best p1 for a forced commit).  Where a
  decision sits closer than that, the GPU may take any of the tied choices
  and the oracle is teacher-forced to it;
* the engine's own rule: its commit set is the commit rule applied to its own
  probabilities, committed tokens are its own top-1 ids, accepted lengths
  are the agreeing prefixes of its own draft and verify ids.

Which confidences decide (`decide`):
  "oracle"  the oracle's own hidden rows (fp32 models, where the GPU's hidden
            rows agree with the oracle's to ~1e-6);
  "gpu"     the oracle's LM head applied to the GPU's final hidden rows: the
            fused LM head + commit is checked at the 1e-3 bar on the very rows
            it read (bf16 models, where one-ulp storage flips in the hidden
            rows move p1 by up to a few 1e-2).  The oracle's own rows are then
            held to the looser `secondary` bar as well.

No expected value comes from the GPU: hidden rows are compared with the
oracle's, decisions with the oracle's scores; GPU outputs enter the oracle
only as teacher-forced tokens at excluded positions and, with decide="gpu",
as the input rows of the LM-head check.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional

import numpy as np

import oracle as O

MARGIN = 1e-3
NOISY, APPEND, DRAFT, VERIFY, AR, QUAD_VERIFY, QUAD_CAND, ROUTE_FULL, ROUTE_TEXT = 1, 2, 3, 4, 5, 6, 7, 8, 9
NT = 16
WORDS = 112


@dataclasses.dataclass
class Rec:
    kind: int
    L: int
    n_rows: int
    n_clean: int
    R: int
    tok_in: np.ndarray
    msk_in: np.ndarray
    top1: np.ndarray
    p1: np.ndarray
    tok_out: np.ndarray
    msk_out: np.ndarray
    seed_out: int
    len_out: int
    x: np.ndarray          # [n_rows, H] float64 (exact bf16 / fp32 values)


def parse_trace(raw: np.ndarray, count: int, rec_bytes: int, hidden: int, bf16: bool) -> List[Rec]:
    """Records of a trace buffer copied to the host (uint8 array)."""
    out = []
    raw = np.ascontiguousarray(raw).view(np.uint8)
    for i in range(count):
        r = raw[i * rec_bytes:(i + 1) * rec_bytes]
        w = r[:WORDS * 4].view(np.int32)
        n = int(w[2])
        if bf16:
            u = r[WORDS * 4:WORDS * 4 + NT * hidden * 2].view(np.uint16).astype(np.uint32) << 16
            x = u.view(np.float32).reshape(NT, hidden)
        else:
            x = r[WORDS * 4:WORDS * 4 + NT * hidden * 4].view(np.float32).reshape(NT, hidden)
        out.append(Rec(kind=int(w[0]), L=int(w[1]), n_rows=n, n_clean=int(w[3]), R=int(w[4]),
                       tok_in=w[8:8 + n].copy(), msk_in=w[24:24 + n].astype(bool), top1=w[40:40 + NT].copy(),
                       p1=w[56:56 + NT].view(np.float32).astype(np.float64), tok_out=w[72:72 + n].copy(),
                       msk_out=w[88:88 + n].astype(bool), seed_out=int(w[104]), len_out=int(w[105]),
                       x=x[:n].astype(np.float64)))
    return out


@dataclasses.dataclass
class Tally:
    forwards: int = 0
    ids_exact: int = 0           # ids held bit-exact (margin >= MARGIN)
    ids_excluded: int = 0        # ids inside the margin (any tied choice accepted)
    commits_exact: int = 0       # commit decisions held bit-exact
    commits_excluded: int = 0
    accepts_exact: int = 0
    accepts_excluded: int = 0
    secondary_checked: int = 0
    hidden_max_err: float = 0.0
    p1_max_err: float = 0.0


class Replay:
    """Walks a trace of threshold, speculative or AR decoding.

    model: an oracle model prefilled by the oracle itself (model.L and
    model.last_conf set); seed: the oracle's AR seed from that prefill.
    hidden_check(x_gpu, x_oracle, what) asserts the hidden bar.  p1_tol
    bounds |p1(GPU) - p1(deciding oracle)|.  seed_bar: margin for the first
    AR seed, which comes from the prefill (scored by the oracle's own rows:
    the prefill is not traced; None: not checked, only teacher-forced).
    hidden_fn(index, record) returns the
    oracle's final rows of a record computed beforehand (layer-major replay,
    see layer_major_hidden); by default each record runs model.forward."""

    def __init__(self, model: O.OracleModel, seed: int, B: int, tau: float, decide: str,
                 hidden_check: Callable, p1_tol: float = 2e-4, secondary: Optional[float] = None,
                 seed_bar: float = MARGIN, hidden_fn: Optional[Callable] = None):
        assert decide in ("oracle", "gpu")
        self.m, self.B, self.tau, self.decide = model, B, tau, decide
        self.hidden_check, self.p1_tol, self.secondary = hidden_check, p1_tol, secondary
        self.hidden_fn = hidden_fn
        self.t = Tally()
        self.seed = seed
        self.seed_conf = model.last_conf      # scores the first seed (row 0)
        self.seed_bar = seed_bar
        self.tokens: List[int] = []

    # -- scoring -------------------------------------------------------------
    def _oracle_rows(self, rec: Rec, idx: int) -> np.ndarray:
        if self.hidden_fn is not None:
            return self.hidden_fn(idx, rec)
        x = self.m.forward(self.m.embed(rec.tok_in), rec.L, rec.n_clean)
        return x

    def _confs(self, rec: Rec, x_o: np.ndarray):
        """(deciding conf, oracle's own conf) of the record's rows."""
        c_o = self.m.logits_conf(x_o)
        if self.decide == "oracle":
            return c_o, c_o
        return self.m.logits_conf(rec.x), c_o

    def _id(self, gpu_id: int, c: O.Conf, r: int, what: str) -> None:
        if c.p1[r] - c.p2[r] >= MARGIN:
            assert gpu_id == c.top1[r], (what, r, gpu_id, int(c.top1[r]), float(c.p1[r]), float(c.p2[r]))
            self.t.ids_exact += 1
        else:
            assert gpu_id in (int(c.top1[r]), int(c.top2[r])), (what, r, gpu_id, int(c.top1[r]), int(c.top2[r]))
            self.t.ids_excluded += 1

    def _secondary(self, gpu_p1: float, gpu_id: int, c: O.Conf, r: int, what: str) -> None:
        if self.secondary is None or self.decide == "oracle":
            return
        d = self.secondary
        assert abs(gpu_p1 - c.p1[r]) <= d, (what, r, gpu_p1, float(c.p1[r]))
        if c.p1[r] - c.p2[r] >= d:
            assert gpu_id == c.top1[r], (what, r, gpu_id, int(c.top1[r]))
        self.t.secondary_checked += 1

    def _row_checks(self, rec: Rec, rows, c: O.Conf, c_o: O.Conf, what: str) -> None:
        for r in rows:
            err = abs(rec.p1[r] - c.p1[r])
            self.t.p1_max_err = max(self.t.p1_max_err, err)
            assert err <= self.p1_tol, (what, r, float(rec.p1[r]), float(c.p1[r]))
            self._secondary(rec.p1[r], int(rec.top1[r]), c_o, r, what)

    def _seed_check(self, gpu_seed: int) -> None:
        c = self.seed_conf
        if self.seed_bar is None:   # the first seed is only teacher-forced
            c = None
        if c is not None:
            if c.p1[0] - c.p2[0] >= self.seed_bar:
                assert gpu_seed == c.top1[0], ("seed", gpu_seed, int(c.top1[0]))
                self.t.ids_exact += 1
            else:
                assert gpu_seed in (int(c.top1[0]), int(c.top2[0])), ("seed", gpu_seed)
                self.t.ids_excluded += 1
        self.seed = gpu_seed      # teacher-forced
        self.seed_bar = MARGIN    # later seeds come from traced rows

    def _forward(self, rec: Rec, idx: int, what: str):
        assert rec.L == self.m.L, (what, rec.L, self.m.L)
        x_o = self._oracle_rows(rec, idx)
        self.hidden_check(rec.x, x_o, what)
        self.t.hidden_max_err = max(self.t.hidden_max_err, float(np.max(np.abs(rec.x - x_o))))
        self.t.forwards += 1
        return self._confs(rec, x_o)

    # -- the three drivers -----------------------------------------------------
    def threshold(self, recs: List[Rec], max_new: int) -> List[int]:
        B, tau, mask_id = self.B, self.tau, self.m.d.mask_id
        i = 0
        while len(self.tokens) < max_new:
            rec = recs[i]
            assert rec.kind == NOISY, (i, rec.kind)
            self._seed_check(int(rec.tok_in[0]))
            toks = [self.seed] + [mask_id] * (B - 1)
            masked = [False] + [True] * (B - 1)
            while any(masked):
                rec = recs[i]
                assert rec.kind == NOISY and rec.n_rows == B and rec.n_clean == 0 and rec.R == B - 1, (i, rec)
                assert list(rec.tok_in) == toks and list(rec.msk_in) == masked, (i, rec.tok_in, toks)
                c, c_o = self._forward(rec, i, f"noisy #{i}")
                self._row_checks(rec, [j - 1 for j in range(1, B) if masked[j]], c, c_o, f"noisy #{i}")
                self._commits(rec, c, masked, toks, tau, i)
                toks, masked = list(rec.tok_out), list(rec.msk_out)
                i += 1
            rec = recs[i]
            assert rec.kind == APPEND and rec.n_clean == B and list(rec.tok_in) == toks, (i, rec.kind)
            c, c_o = self._forward(rec, i, f"append #{i}")
            self.m.L += B
            assert rec.len_out == self.m.L, (i, rec.len_out, self.m.L)
            self._row_checks(rec, [B - 1], c, c_o, f"append #{i}")
            assert rec.seed_out == rec.top1[B - 1]
            self.seed_conf = O.Conf(p1=c.p1[B - 1:], top1=c.top1[B - 1:], p2=c.p2[B - 1:], top2=c.top2[B - 1:])
            self.tokens.extend(toks)
            i += 1
        self._next = i
        return self.tokens[:max_new]

    def _commits(self, rec: Rec, c: O.Conf, masked, toks, tau: float, i: int) -> None:
        B = self.B
        p1g = np.zeros(B)
        topg = np.zeros(B, dtype=np.int64)
        po = np.zeros(B)
        for j in range(1, B):
            p1g[j], topg[j], po[j] = rec.p1[j - 1], rec.top1[j - 1], c.p1[j - 1]
        Cg = [j for j in range(B) if masked[j] and not rec.msk_out[j]]
        # the engine's own rule on its own probabilities, bit for bit
        assert Cg == O.threshold_commit(p1g, masked, tau), (i, Cg, list(p1g))
        for j in range(B):
            want = topg[j] if j in Cg else toks[j]
            assert rec.tok_out[j] == want, (i, j)
        # against the oracle's scores, except inside the margin
        live = [j for j in range(B) if masked[j]]
        forced = not any(p1g[j] >= tau for j in live)
        for j in live:
            if abs(po[j] - tau) < MARGIN:
                self.t.commits_excluded += 1
                continue
            if po[j] >= tau:
                assert j in Cg, (i, j, po[j])
                self.t.commits_exact += 1
            elif not forced:
                assert j not in Cg, (i, j, po[j])
                self.t.commits_exact += 1
        if forced:
            assert not any(po[j] >= tau + MARGIN for j in live), (i, "forced commit while the oracle passes")
            (jg,) = Cg
            best = max(po[j] for j in live)
            assert po[jg] >= best - MARGIN, (i, jg, po[jg], best)
            second = max([po[j] for j in live if po[j] < best] + [-1.0])
            jo = min(j for j in live if po[j] == best)
            if best - second >= MARGIN and best <= tau - MARGIN:
                assert jg == jo, (i, jg, jo)
                self.t.commits_exact += 1
            else:
                self.t.commits_excluded += 1
        for j in Cg:
            self._id(int(topg[j]), c, j - 1, f"noisy #{i} id")

    def speculative(self, recs: List[Rec], max_new: int, final_L: int, final_seed: int) -> List[int]:
        B, mask_id = self.B, self.m.d.mask_id
        i = 0
        while len(self.tokens) < max_new:
            dr, ve = recs[i], recs[i + 1]
            assert dr.kind == DRAFT and ve.kind == VERIFY, (i, dr.kind, ve.kind)
            self._seed_check(int(dr.tok_in[0]))
            toks = [self.seed] + [mask_id] * (B - 1)
            assert list(dr.tok_in) == toks and list(dr.msk_in) == [False] + [True] * (B - 1)
            c, c_o = self._forward(dr, i, f"draft #{i}")
            self._row_checks(dr, range(B - 1), c, c_o, f"draft #{i}")
            draft = [self.seed] + [int(dr.top1[j - 1]) for j in range(1, B)]
            assert list(dr.tok_out) == draft, (i, list(dr.tok_out), draft)
            for j in range(1, B):
                self._id(draft[j], c, j - 1, f"draft #{i}")
            L = self.m.L
            assert list(ve.tok_in) == draft and ve.n_clean == B and ve.L == L
            g, g_o = self._forward(ve, i + 1, f"verify #{i + 1}")
            self._row_checks(ve, range(B), g, g_o, f"verify #{i + 1}")
            ver = [self.seed] + [int(ve.top1[j - 1]) for j in range(1, B)]
            k = O.prefix_accept(ver, draft)
            # the engine's accept: the next round starts at L + k with seed v_k
            if i + 2 < len(recs):
                nL, nseed = recs[i + 2].L, int(recs[i + 2].tok_in[0])
            else:
                nL, nseed = final_L, final_seed
            assert nL == L + k, (i, nL, L, k)
            assert nseed == int(ve.top1[k - 1]), (i, nseed)
            # verifier ids on the accepted prefix and at its end, against the oracle
            sure = all(g.p1[j - 1] - g.p2[j - 1] >= MARGIN for j in range(1, min(k + 1, B)))
            for j in range(1, min(k + 1, B)):
                self._id(ver[j], g, j - 1, f"verify #{i + 1}")
            if sure:
                self.t.accepts_exact += 1
            else:
                self.t.accepts_excluded += 1
            self.tokens.extend(draft[:k])
            self.m.L = L + k
            self.seed_conf = O.Conf(p1=g.p1[k - 1:k], top1=g.top1[k - 1:k], p2=g.p2[k - 1:k],
                                    top2=g.top2[k - 1:k])
            i += 2
        self._next = i
        return self.tokens[:max_new]

    def quadratic(self, recs: List[Rec], max_new: int, final_L: int, final_seed: int) -> List[int]:
        """Quadratic self-speculative decoding: a diffusion draft pass, then per
        round one fused forward (the oracle's forward_quadratic over the
        draft) recorded as its verify rows (QUAD_VERIFY) and the chosen
        candidate block's rows (QUAD_CAND, cache length already L + k)."""
        B, mask_id = self.B, self.m.d.mask_id
        assert B >= 2
        dr = recs[0]
        assert dr.kind == DRAFT, dr.kind
        self._seed_check(int(dr.tok_in[0]))
        toks = [self.seed] + [mask_id] * (B - 1)
        assert list(dr.tok_in) == toks and list(dr.msk_in) == [False] + [True] * (B - 1)
        c, c_o = self._forward(dr, 0, "draft #0")
        self._row_checks(dr, range(B - 1), c, c_o, "draft #0")
        draft = [self.seed] + [int(dr.top1[j - 1]) for j in range(1, B)]
        assert list(dr.tok_out) == draft
        for j in range(1, B):
            self._id(draft[j], c, j - 1, "draft #0")
        i = 1
        while len(self.tokens) < max_new:
            rv, rc = recs[i], recs[i + 1]
            assert rv.kind == QUAD_VERIFY and rc.kind == QUAD_CAND, (i, rv.kind, rc.kind)
            L = self.m.L
            assert rv.L == L and list(rv.tok_in) == draft, (i, rv.L, L)
            x_all = O.forward_quadratic(self.m, draft, L)
            self.hidden_check(rv.x, x_all[:B], f"quad verify #{i}")
            self.t.hidden_max_err = max(self.t.hidden_max_err, float(np.max(np.abs(rv.x - x_all[:B]))))
            self.t.forwards += 1
            g, g_o = self._confs(rv, x_all[:B])
            self._row_checks(rv, range(B), g, g_o, f"quad verify #{i}")
            ver = [draft[0]] + [int(rv.top1[j - 1]) for j in range(1, B)]
            k = O.prefix_accept(ver, draft)
            sure = all(g.p1[j - 1] - g.p2[j - 1] >= MARGIN for j in range(1, min(k + 1, B)))
            for j in range(1, min(k + 1, B)):
                self._id(ver[j], g, j - 1, f"quad verify #{i}")
            self.t.accepts_exact += 1 if sure else 0
            self.t.accepts_excluded += 0 if sure else 1
            # the engine kept k tokens and seeded the next draft with v_k
            assert rc.L == L + k, (i, rc.L, L, k)
            v_k = int(rv.top1[k - 1])
            assert int(rc.tok_in[0]) == v_k and list(rc.msk_in) == [False] + [True] * (B - 1)
            xc = x_all[B + (k - 1) * B:B + k * B]
            self.hidden_check(rc.x, xc, f"quad candidate #{i + 1}")
            cc, cc_o = self._confs(rc, xc)
            self._row_checks(rc, range(B - 1), cc, cc_o, f"quad candidate #{i + 1}")
            nd = [v_k] + [int(rc.top1[j - 1]) for j in range(1, B)]
            assert list(rc.tok_out) == nd, (i, list(rc.tok_out), nd)
            for j in range(1, B):
                self._id(nd[j], cc, j - 1, f"quad candidate #{i + 1}")
            self.tokens.extend(draft[:k])
            self.m.L = L + k
            draft = nd
            i += 2
        assert self.m.L == final_L and draft[0] == final_seed, (self.m.L, final_L, draft[0], final_seed)
        self._next = i
        return self.tokens[:max_new]

    def _append(self, recs: List[Rec], i: int, toks) -> None:
        B = self.B
        rec = recs[i]
        assert rec.kind == APPEND and rec.n_clean == B and list(rec.tok_in) == toks, (i, rec.kind)
        c, c_o = self._forward(rec, i, f"append #{i}")
        self.m.L += B
        assert rec.len_out == self.m.L, (i, rec.len_out, self.m.L)
        self._row_checks(rec, [B - 1], c, c_o, f"append #{i}")
        assert rec.seed_out == rec.top1[B - 1]
        self.seed_conf = O.Conf(p1=c.p1[B - 1:], top1=c.top1[B - 1:], p2=c.p2[B - 1:], top2=c.top2[B - 1:])
        self.tokens.extend(toks)

    def _set_check(self, chosen, p1_oracle, masked, n, what) -> None:
        """The n positions the engine chose by its own confidences, against the
        choice the deciding confidences make, wherever the n-th and (n+1)-th
        largest are at least MARGIN apart (the choice is then unique)."""
        live = sorted((-p1_oracle[j], j) for j in range(self.B) if masked[j])
        if n < len(live) and -live[n - 1][0] - (-live[n][0]) < MARGIN:
            self.t.commits_excluded += 1
            return
        assert sorted(chosen) == sorted(j for _, j in live[:n]), (what, sorted(chosen), live[:n + 1])
        self.t.commits_exact += 1

    def routing(self, recs: List[Rec], max_new: int, k: int, n_vis: int) -> List[int]:
        """Certificate-guided routing [LOWN steps (1)-(3)]: FULL passes set the
        anchors, TEXT-ONLY passes (vision slots hidden) are certified against
        them.  The engine's own rule on its own values is held exactly (the
        certified length, the committed positions and ids, read from the next
        record's block state); its values are held to the oracle."""
        B, mask_id = self.B, self.m.d.mask_id
        i = 0
        while len(self.tokens) < max_new:
            self._seed_check(int(recs[i].tok_in[0]))
            toks = [self.seed] + [mask_id] * (B - 1)
            masked = [False] + [True] * (B - 1)
            anc_id = anc_p1 = text_top = None
            while any(masked):
                kk = min(k, sum(masked))
                rec, nxt = recs[i], recs[i + 1]
                assert list(rec.tok_in) == toks and list(rec.msk_in) == masked, (i, list(rec.tok_in), toks)
                L = self.m.L
                assert rec.L == L
                top = np.array([-1] + [int(rec.top1[j - 1]) for j in range(1, B)])
                p1g = np.array([0.0] + [float(rec.p1[j - 1]) for j in range(1, B)])
                live = [j for j in range(B) if masked[j]]
                if anc_id is not None:
                    assert rec.kind == ROUTE_TEXT, (i, rec.kind)
                    x_o = self.m.forward(self.m.embed(toks), L, 0, hide=n_vis)
                    self.hidden_check(rec.x, x_o, f"text #{i}")
                    self.t.forwards += 1
                    c, c_o = self._confs(rec, x_o)
                    self._row_checks(rec, [j - 1 for j in live], c, c_o, f"text #{i}")
                    text_top = top
                    order = O.certificate_order(anc_p1, masked)
                    n = O.certificate_scan(anc_id, anc_p1, text_top, masked)
                    for j in order[:n + 1]:           # the scanned rows decide the certificate
                        self._id(int(text_top[j]), c, j - 1, f"text #{i}")
                    if n >= kk:
                        want_t, want_m = list(toks), list(masked)
                        for j in order[:n]:
                            want_t[j], want_m[j] = int(anc_id[j]), False
                        assert list(nxt.tok_in) == want_t and list(nxt.msk_in) == want_m, (i, "certified commit")
                        toks, masked = want_t, want_m
                        i += 1
                        continue
                    rec, nxt = recs[i + 1], recs[i + 2]
                    i += 1
                    assert list(rec.tok_in) == toks and list(rec.msk_in) == masked
                    top = np.array([-1] + [int(rec.top1[j - 1]) for j in range(1, B)])
                    p1g = np.array([0.0] + [float(rec.p1[j - 1]) for j in range(1, B)])
                assert rec.kind == ROUTE_FULL, (i, rec.kind)
                x_o = self.m.forward(self.m.embed(toks), L, 0)
                self.hidden_check(rec.x, x_o, f"full #{i}")
                self.t.forwards += 1
                c, c_o = self._confs(rec, x_o)
                self._row_checks(rec, [j - 1 for j in live], c, c_o, f"full #{i}")
                if text_top is None:
                    order = O.certificate_order(p1g, masked)
                else:
                    order = O.divergence_first_order(top, p1g, text_top, masked)
                want_t, want_m = list(toks), list(masked)
                for j in order[:kk]:
                    want_t[j], want_m[j] = int(top[j]), False
                    self._id(int(top[j]), c, j - 1, f"full #{i}")
                assert list(nxt.tok_in) == want_t and list(nxt.msk_in) == want_m, (i, "FULL commit")
                if text_top is None:   # the plain top-k choice, also by the deciding confidences
                    po = np.array([0.0] + [float(c.p1[j - 1]) for j in range(1, B)])
                    self._set_check(order[:kk], po, masked, kk, f"full #{i}")
                anc_id, anc_p1 = top, p1g
                toks, masked = want_t, want_m
                i += 1
            self._append(recs, i, toks)
            i += 1
        self._next = i
        return self.tokens[:max_new]

    def autoregressive(self, recs: List[Rec], max_new: int) -> List[int]:
        i = 0
        while len(self.tokens) < max_new:
            rec = recs[i]
            assert rec.kind == AR and rec.n_rows == 1 and rec.n_clean == 1, (i, rec.kind)
            self._seed_check(int(rec.tok_in[0]))
            c, c_o = self._forward(rec, i, f"ar #{i}")
            self.m.L += 1
            self._row_checks(rec, [0], c, c_o, f"ar #{i}")
            assert rec.seed_out == rec.top1[0] and rec.len_out == self.m.L
            self.seed_conf = c
            self.tokens.append(self.seed)
            i += 1
        self._next = i
        return self.tokens[:max_new]


def layer_major_hidden(model: O.OracleModel, passes, layer_weights: Callable[[int], dict]):
    """Final hidden rows of a sequence of forwards, computed layer by layer.

    passes: list of (input rows [n, H], cache slot of row 0, clean rows).
    For each layer the weights are drawn once (layer_weights(l) -> the
    oracle's '{l}.w*' matrices) and every forward's rows pass through that
    layer in order.  A forward at a layer reads only that layer's cache as
    the forwards before it left it, so this equals running the forwards one
    after another through all layers.  Returns one [n, H] array per pass;
    model.K / model.V end as after the last forward (model.L unchanged)."""
    xs = [np.asarray(x, dtype=np.float64) for x, _, _ in passes]
    for l in range(model.d.n_layers):
        w = layer_weights(l)
        saved = model._w
        model._w = dict(saved or {})
        model._w.update(w)
        for i, (_, L, n_clean) in enumerate(passes):
            xs[i] = model.layer(l, xs[i], L, n_clean)
        model._w = saved
    return xs
