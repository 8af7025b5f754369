"""CPU oracle of the block-diffusion decode step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may import this module.  The product path (the C-ABI library and
its Python binding) never calls it and shares no code with it.

Everything is plain numpy in float64.  Matrix products use numpy's matmul as
a library primitive; nothing is blocked, fused or reordered beyond the
definitions below.  Where the GPU stores an activation in bf16, the oracle
rounds the exact fp64 value to bf16 at the same point (``bf16_round``), so
that "bf16 model" means the same thing on both sides; all other arithmetic
(norm factors, RoPE angles, softmax, accumulations) stays in fp64.

Sources (page titles as they appear on the pages):
  [FDV]  Fast-dVLM technical overview (ocdem.com news article)
  [FDVW] Fast-dVLM walkthrough (itsolotime.com archive 34466)
  [LOWN] Look Only When Needed: Certificate-Guided Visual Routing for
         Efficient Diffusion VLMs
  [DAVET] DAVET PaperDaily article (generic dVLM commit rule only)

Readings taken where the pages are silent or garbled (each is listed with
its reason in the repository's design notes):
  shift=1   masked position j is scored by the hidden row of position j-1
            (row -1 = the last committed row); shift=0 is kept as an option.
  ar_seed   the block's first token is the AR prediction, committed outright.
  N2C       noisy tokens see the clean tokens of PRECEDING blocks only (the
            prose); the printed lower-triangular N2C matrix is not used.
  commit    p1 >= threshold; if none passes, the masked position with the
            highest p1 (lowest position on ties) is committed.
  argmax    lowest vocabulary id among equal maxima.
  top-k     (next step) the k most confident masked positions per iteration,
            lower position first on ties.
  paged     (next step) slot s of a sequence lives in row s mod P of page
            table[s div P]; a batch is the per-sequence definition per entry.
  fp8       (next step, not on the bf16 path) W8A8 in E4M3, finite variant,
            round to nearest even, saturating at 448; one scale per weight
            output channel and per activation token (amax / 448);
            SmoothQuant factors with alpha = 0.5.  The fp8 model (next
            step) runs the four projections of every layer W8A8 and keeps
            the LM head, norms, RoPE, attention and storage points as in
            the bf16 model.
  norms     RMSNorm gain 1, eps 1e-6, no biases; RoPE rotate-half, base 1e4.
  lown      (next step) TEXT-ONLY = the vision cache slots hidden from the
            block's queries, position ids unchanged; each block opens with a
            FULL pass unmasking min(k, masked) by confidence; the certified
            prefix is unmasked with the anchor ids; the FULL branch puts
            divergent positions first, each group by FULL confidence.
  quadratic (next step) one fused forward = the draft's causal verify rows
            plus one all-[MASK] candidate block per possible accepted length
            k, at positions L+k.., seeing the context and verify rows 0..k-1;
            the next draft = [verifier's token] + the chosen candidate's top-1.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against brute force, closed forms, library routines or the pages' printed
mask example.  Parity unpinned: none.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np

NEG_INF = -np.inf


# ----------------------------------------------------------------------------
# Storage rounding
# ----------------------------------------------------------------------------
def bf16_round(x) -> np.ndarray:
    """Round real values to the nearest bfloat16 (8 significant bits, ties to
    even), returned as float64.  Direct from the exact value: no detour
    through fp32 (which could double-round)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                    # x = m * 2**e, 0.5 <= |m| < 1
    r = np.round(m * 256.0)               # numpy rounds half to even
    return np.ldexp(r, e - 8)


# ----------------------------------------------------------------------------
# FP8 W8A8 linear layer (next step of the weight stream; not on the bf16 path)
# ----------------------------------------------------------------------------
# [FDV §2.3.2] names SmoothQuant W8A8 FP8 as the final serving step.  The pages
# give no formats or granularity; readings taken: E4M3 (finite variant) for
# both operands, one scale per weight output channel and per activation token
# (amax / 448), round to nearest even, SmoothQuant factors with alpha = 0.5.
E4M3_MAX = 448.0


def e4m3_round(x) -> np.ndarray:
    """Round real values to FP8 E4M3 (4 exponent bits with bias 7, 3 mantissa
    bits, subnormals down to 2^-9, largest finite 448), ties to even, returned
    as float64.  Magnitudes beyond 448 saturate to 448 (the per-row scales
    below keep every quantised value within range)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    _, e = np.frexp(a)                     # leading bit of a is 2^(e-1)
    e = np.maximum(e, -5)                  # below 2^-6: the subnormal spacing 2^-9
    q = np.ldexp(1.0, e - 4)               # 3 mantissa bits below the leading bit
    r = np.round(a / q) * q                # numpy rounds half to even
    return np.sign(x) * np.minimum(r, E4M3_MAX)


def fp8_quantize_rows(A: np.ndarray):
    """Per-row FP8 quantisation: scale s_r = max_k |A[r, k]| / 448 (1 for an
    all-zero row) and codes A_q = e4m3(A / s_r); A ~ s_r * A_q.  Rows are
    output channels for weights [out, in] and tokens for activations."""
    A = np.asarray(A, dtype=np.float64)
    amax = np.max(np.abs(A), axis=1)
    s = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    return e4m3_round(A / s[:, None]), s


def fp8_linear(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """W8A8 product y[t, o] = a_t * s_o * sum_k xq[t, k] Wq[o, k] of per-token
    quantised activations and per-output-channel quantised weights; the
    products of two E4M3 values and their sums are exact in float64 for the
    layer sizes here (every term is a multiple of 2^-18 below 2^18)."""
    xq, a = fp8_quantize_rows(x)
    wq, s = fp8_quantize_rows(W)
    return (xq @ wq.T) * a[:, None] * s[None, :]


def smooth_factors(x_amax: np.ndarray, w_amax: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """SmoothQuant factor per input channel k: m_k = x_amax_k^alpha /
    w_amax_k^(1 - alpha).  The layer then quantises x / m and W * m (per input
    channel), whose product equals x W^T before quantisation."""
    return np.power(np.asarray(x_amax, dtype=np.float64), alpha) / np.power(np.asarray(w_amax, dtype=np.float64),
                                                                            1.0 - alpha)


# ----------------------------------------------------------------------------
# Decoder-layer pieces (plain definitions)
# ----------------------------------------------------------------------------
def rms_factor(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """1 / sqrt(mean(x^2) + eps) per row (RMSNorm with unit gain)."""
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rmsnorm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm with unit gain: x / sqrt(mean(x^2) + eps)."""
    return np.asarray(x, dtype=np.float64) * rms_factor(x, eps)


def rope(x: np.ndarray, pos: Sequence[int], base: float = 10000.0) -> np.ndarray:
    """Rotate-half rotary embedding.

    x: [n, heads, D]; pos: [n] absolute positions.  For i < D/2 the pair
    (x_i, x_{i+D/2}) is rotated by theta_i = pos * base**(-2i/D)."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    half = D // 2
    inv = base ** (-2.0 * np.arange(half, dtype=np.float64) / D)
    theta = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]   # [n, half]
    c = np.cos(theta)[:, None, :]
    s = np.sin(theta)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


# ----------------------------------------------------------------------------
# Attention masks and attention  [FDV §2.2.1 masks; FDVW §4.1]
# ----------------------------------------------------------------------------
def mask_from_roles(q_noisy: Sequence[bool], q_block: Sequence[int], q_pos: Sequence[int],
                    k_noisy: Sequence[bool], k_block: Sequence[int], k_pos: Sequence[int]) -> np.ndarray:
    """Dense 0/1 visibility matrix from token roles (the three rules).

    N2N: a noisy query sees the noisy keys of its own block (bidirectional).
    N2C: a noisy query sees the clean keys of strictly preceding blocks.
    C2C: a clean query sees clean keys at positions <= its own (causal).
    A clean query never sees a noisy key."""
    nq, nk = len(q_noisy), len(k_noisy)
    m = np.zeros((nq, nk), dtype=np.int64)
    for i in range(nq):
        for j in range(nk):
            if q_noisy[i] and k_noisy[j]:
                m[i, j] = int(q_block[i] == k_block[j])
            elif q_noisy[i] and not k_noisy[j]:
                m[i, j] = int(k_block[j] < q_block[i])
            elif not q_noisy[i] and not k_noisy[j]:
                m[i, j] = int(k_pos[j] <= q_pos[i])
    return m


def dense_masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray,
                           scale: float) -> np.ndarray:
    """Brute force: q [nq, Hq, D], k/v [nk, Hkv, D], mask [nq, nk]; GQA group
    Hq/Hkv.  Explicit masked softmax per (query, head)."""
    nq, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = np.zeros((nq, Hq, D))
    for i in range(nq):
        vis = np.nonzero(mask[i])[0]
        for h in range(Hq):
            g = h // G
            s = np.array([scale * float(np.dot(q[i, h], k[j, g])) for j in vis])
            p = np.exp(s - s.max())
            p = p / p.sum()
            out[i, h] = sum(p[t] * v[vis[t], g] for t in range(len(vis)))
    return out


def block_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, L: int, n_clean: int,
                    scale: float, hide: int = 0) -> np.ndarray:
    """Attention of one step's rows against the KV cache.

    q: [n, Hq, D] for rows at cache slots L .. L+n-1 (their K/V already in the
    cache).  K, V: [Hkv, >= L+n, D].  Rows 0..n_clean-1 are clean (causal:
    row t sees slots 0..L+t); the remaining rows form the noisy block and see
    every slot 0..L+n-1 (the whole cache through N2C plus the whole block
    through N2N).  ``hide``: slots 0..hide-1 are invisible to every row (the
    TEXT-ONLY pass of certificate routing drops the vision tokens, which sit
    at the front of the cache; positions are unchanged) [LOWN method step (2)]."""
    q = np.asarray(q, dtype=np.float64)
    n, Hq, D = q.shape
    Hkv = K.shape[0]
    G = Hq // Hkv
    out = np.zeros((n, Hq, D))
    for t in range(n):
        vis = (L + t + 1) if t < n_clean else (L + n)
        for h in range(Hq):
            g = h // G
            s = scale * (K[g, hide:vis] @ q[t, h])
            p = np.exp(s - s.max())
            p /= p.sum()
            out[t, h] = p @ V[g, hide:vis]
    return out


def paged_gather(pages: np.ndarray, block_table: Sequence[int], n: int) -> np.ndarray:
    """Logical cache slots 0..n-1 of one sequence from a paged store [FDV
    §2.3.2, paged KV cache management].  pages: [n_pages, Hkv, P, D]; logical
    slot s lives in row s mod P of page block_table[s div P].  Returns
    [Hkv, n, D] in logical order."""
    P = pages.shape[2]
    out = np.zeros((pages.shape[1], n, pages.shape[3]))
    for s in range(n):
        out[:, s] = pages[block_table[s // P], :, s % P]
    return out


def paged_block_attention(q: np.ndarray, K_pages: np.ndarray, V_pages: np.ndarray, block_table: Sequence[int],
                          L: int, n_clean: int, scale: float, hide: int = 0) -> np.ndarray:
    """block_attention over a paged cache: the step's rows sit at logical
    slots L..L+n-1 (their K/V already stored through the same table)."""
    n = q.shape[0]
    K = paged_gather(K_pages, block_table, L + n)
    V = paged_gather(V_pages, block_table, L + n)
    return block_attention(q, K, V, L, n_clean, scale, hide)


# ----------------------------------------------------------------------------
# Confidence, commit, certificate, accept
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class Conf:
    p1: np.ndarray     # top-1 probability per row
    top1: np.ndarray   # lowest id attaining the max logit
    p2: np.ndarray     # second-largest probability (margin checks)
    top2: Optional[np.ndarray] = None   # the runner-up id: lowest id attaining the max
                                        # logit once top1 is set aside (near-tie checks)


def confidence_from_logits(logits: np.ndarray) -> Conf:
    """Top-1 confidence = max softmax probability over the vocabulary
    [LOWN method step (1): s = max_w p(y_i = w | ...)], argmax = lowest id."""
    lg = np.asarray(logits, dtype=np.float64)
    m = lg.max(axis=-1, keepdims=True)
    e = np.exp(lg - m)
    s = e.sum(axis=-1)
    p1 = 1.0 / s
    top1 = np.argmax(lg, axis=-1).astype(np.int64)      # first maximum
    part = np.partition(lg, -2, axis=-1)[..., -2]
    p2 = np.exp(part - m[..., 0]) / s
    rest = lg.copy()
    np.put_along_axis(rest, top1[..., None], -np.inf, axis=-1)
    top2 = np.argmax(rest, axis=-1).astype(np.int64)
    return Conf(p1=p1, top1=top1, p2=p2, top2=top2)


def lm_head_conf(hidden: np.ndarray, W: np.ndarray, row_scale: Optional[np.ndarray] = None) -> Conf:
    """logits = row_scale * (hidden @ W^T) (row_scale = final RMSNorm factor or 1)."""
    lg = np.asarray(hidden, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T
    if row_scale is not None:
        lg = lg * np.asarray(row_scale, dtype=np.float64).reshape(-1, 1)
    return confidence_from_logits(lg)


def threshold_commit(p1: Sequence[float], masked: Sequence[bool], tau: float) -> List[int]:
    """Commit every masked row with p1 >= tau; when none passes, commit the
    masked row with the highest p1 (lowest index on ties).
    [FDV §4.1 threshold 0.9; DAVET generic commit rule]"""
    R = len(p1)
    C = [r for r in range(R) if masked[r] and p1[r] >= tau]
    if not C:
        best = None
        for r in range(R):
            if masked[r] and (best is None or p1[r] > p1[best]):
                best = r
        if best is not None:
            C = [best]
    return C


def topk_commit(p1: Sequence[float], masked: Sequence[bool], k: int) -> List[int]:
    """Commit the k masked rows of highest p1 (all of them when fewer remain),
    lower index first on ties: the confidence-ordered unmasking of a fixed
    number of positions per step [LOWN, background on confidence-guided
    unmasking]."""
    idx = [r for r in range(len(p1)) if masked[r]]
    idx.sort(key=lambda r: (-float(p1[r]), r))
    return sorted(idx[:max(k, 0)])


def certificate_scan(anchor_id: Sequence[int], anchor_conf: Sequence[float],
                     top1: Sequence[int], participants: Optional[Sequence[bool]] = None) -> int:
    """Longest certified prefix [LOWN method step (2)]: visit positions in
    descending anchor confidence (lower index first on ties) and stop at the
    first whose new top-1 differs from its anchor; return the count before it."""
    R = len(anchor_id)
    idx = [i for i in range(R) if participants is None or participants[i]]
    idx.sort(key=lambda i: (-float(anchor_conf[i]), i))
    n = 0
    for i in idx:
        if int(top1[i]) != int(anchor_id[i]):
            break
        n += 1
    return n


def certificate_order(anchor_conf: Sequence[float], participants: Sequence[bool]) -> List[int]:
    """Positions in the order the certificate scan visits them: descending
    anchor confidence, lower index first on ties [LOWN method step (2)]."""
    idx = [i for i in range(len(anchor_conf)) if participants[i]]
    idx.sort(key=lambda i: (-float(anchor_conf[i]), i))
    return idx


def divergence_first_order(full_top1: Sequence[int], full_conf: Sequence[float], text_top1: Sequence[int],
                           participants: Sequence[bool]) -> List[int]:
    """Unmasking order of the FULL branch [LOWN method step (3)]: positions
    whose TEXT-ONLY and FULL top-1 differ first, then the others; each group
    by descending FULL confidence, lower index first on ties."""
    idx = [i for i in range(len(full_top1)) if participants[i]]
    idx.sort(key=lambda i: (int(text_top1[i]) == int(full_top1[i]), -float(full_conf[i]), i))
    return idx


def prefix_accept(verify_ids: Sequence[int], draft_ids: Sequence[int]) -> int:
    """Longest prefix on which the causal pass's argmax equals the draft
    [FDV §2.3.1 longest-prefix acceptance]."""
    k = 0
    for a, b in zip(verify_ids, draft_ids):
        if int(a) != int(b):
            break
        k += 1
    return k


# ----------------------------------------------------------------------------
# Model
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class Dims:
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    inter: int
    vocab: int
    rope_base: float = 10000.0
    eps: float = 1e-6

    @property
    def mask_id(self) -> int:
        return self.vocab - 1


class OracleModel:
    """The decoder as plain definitions.

    weights: dict with "embed" [V,H], "lm_head" [V,H] and per layer l the
    matrices "l.wq", "l.wk", "l.wv", "l.wo", "l.wg", "l.wu", "l.wd" ([out,in]).
    A callable ``weights_fn(name)`` may be given instead, to regenerate big
    matrices on demand.  ``bf16``: round activations at the GPU's storage
    points (q/k/v after RoPE, attention output, residual stream, SwiGLU
    activation)."""

    def __init__(self, dims: Dims, weights=None, weights_fn=None, bf16: bool = True,
                 Lmax: int = 4096, fp8: bool = False, smooth: Optional[Dict[str, np.ndarray]] = None):
        self.d = dims
        self._w = weights
        self._wfn = weights_fn
        self.bf16 = bf16
        self.Lmax = Lmax
        # W8A8 decoder projections (next step of the weight stream): the four
        # projections of every layer go through fp8_linear on the activations
        # they consume; the LM head, norms, RoPE, attention and the bf16
        # storage points stay as in the bf16 model.  `smooth` maps a weight
        # name to its SmoothQuant factors m (x / m and W * m are quantised).
        self.fp8 = fp8
        self.smooth = smooth or {}
        self.K = [np.zeros((dims.n_kv_heads, Lmax, dims.head_dim)) for _ in range(dims.n_layers)]
        self.V = [np.zeros((dims.n_kv_heads, Lmax, dims.head_dim)) for _ in range(dims.n_layers)]
        self.L = 0

    def w(self, name: str) -> np.ndarray:
        if self._w is not None and name in self._w:
            return self._w[name]
        return np.asarray(self._wfn(name), dtype=np.float64)

    def rnd(self, x: np.ndarray) -> np.ndarray:
        return bf16_round(x) if self.bf16 else x

    def lin(self, a: np.ndarray, name: str) -> np.ndarray:
        """a W^T for the decoder matrix `name` ([out, in]); W8A8 in fp8 mode."""
        W = self.w(name)
        if not self.fp8:
            return a @ W.T
        m = self.smooth.get(name)
        if m is not None:
            return fp8_linear(a / m[None, :], W * m[None, :])
        return fp8_linear(a, W)

    # -- one decoder layer ---------------------------------------------------
    def layer(self, l: int, x: np.ndarray, L: int, n_clean: int, write_kv: bool = True, hide: int = 0) -> np.ndarray:
        d = self.d
        n = x.shape[0]
        D, Hq, Hkv = d.head_dim, d.n_q_heads, d.n_kv_heads
        pos = np.arange(L, L + n)
        h = x * rms_factor(x, d.eps)
        q = self.lin(h, f"{l}.wq").reshape(n, Hq, D)
        k = self.lin(h, f"{l}.wk").reshape(n, Hkv, D)
        v = self.lin(h, f"{l}.wv").reshape(n, Hkv, D)
        q = self.rnd(rope(q, pos, d.rope_base))
        k = self.rnd(rope(k, pos, d.rope_base))
        v = self.rnd(v)
        if write_kv:
            self.K[l][:, L:L + n] = k.transpose(1, 0, 2)
            self.V[l][:, L:L + n] = v.transpose(1, 0, 2)
        a = block_attention(q, self.K[l], self.V[l], L, n_clean, 1.0 / math.sqrt(D), hide)
        a = self.rnd(a).reshape(n, Hq * D)
        x = self.rnd(x + self.lin(a, f"{l}.wo"))
        h2 = x * rms_factor(x, d.eps)
        g = self.lin(h2, f"{l}.wg")
        u = self.lin(h2, f"{l}.wu")
        act = self.rnd(silu(g) * u)
        x = self.rnd(x + self.lin(act, f"{l}.wd"))
        return x

    def embed(self, ids: Sequence[int]) -> np.ndarray:
        E = self.w("embed")
        return np.asarray(E[np.asarray(ids, dtype=np.int64)], dtype=np.float64)

    def forward(self, x: np.ndarray, L: int, n_clean: int, hide: int = 0) -> np.ndarray:
        """Run all layers over rows at slots L..L+n-1; returns the final
        residual stream (before the final norm).  K/V of these rows are
        written to the cache; the cache length is NOT advanced here.  ``hide``:
        cache slots 0..hide-1 are invisible (TEXT-ONLY pass, see
        block_attention)."""
        for l in range(self.d.n_layers):
            x = self.layer(l, x, L, n_clean, hide=hide)
        return x

    def logits_conf(self, x: np.ndarray) -> Conf:
        """Final RMSNorm + LM head + confidence."""
        return lm_head_conf(x, self.w("lm_head"), rms_factor(x, self.d.eps)[:, 0])


# ----------------------------------------------------------------------------
# Decode drivers
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class DecodeTrace:
    tokens: List[int]
    nfe: int = 0
    commits_per_iter: List[int] = dataclasses.field(default_factory=list)
    accept_lens: List[int] = dataclasses.field(default_factory=list)
    drafts: List[List[int]] = dataclasses.field(default_factory=list)   # speculative drafts, per round
    # smallest decision margin met along the trajectory (for parity exclusion)
    min_margin: float = math.inf
    margins: List[float] = dataclasses.field(default_factory=list)


def prefill(model: OracleModel, vision: Optional[np.ndarray], ids: Sequence[int]) -> int:
    """Causal pass over [vision rows | text ids]; returns the AR seed token
    (argmax of the LM head at the last context row) and sets model.L."""
    rows = []
    if vision is not None and len(vision):
        rows.append(np.asarray(vision, dtype=np.float64))
    if len(ids):
        rows.append(model.embed(ids))
    x = np.concatenate(rows, axis=0)
    n = x.shape[0]
    xo = model.forward(x, 0, n_clean=n)
    model.L = n
    c = model.logits_conf(xo[-1:])
    model.last_conf = c
    return int(c.top1[0])


def _note_argmax_margin(tr: DecodeTrace, c: Conf, rows) -> None:
    for r in rows:
        m = float(c.p1[r] - c.p2[r])
        tr.margins.append(m)
        tr.min_margin = min(tr.min_margin, m)


def decode_threshold(model: OracleModel, seed_token: int, B: int, tau: float, max_new: int,
                     shift: int = 1, ar_seed: int = 1, on_iter=None, on_block=None,
                     commit_k: Optional[int] = None) -> DecodeTrace:
    """Threshold (MDM-style) block decoding [FDV §2.2.1, §2.2.2, §4.1].

    Per block: the first token is the AR seed (ar_seed=1); the remaining
    positions start as [MASK].  Each iteration runs the whole block as noisy
    rows over the cache (its K/V go to slots L..L+B-1 without advancing L),
    scores the still-masked positions (position j from row j-shift; row -1 is
    the previous pass's last row) and commits per ``threshold_commit``.  When
    the block is complete a causal pass over it makes its K/V final, advances
    L by B and yields the next block's seed from its last row.

    ``commit_k``: commit per ``topk_commit`` (the k most confident masked
    positions each iteration) instead of the threshold rule; tau is unused.

    Optional observers (they do not change the trajectory): on_iter(L, toks,
    masked, p1, top1, p2) before each iteration's commit, with the scores per
    block position; on_block(L, toks) before each block's causal pass."""
    d = model.d
    tr = DecodeTrace(tokens=[])
    seed = seed_token
    prev_conf = model.last_conf
    while len(tr.tokens) < max_new:
        L = model.L
        toks = [d.mask_id] * B
        masked = [True] * B
        if ar_seed:
            toks[0] = seed
            masked[0] = False
        while any(masked):
            x = model.forward(model.embed(toks), L, n_clean=0)
            c = model.logits_conf(x)
            p1 = np.zeros(B)
            top = np.zeros(B, dtype=np.int64)
            p2 = np.zeros(B)
            for j in range(B):
                r = j - shift
                cc, rr = (prev_conf, 0) if r < 0 else (c, r)
                p1[j], top[j], p2[j] = cc.p1[rr], cc.top1[rr], cc.p2[rr]
            if on_iter is not None:
                on_iter(L, list(toks), list(masked), p1.copy(), top.copy(), p2.copy())
            if commit_k is not None:
                C = topk_commit(p1, masked, commit_k)
                rest = [p1[j] for j in range(B) if masked[j] and j not in C]
                margins = [p1[j] - p2[j] for j in C]
                if rest:
                    margins.append(min(p1[j] for j in C) - max(rest))
                for mg in margins:
                    tr.margins.append(float(mg))
                    tr.min_margin = min(tr.min_margin, float(mg))
            else:
                C = threshold_commit(p1, masked, tau)
            for j in range(B):
                if commit_k is None and masked[j]:
                    mg = min(abs(p1[j] - tau), p1[j] - p2[j])
                    tr.margins.append(mg)
                    tr.min_margin = min(tr.min_margin, mg)
            if commit_k is None and len(C) == 1 and not (p1[C[0]] >= tau):
                others = [p1[j] for j in range(B) if masked[j] and j != C[0]]
                if others:
                    mg = float(p1[C[0]] - max(others))
                    tr.margins.append(mg)
                    tr.min_margin = min(tr.min_margin, mg)
            for j in C:
                toks[j] = int(top[j])
                masked[j] = False
            tr.commits_per_iter.append(len(C))
            tr.nfe += 1
        if on_block is not None:
            on_block(L, list(toks))
        x = model.forward(model.embed(toks), L, n_clean=B)
        model.L = L + B
        c = model.logits_conf(x)
        tr.nfe += 1
        _note_argmax_margin(tr, c, [B - 1])
        prev_conf = Conf(p1=c.p1[B - 1:], top1=c.top1[B - 1:], p2=c.p2[B - 1:],
                         top2=None if c.top2 is None else c.top2[B - 1:])
        seed = int(c.top1[B - 1])
        tr.tokens.extend(toks)
    tr.tokens = tr.tokens[:max_new]
    return tr


def decode_spec_linear(model: OracleModel, seed_token: int, B: int, max_new: int, on_round=None) -> DecodeTrace:
    """Linear self-speculative decoding [FDV §2.3.1]: a diffusion draft pass
    (every position takes its argmax), then a causal verify pass over the
    draft; the longest prefix on which the verifier agrees is kept (position
    0, the AR seed, always), L advances by its length and the verifier's
    prediction right after it seeds the next round (shift=1).

    Optional observer (it does not change the trajectory): on_round(L,
    draft_input, draft_conf, draft, verify_conf, k, next_seed) after each
    round, with the draft pass's input tokens and the per-row confidences of
    both passes (row r scores position r + 1)."""
    d = model.d
    tr = DecodeTrace(tokens=[])
    seed = seed_token
    while len(tr.tokens) < max_new:
        L = model.L
        toks = [seed] + [d.mask_id] * (B - 1)
        x = model.forward(model.embed(toks), L, n_clean=0)
        c = model.logits_conf(x)
        _note_argmax_margin(tr, c, range(B - 1))
        draft = [seed] + [int(c.top1[j - 1]) for j in range(1, B)]
        tr.nfe += 1
        x = model.forward(model.embed(draft), L, n_clean=B)
        g = model.logits_conf(x)
        _note_argmax_margin(tr, g, range(B))
        tr.nfe += 1
        verify = [seed] + [int(g.top1[j - 1]) for j in range(1, B)]
        k = prefix_accept(verify, draft)
        tr.accept_lens.append(k)
        tr.tokens.extend(draft[:k])
        model.L = L + k
        seed = int(g.top1[k - 1])
        if on_round is not None:
            on_round(L, list(toks), c, list(draft), g, k, seed)
    tr.tokens = tr.tokens[:max_new]
    return tr


def decode_ar(model: OracleModel, seed_token: int, max_new: int) -> DecodeTrace:
    """Greedy autoregressive decoding, one token per forward (comparator)."""
    tr = DecodeTrace(tokens=[])
    seed = seed_token
    while len(tr.tokens) < max_new:
        L = model.L
        x = model.forward(model.embed([seed]), L, n_clean=1)
        model.L = L + 1
        c = model.logits_conf(x)
        _note_argmax_margin(tr, c, [0])
        tr.nfe += 1
        tr.tokens.append(seed)
        seed = int(c.top1[0])
    return tr


# ----------------------------------------------------------------------------
# Quadratic self-speculative decoding  [FDV §2.3.1, the variant that fuses
# draft and verify into one forward at O(B^2) cost]
# ----------------------------------------------------------------------------
def quadratic_attention(q_ver: np.ndarray, q_cand: np.ndarray, K: np.ndarray, V: np.ndarray, L: int,
                        k_cand: np.ndarray, v_cand: np.ndarray, scale: float) -> np.ndarray:
    """Attention of one fused forward.

    q_ver [B, Hq, D]: the causal verify rows of the draft at slots L..L+B-1,
    whose K/V are already in the cache K, V [Hkv, >= L+B, D]; row t sees
    slots 0..L+t.  q_cand [B, B, Hq, D]: candidate block i (0-based; it
    stands for "the first i+1 draft tokens accepted") holds B noisy rows at
    positions L+i+1 .. L+i+B; its K/V k_cand, v_cand [B, B, Hkv, D] stay out
    of the cache.  A candidate row sees the cache slots 0..L+i (the context
    and the accepted verify rows, N2C) and the B rows of its own candidate
    block (N2N), nothing of the other candidates.  Returns [B + B*B, Hq, D]:
    verify rows, then the candidate blocks in order."""
    B, Hq, D = q_ver.shape
    Hkv = K.shape[0]
    G = Hq // Hkv
    out = [block_attention(q_ver, K, V, L, B, scale)]
    for i in range(B):
        o = np.zeros((B, Hq, D))
        for r in range(B):
            for h in range(Hq):
                g = h // G
                keys = np.concatenate([K[g, :L + i + 1], k_cand[i, :, g]], axis=0)
                vals = np.concatenate([V[g, :L + i + 1], v_cand[i, :, g]], axis=0)
                sc = scale * (keys @ q_cand[i, r, h])
                p = np.exp(sc - sc.max())
                p /= p.sum()
                o[r, h] = p @ vals
        out.append(o)
    return np.concatenate(out, axis=0)


def forward_quadratic(model: OracleModel, draft: Sequence[int], L: int) -> np.ndarray:
    """One fused draft+verify forward over B + B*B rows: the draft's verify
    rows (clean, causal, K/V written to slots L..L+B-1) and B candidate blocks
    of B [MASK] rows each (candidate i at positions L+i+1 .. L+i+B, K/V kept
    out of the cache).  Same layer arithmetic and bf16 storage points as
    OracleModel.layer.  Returns the final residual rows [B + B*B, H]."""
    d = model.d
    B = len(draft)
    D, Hq, Hkv = d.head_dim, d.n_q_heads, d.n_kv_heads
    x = np.concatenate([model.embed(draft), model.embed([d.mask_id] * (B * B))], axis=0)
    pos = np.concatenate([np.arange(L, L + B)] + [np.arange(L + i + 1, L + i + 1 + B) for i in range(B)])
    n = x.shape[0]
    for l in range(d.n_layers):
        h = x * rms_factor(x, d.eps)
        q = model.lin(h, f"{l}.wq").reshape(n, Hq, D)
        k = model.lin(h, f"{l}.wk").reshape(n, Hkv, D)
        v = model.lin(h, f"{l}.wv").reshape(n, Hkv, D)
        q = model.rnd(rope(q, pos, d.rope_base))
        k = model.rnd(rope(k, pos, d.rope_base))
        v = model.rnd(v)
        model.K[l][:, L:L + B] = k[:B].transpose(1, 0, 2)
        model.V[l][:, L:L + B] = v[:B].transpose(1, 0, 2)
        a = quadratic_attention(q[:B], q[B:].reshape(B, B, Hq, D), model.K[l], model.V[l], L,
                                k[B:].reshape(B, B, Hkv, D), v[B:].reshape(B, B, Hkv, D),
                                1.0 / math.sqrt(D))
        a = model.rnd(a).reshape(n, Hq * D)
        x = model.rnd(x + model.lin(a, f"{l}.wo"))
        h2 = x * rms_factor(x, d.eps)
        g = model.lin(h2, f"{l}.wg")
        u = model.lin(h2, f"{l}.wu")
        act = model.rnd(silu(g) * u)
        x = model.rnd(x + model.lin(act, f"{l}.wd"))
    return x


def decode_spec_quadratic(model: OracleModel, seed_token: int, B: int, max_new: int) -> DecodeTrace:
    """Quadratic self-speculative decoding [FDV §2.3.1].  The first draft
    comes from one diffusion pass as in the linear variant.  Every later
    forward is fused: it verifies the current draft causally (v_j = top-1 of
    verify row j-1, v_0 = the seed) and, for every possible accepted length
    k = 1..B, drafts the next block in candidate block k-1, whose rows sit at
    positions L+k .. L+k+B-1.  After the longest agreeing prefix k is kept
    (L advances by k), the next draft is [v_k] followed by the top-1 of
    candidate block k-1's rows 0..B-2 (shift=1: a row scores the position
    after it).  One forward per round instead of two; the output equals
    greedy AR decoding, since only verified tokens are kept."""
    d = model.d
    tr = DecodeTrace(tokens=[])
    L = model.L
    x = model.forward(model.embed([seed_token] + [d.mask_id] * (B - 1)), L, n_clean=0)
    c = model.logits_conf(x)
    _note_argmax_margin(tr, c, range(B - 1))
    draft = [seed_token] + [int(c.top1[j - 1]) for j in range(1, B)]
    tr.nfe += 1
    while len(tr.tokens) < max_new:
        L = model.L
        tr.drafts.append(list(draft))
        x = forward_quadratic(model, draft, L)
        c = model.logits_conf(x)
        tr.nfe += 1
        _note_argmax_margin(tr, c, range(B))
        verify = [draft[0]] + [int(c.top1[j - 1]) for j in range(1, B)]
        k = prefix_accept(verify, draft)
        tr.accept_lens.append(k)
        tr.tokens.extend(draft[:k])
        model.L = L + k
        rows = B + (k - 1) * B
        _note_argmax_margin(tr, c, range(rows, rows + B - 1))
        draft = [int(c.top1[k - 1])] + [int(c.top1[rows + j - 1]) for j in range(1, B)]
    tr.tokens = tr.tokens[:max_new]
    return tr


# ----------------------------------------------------------------------------
# Certificate-guided visual routing inside block decoding  [LOWN method
# steps (1)-(3)]
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class LownTrace:
    tokens: List[int]
    n_full: int = 0          # FULL noisy forwards (vision visible)
    n_text: int = 0          # TEXT-ONLY noisy forwards (vision hidden)
    n_causal: int = 0        # causal append passes
    accepted: List[int] = dataclasses.field(default_factory=list)   # positions unmasked per step
    text_branch: List[bool] = dataclasses.field(default_factory=list)


def decode_lown(model: OracleModel, seed_token: int, B: int, k: int, n_vis: int, max_new: int,
                shift: int = 1, on_pass=None, on_block=None) -> LownTrace:
    """Certificate-guided visual routing [LOWN method steps (1)-(3)] inside
    block decoding.  Per block (first token = the AR seed, the rest [MASK]):
    a FULL noisy forward sets the anchors (top-1 id and confidence of every
    masked position, position j scored by row j - shift) and unmasks the k
    most confident positions.  Each later step runs a TEXT-ONLY noisy forward
    (cache slots 0..n_vis-1, the vision rows, hidden; positions unchanged) and
    scans the masked positions in descending anchor confidence while the
    TEXT-ONLY top-1 equals the anchor: if that certified prefix holds at least
    min(k, masked) positions, all of it is unmasked with the anchor ids;
    otherwise a FULL forward refreshes the anchors and min(k, masked)
    positions are unmasked with the FULL ids, divergent positions (TEXT-ONLY
    top-1 != FULL top-1) first.  A causal pass then appends the block.

    Optional observers (they do not change the trajectory): on_pass(kind, L,
    toks, p1, top1) after each noisy pass ("full" or "text"), with the block
    tokens it ran on and its scores per block position; on_block(L, toks)
    before each block's causal pass."""
    d = model.d
    tr = LownTrace(tokens=[])
    seed = seed_token
    prev_conf = model.last_conf

    def scores(c, pc):
        p1, top = np.zeros(B), np.zeros(B, dtype=np.int64)
        for j in range(B):
            r = j - shift
            cc, rr = (pc, 0) if r < 0 else (c, r)
            p1[j], top[j] = cc.p1[rr], cc.top1[rr]
        return p1, top

    while len(tr.tokens) < max_new:
        L = model.L
        toks = [d.mask_id] * B
        masked = [True] * B
        toks[0], masked[0] = seed, False
        anchor_id, anchor_conf = None, None
        text_top = None
        while any(masked):
            kk = min(k, sum(masked))
            if anchor_id is not None:
                x = model.forward(model.embed(toks), L, n_clean=0, hide=n_vis)
                text_p1, text_top = scores(model.logits_conf(x), prev_conf)
                tr.n_text += 1
                if on_pass is not None:
                    on_pass("text", L, list(toks), text_p1.copy(), text_top.copy())
                order = certificate_order(anchor_conf, masked)
                n = certificate_scan(anchor_id, anchor_conf, text_top, masked)
                if n >= kk:
                    for j in order[:n]:
                        toks[j], masked[j] = int(anchor_id[j]), False
                    tr.accepted.append(n)
                    tr.text_branch.append(True)
                    continue
            x = model.forward(model.embed(toks), L, n_clean=0)
            full_p1, full_top = scores(model.logits_conf(x), prev_conf)
            tr.n_full += 1
            if on_pass is not None:
                on_pass("full", L, list(toks), full_p1.copy(), full_top.copy())
            anchor_id, anchor_conf = full_top.copy(), full_p1.copy()
            if text_top is None:
                order = certificate_order(full_p1, masked)
            else:
                order = divergence_first_order(full_top, full_p1, text_top, masked)
            for j in order[:kk]:
                toks[j], masked[j] = int(full_top[j]), False
            tr.accepted.append(kk)
            tr.text_branch.append(False)
        if on_block is not None:
            on_block(L, list(toks))
        x = model.forward(model.embed(toks), L, n_clean=B)
        model.L = L + B
        c = model.logits_conf(x)
        tr.n_causal += 1
        prev_conf = Conf(p1=c.p1[B - 1:], top1=c.top1[B - 1:], p2=c.p2[B - 1:],
                         top2=None if c.top2 is None else c.top2[B - 1:])
        seed = int(c.top1[B - 1])
        take = min(B, max_new - len(tr.tokens))
        tr.tokens.extend(toks[:take])
    return tr


# ----------------------------------------------------------------------------
# Weight helpers for tests and the CPU baseline (the generator draws values;
# here they are only arranged under the names the oracle uses)
# ----------------------------------------------------------------------------
def weights_from_generator(gen, dims, seed: int) -> Dict[str, np.ndarray]:
    """Materialise every matrix of a (small) model as float64."""
    out = {"embed": np.asarray(gen.embedding_weight(dims, seed)[1], dtype=np.float64),
           "lm_head": np.asarray(gen.lm_head_weight(dims, seed)[1], dtype=np.float64)}
    for l in range(dims.n_layers):
        for nm in gen.layer_weight_names():
            out[f"{l}.{nm}"] = np.asarray(gen.layer_weight(dims, seed, l, nm)[1], dtype=np.float64)
    return out


def dims_from(gdims) -> Dims:
    return Dims(n_layers=gdims.n_layers, hidden=gdims.hidden, n_q_heads=gdims.n_q_heads,
                n_kv_heads=gdims.n_kv_heads, head_dim=gdims.head_dim, inter=gdims.inter,
                vocab=gdims.vocab, rope_base=gdims.rope_base, eps=gdims.eps)
