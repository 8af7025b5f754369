"""End-to-end block decoding through the engine's own CUDA-graph path vs the
oracle, on small models: the tiny fp32 model (first configuration: 64-token
context of 32 vision embeddings, 16 prompt and 16 committed ids, one B=4
block, threshold 0.9) and a reduced-depth bf16 model with the same per-head
shapes as the Qwen2.5-3B decoder.

Every forward the engine's decode driver runs is recorded by its trace hook
(dvlm_engine_set_trace) and replayed against the oracle, teacher-forced
(tests/decode_replay.py): the oracle runs the same forward over its own cache,
the hidden rows must agree (1e-4 fp32; 2e-2 plus one storage ulp bf16), and
every top-1 id, commit set, accepted length and seed must be bit-exact
wherever its deciding confidences are at least 1e-3 from the boundary; inside
that margin the GPU may take any of the tied choices and the oracle follows
it.

fp32: the deciding confidences are the oracle's own (GPU and oracle hidden
rows agree to ~1e-6).  bf16: a value whose fp32 and fp64 sums fall on either
side of a bf16 rounding boundary lands one storage ulp apart, and the LM head
(N(0, 0.02) x 25 weights) turns such a flip into a p1 difference of a few
1e-2, so the 1e-3 bar is applied to the oracle's LM head on the GPU's own
final hidden rows (the rows the fused LM head + commit read), and the
oracle's own rows hold the decisions to DELTA = 0.1."""
import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import dvlm_gen as gen
import oracle as O
from decode_replay import NOISY, Replay, parse_trace
from dvlm_gen.device import DeviceModel, kv_buffers
from gpu_util import assert_bf16_close, assert_ok, f64, max_abs, status, ws_tensor

pytestmark = pytest.mark.gpu
MARGIN = 1e-3
# bound on |p1(GPU) - p1(oracle)| for the bf16 reduced model on the oracle's
# own hidden rows: hidden states one storage ulp apart in a few elements move
# p1 by a few 1e-2 (GPU against oracle: up to 0.03 measured; a CPU model of
# such rounding flips: up to 0.066, tests/test_precision_model.py)
DELTA = 0.1

SMALL_BF16 = gen.ModelDims(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=1, head_dim=128, inter=1024,
                           vocab=4096, lm_scale=25.0, dtype="bf16")


class Setup:
    def __init__(self, dims, seed, cuda, n_vis, n_prompt, n_comm, Lmax=512, options=None):
        self.dims, self.seed, self.cuda = dims, seed, cuda
        self.dm = DeviceModel(dims, seed, device=cuda)
        self.kc, self.vc = kv_buffers(dims, Lmax, device=cuda)
        cm = self.dm.c_model()
        self.ws = ws_tensor(dv.engine_workspace_size(cm, Lmax, 16, 128), cuda)
        self.eng = dv.Engine(cm, self.kc, self.vc, Lmax, 16, 128, self.ws)
        for name, value in (options or {}).items():
            self.eng.set_option(name, value)
            assert self.eng.get_option(name) == value
        self.vis_t, self.vis, self.ids = gen.decode_context(dims, seed, n_vis, n_prompt, n_comm)
        self.w = O.weights_from_generator(gen, dims, seed)
        self.od = O.dims_from(dims)
        self.Lmax = Lmax

    def gpu(self, mode, B, tau, n_new, use_graphs=1):
        eng = self.eng
        vis = self.vis_t.to(self.cuda)
        ids = torch.from_numpy(self.ids).to(self.cuda)
        eng.prefill(vis, vis.shape[0], ids, len(self.ids))
        cfg = dv.DecodeCfg(B, tau, mode, 1, n_new, use_graphs)
        out = torch.zeros(n_new, dtype=torch.int32, device=self.cuda)
        st = dv.Stats()
        eng.generate(cfg, out, st)
        eng.check()
        return out.cpu().numpy().tolist(), st

    def traced(self, mode, B, tau, n_new, use_graphs=1, cap=512):
        """Decode with the engine's forward trace on: (tokens, stats, records, final L, final seed)."""
        rb = dv.engine_trace_record_bytes(self.dm.c_model())
        buf = torch.zeros(cap * rb, dtype=torch.uint8, device=self.cuda)
        cnt = torch.zeros(4, dtype=torch.int32, device=self.cuda)
        self.eng.set_trace(buf, cnt)
        try:
            tokens, st = self.gpu(mode, B, tau, n_new, use_graphs)
        finally:
            self.eng.set_trace(None, None)
        n = int(cnt[0].item())
        assert 0 < n < cap
        L, seed = self.eng.position()
        recs = parse_trace(buf.cpu().numpy(), n, rb, self.dims.hidden, self.dims.dtype == "bf16")
        return tokens, st, recs, L, seed

    def oracle_model(self):
        m = O.OracleModel(self.od, weights=self.w, bf16=self.dims.dtype == "bf16", Lmax=self.Lmax)
        s = O.prefill(m, self.vis.astype(np.float64), self.ids)
        return m, s

    def oracle(self, mode, B, tau, n_new):
        m, s = self.oracle_model()
        if mode == dv.MODE_THRESHOLD:
            return O.decode_threshold(m, s, B, tau, n_new), m
        if mode == dv.MODE_SPEC_LINEAR:
            return O.decode_spec_linear(m, s, B, n_new), m
        return O.decode_ar(m, s, n_new), m


def _fp32_hidden(a, b, what):
    assert max_abs(a, b) < 1e-4, (what, max_abs(a, b))


def _bf16_hidden(a, b, what):
    assert_bf16_close(a, b, 2e-2, what)


def replay_trace(s, mode, B, tau, n_new, tokens, st, recs, L, seed):
    """Holds a traced engine run to the oracle (teacher-forced); returns the
    replay (its tallies) and the oracle model (its cache)."""
    m, so = s.oracle_model()
    if s.dims.dtype == "bf16":
        rp = Replay(m, so, B, tau, decide="gpu", hidden_check=_bf16_hidden, secondary=DELTA, seed_bar=DELTA)
    else:
        rp = Replay(m, so, B, tau, decide="oracle", hidden_check=_fp32_hidden)
    if mode == dv.MODE_THRESHOLD:
        got = rp.threshold(recs, n_new)
    elif mode == dv.MODE_SPEC_LINEAR:
        got = rp.speculative(recs, n_new, L, seed)
    else:
        got = rp.autoregressive(recs, n_new)
    # the engine's emitted tokens are the committed blocks of its own trace,
    # and its counters count exactly these forwards
    assert got == tokens
    assert rp._next == len(recs) == st.nfe
    if mode == dv.MODE_THRESHOLD:
        per_iter = [int(np.sum(r.msk_in & ~r.msk_out)) for r in recs if r.kind == NOISY]
        hist = np.bincount(per_iter, minlength=dv.binding.HIST)[:dv.binding.HIST]
        assert list(st.commit_hist) == hist.tolist()
    return rp, m


@pytest.fixture(scope="module")
def tiny0(cuda):
    return Setup(gen.TINY, 0, cuda, 32, 16, 16, Lmax=128)


@pytest.fixture(scope="module")
def tiny4(cuda):
    return Setup(gen.TINY, 4, cuda, 32, 16, 16, Lmax=128)


def test_tiny_fp32_block_step_seed0(tiny0):
    """The tiny configuration exactly as stated: seed 0, one B=4 block,
    threshold 0.9, every decision bit-exact outside the 1e-3 margin, and the
    exact KV cache --
    the 64 prefilled context slots and the appended block -- within 1e-4."""
    tokens, st, recs, L, seed = tiny0.traced(dv.MODE_THRESHOLD, 4, 0.9, 4)
    rp, m = replay_trace(tiny0, dv.MODE_THRESHOLD, 4, 0.9, 4, tokens, st, recs, L, seed)
    assert L == m.L == 68
    kc = f64(tiny0.kc[0, 0, :, :L])
    vc = f64(tiny0.vc[0, 0, :, :, :L]).transpose(0, 2, 1)
    assert max_abs(kc, m.K[0][:, :L]) < 1e-4
    assert max_abs(vc, m.V[0][:, :L]) < 1e-4
    # four ids (the AR seed and three commits) and three forced commits; the
    # oracle's second forced commit picks between two positions whose p1
    # differ by 7.2e-5, the one decision inside the margin
    t = rp.t
    assert t.ids_exact == 4 and t.ids_excluded == 0, t
    assert t.commits_exact + t.commits_excluded == 3 and t.commits_excluded <= 1, t
    print(f"config 1: {t}")


@pytest.mark.parametrize("mode", [dv.MODE_THRESHOLD, dv.MODE_SPEC_LINEAR, dv.MODE_AR])
def test_tiny_fp32_modes_seed4(tiny4, mode):
    tokens, st, recs, L, seed = tiny4.traced(mode, 4, 0.9, 16)
    rp, m = replay_trace(tiny4, mode, 4, 0.9, 16, tokens, st, recs, L, seed)
    # a well-conditioned trajectory: nothing inside the margin, so the whole
    # run equals the oracle's own decode
    tr, _ = tiny4.oracle(mode, 4, 0.9, 16)
    assert tr.min_margin >= MARGIN
    assert tokens == tr.tokens and st.nfe == tr.nfe
    assert rp.t.ids_excluded == rp.t.commits_excluded == 0
    if mode == dv.MODE_SPEC_LINEAR:
        hist = np.bincount(tr.accept_lens, minlength=dv.binding.HIST)[:dv.binding.HIST]
        assert list(st.accept_hist) == hist.tolist()


def test_tiny_fp32_graphs_match_eager(tiny4):
    a, sa = tiny4.gpu(dv.MODE_THRESHOLD, 4, 0.9, 16, use_graphs=1)
    b, sb = tiny4.gpu(dv.MODE_THRESHOLD, 4, 0.9, 16, use_graphs=0)
    assert a == b and sa.nfe == sb.nfe


def test_trace_does_not_change_the_decode(tiny4):
    a, sa = tiny4.gpu(dv.MODE_SPEC_LINEAR, 4, 0.9, 16)
    b, sb, _, _, _ = tiny4.traced(dv.MODE_SPEC_LINEAR, 4, 0.9, 16)
    assert a == b and sa.nfe == sb.nfe and list(sa.accept_hist) == list(sb.accept_hist)


@pytest.mark.parametrize("seed,mode", [(6, dv.MODE_SPEC_LINEAR)])
def test_bf16_reduced_model_matches_oracle(cuda, seed, mode):
    """2 layers, hidden 1024, 8/1 heads of 128, SwiGLU 1024, vocab 4096;
    48-token context (32 vision + 16 prompt), B=16, 32 tokens, speculative:
    the whole trajectory equals the oracle's own (its smallest argmax margin
    is 0.012)."""
    s = Setup(SMALL_BF16, seed, cuda, 32, 16, 0)
    tokens, st = s.gpu(mode, 16, 0.9, 32)
    tr, m = s.oracle(mode, 16, 0.9, 32)
    assert tr.min_margin >= MARGIN
    assert tokens == tr.tokens and st.nfe == tr.nfe
    s.eng.close()


@pytest.mark.parametrize("seed,mode,persistent", [(1, dv.MODE_THRESHOLD, 0), (3, dv.MODE_THRESHOLD, 0),
                                                  (6, dv.MODE_SPEC_LINEAR, 0), (2, dv.MODE_SPEC_LINEAR, 0),
                                                  (1, dv.MODE_THRESHOLD, 1), (6, dv.MODE_SPEC_LINEAR, 1)])
def test_bf16_reduced_model_engine_path(cuda, seed, mode, persistent):
    """The engine's own graph-driven decode of the reduced bf16 model (B=16,
    tau 0.9, 32 tokens; in-graph commit, shift-1 row mapping, block set-up,
    emission and, for speculative decoding, the accept kernel), every forward
    replayed against the oracle: decisions bit-exact at the 1e-3 bar on the
    rows the LM head read, within DELTA on the oracle's own rows, hidden rows
    within 2e-2 plus one storage ulp.  persistent=1: each forward is one
    persistent launch (QKV, attention, merge, O-projection, gate/up, down
    per layer); at this size most CTAs of a GEMM phase hold one k block or
    none, so every output tile is split over many CTAs."""
    s = Setup(SMALL_BF16, seed, cuda, 32, 16, 0, options={"persistent": persistent} if persistent else None)
    tokens, st, recs, L, sd = s.traced(mode, 16, 0.9, 32)
    rp, m = replay_trace(s, mode, 16, 0.9, 32, tokens, st, recs, L, sd)
    t = rp.t
    assert t.ids_exact > 0 and t.secondary_checked > 0, t
    if mode == dv.MODE_THRESHOLD:
        assert t.commits_exact > 0, t
    print(f"seed {seed} mode {mode}: {t}")
    s.eng.close()


def test_bf16_reduced_model_routing_teacher_forced(cuda):
    """Certificate-guided routing (B=16, k=2, 32 tokens; the 32 vision rows
    hidden in TEXT-ONLY passes) of the reduced bf16 model, per pass and
    teacher-forced: each FULL pass of the oracle's trajectory replayed with
    the engine's forward, each TEXT-ONLY pass with its TEXT-ONLY forward,
    then the fused LM head; top-1 ids compared wherever the oracle's margin
    is at least DELTA, p1 within DELTA; finished blocks appended causally."""
    s = Setup(SMALL_BF16, 1, cuda, 32, 16, 0)
    eng, d, dev = s.eng, SMALL_BF16, cuda
    B, k, n_vis = 16, 2, 32
    eng.prefill(s.vis_t.to(dev), n_vis, torch.from_numpy(s.ids).to(dev), 16)
    _, seed_gpu = eng.position()
    lw = ws_tensor(dv.lmhead_workspace_size(B, d.vocab, d.hidden, dv.DVLM_BF16), dev)
    x = torch.zeros((B, d.hidden), dtype=torch.bfloat16, device=dev)
    counts = {"full": 0, "text": 0, "top1": 0}

    def on_pass(kind, L, toks, p1o, topo):
        assert eng.position()[0] == L
        t = torch.tensor(toks, dtype=torch.int32, device=dev)
        if kind == "full":
            eng.forward(B, 0, d.n_layers, tokens=t, x_out=x)
        else:
            eng.forward_text_only(B, n_vis, tokens=t, x_out=x)
        top = torch.zeros(B, dtype=torch.int32, device=dev)
        p1 = torch.zeros(B, dtype=torch.float32, device=dev)
        st = status(dev)
        dv.lmhead_conf_commit(x, s.dm.lm_head, R=B, H=d.hidden, V=d.vocab, dtype=dv.DVLM_BF16, apply_rmsnorm=1,
                              top1_id=top, top1_prob=p1, workspace=lw, status=st)
        assert_ok(st)
        p1g, topg = p1.cpu().numpy(), top.cpu().numpy()
        counts[kind] += 1
        for j in range(1, B):  # position j is scored by row j - 1
            assert abs(p1g[j - 1] - p1o[j]) <= DELTA, (kind, j)
            if p1o[j] >= 0.5 + DELTA / 2:          # a p1 above 1/2 leaves the runner-up below 1 - p1
                assert topg[j - 1] == topo[j], (kind, j)
                counts["top1"] += 1

    def on_block(L, toks):
        eng.forward(B, B, d.n_layers, tokens=torch.tensor(toks, dtype=torch.int32, device=dev), advance=True)

    m = O.OracleModel(s.od, weights=s.w, bf16=True, Lmax=s.Lmax)
    seed_o = O.prefill(m, s.vis.astype(np.float64), s.ids)
    assert seed_o == seed_gpu
    tr = O.decode_lown(m, seed_o, B, k, n_vis=n_vis, max_new=32, on_pass=on_pass, on_block=on_block)
    eng.check()
    assert counts["full"] == tr.n_full and counts["text"] == tr.n_text
    assert counts["text"] > 0 and counts["top1"] > 0
    s.eng.close()


@pytest.mark.parametrize("seed,k", [(1, 2), (3, 1)])
def test_bf16_reduced_model_routing_engine_path(cuda, seed, k):
    """Certificate-guided routing driven by the engine itself (mode
    DVLM_MODE_ROUTE: anchors kept on the device, FULL and TEXT-ONLY passes
    captured in CUDA graphs, certified and divergence-first commits), B=16,
    32 tokens, the 32 vision rows hidden in TEXT-ONLY passes; every pass
    replayed against the oracle (the TEXT-ONLY ones with the vision slots
    hidden), the engine's certificate and commits held to the routing rules."""
    s = Setup(SMALL_BF16, seed, cuda, 32, 16, 0)
    rb = dv.engine_trace_record_bytes(s.dm.c_model())
    buf = torch.zeros(256 * rb, dtype=torch.uint8, device=cuda)
    cnt = torch.zeros(4, dtype=torch.int32, device=cuda)
    s.eng.set_trace(buf, cnt)
    try:
        s.eng.prefill(s.vis_t.to(cuda), 32, torch.from_numpy(s.ids).to(cuda), 16)
        out = torch.zeros(32, dtype=torch.int32, device=cuda)
        st = dv.Stats()
        s.eng.generate(dv.DecodeCfg(16, 0.9, dv.MODE_ROUTE, 1, 32, 1, k, 32), out, st)
        s.eng.check()
    finally:
        s.eng.set_trace(None, None)
    recs = parse_trace(buf.cpu().numpy(), int(cnt[0].item()), rb, SMALL_BF16.hidden, True)
    m, so = s.oracle_model()
    rp = Replay(m, so, 16, 0.9, decide="gpu", hidden_check=_bf16_hidden, secondary=DELTA, seed_bar=DELTA)
    got = rp.routing(recs, 32, k, 32)
    assert got == out.cpu().numpy().tolist()
    assert rp._next == len(recs) == st.nfe
    assert st.n_text_passes == sum(r.kind == 9 for r in recs) > 0
    print(f"routing seed {seed} k {k}: {rp.t}, text passes {st.n_text_passes} of {st.nfe}")
    s.eng.close()


def test_engine_refuses_option_pairs_that_can_stall(cuda):
    """5-stage gate/up with 5-stage down: early-launched down CTAs fit beside
    gate/up CTAs and could take the room of gate/up CTAs whose stream-K
    partials the resident ones wait for, so the engine refuses the pair in
    either order (DVLM_ERR_UNSUPPORTED = 3) and keeps its settings."""
    s = Setup(SMALL_BF16, 0, cuda, 32, 16, 0)
    eng = s.eng
    eng.set_option("gateup_stages", 5)
    with pytest.raises(dv.DvlmError) as e:
        eng.set_option("down_stages", 5)
    assert e.value.status == 3
    assert eng.get_option("down_stages") == 10
    eng.set_option("gateup_stages", 10)
    eng.set_option("down_stages", 5)
    with pytest.raises(dv.DvlmError) as e:
        eng.set_option("gateup_stages", 5)
    assert e.value.status == 3
    assert eng.get_option("gateup_stages") == 10
    eng.close()
