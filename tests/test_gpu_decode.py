"""End-to-end block decoding through the engine vs the oracle's decoders on
small models: the tiny fp32 model (first configuration: 64-token context of 32
vision embeddings, 16 prompt and 16 committed ids, one B=4 block, threshold
0.9) and a reduced-depth bf16 model with the same per-head shapes as the
Qwen2.5-3B decoder.

fp32: token sequences and commit counts must match exactly when every
decision on the oracle's trajectory is at least 1e-3 away from its threshold /
runner-up (GPU and oracle p1 agree to ~1e-6 there; the seeds were chosen by
running the oracle alone); otherwise a mismatch is only allowed when the
oracle's trajectory does contain such a near-tie.

bf16: GPU and oracle round to bf16 at the same storage points, but a value
whose fp32 and fp64 sums fall on either side of a bf16 rounding boundary
lands one storage ulp apart, and the LM head (N(0, 0.02) x 25 weights) turns
such a flip into a p1 difference of a few 1e-2.  A whole trajectory can then
branch at a decision the oracle takes with a margin of 1e-2, so the
threshold decoder is checked per iteration instead, teacher-forced: every
noisy forward of the oracle's trajectory is replayed on the GPU with the same
block tokens over the same cache, and top-1 ids and commit decisions must
agree wherever the oracle's margin is at least DELTA."""
import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import dvlm_gen as gen
import oracle as O
from dvlm_gen.device import DeviceModel, kv_buffers
from gpu_util import assert_ok, f64, max_abs, status, ws_tensor

pytestmark = pytest.mark.gpu
MARGIN = 1e-3
# bound on |p1(GPU) - p1(oracle)| for the bf16 reduced model on identical inputs:
# hidden states one storage ulp apart in a few elements move p1 by a few 1e-2
# (GPU against oracle: up to 0.03 measured; a CPU model of such rounding
# flips: up to 0.066, tests/test_precision_model.py)
DELTA = 0.1

SMALL_BF16 = gen.ModelDims(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=1, head_dim=128, inter=1024,
                           vocab=4096, lm_scale=25.0, dtype="bf16")


class Setup:
    def __init__(self, dims, seed, cuda, n_vis, n_prompt, n_comm, Lmax=512):
        self.dims, self.seed, self.cuda = dims, seed, cuda
        self.dm = DeviceModel(dims, seed, device=cuda)
        self.kc, self.vc = kv_buffers(dims, Lmax, device=cuda)
        cm = self.dm.c_model()
        self.ws = ws_tensor(dv.engine_workspace_size(cm, Lmax, 16, 128), cuda)
        self.eng = dv.Engine(cm, self.kc, self.vc, Lmax, 16, 128, self.ws)
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

    def oracle(self, mode, B, tau, n_new):
        m = O.OracleModel(self.od, weights=self.w, bf16=self.dims.dtype == "bf16", Lmax=self.Lmax)
        s = O.prefill(m, self.vis.astype(np.float64), self.ids)
        if mode == dv.MODE_THRESHOLD:
            return O.decode_threshold(m, s, B, tau, n_new), m
        if mode == dv.MODE_SPEC_LINEAR:
            return O.decode_spec_linear(m, s, B, n_new), m
        return O.decode_ar(m, s, n_new), m


def _compare(tokens, st, tr, mode):
    if tr.min_margin >= MARGIN:
        assert tokens == tr.tokens
        assert st.nfe == tr.nfe
        if mode == dv.MODE_THRESHOLD:
            hist = np.bincount(tr.commits_per_iter, minlength=dv.binding.HIST)[:dv.binding.HIST]
            assert list(st.commit_hist) == hist.tolist()
        if mode == dv.MODE_SPEC_LINEAR:
            hist = np.bincount(tr.accept_lens, minlength=dv.binding.HIST)[:dv.binding.HIST]
            assert list(st.accept_hist) == hist.tolist()
    elif tokens != tr.tokens:
        assert tr.min_margin < MARGIN


@pytest.fixture(scope="module")
def tiny0(cuda):
    return Setup(gen.TINY, 0, cuda, 32, 16, 16, Lmax=128)


@pytest.fixture(scope="module")
def tiny4(cuda):
    return Setup(gen.TINY, 4, cuda, 32, 16, 16, Lmax=128)


def test_tiny_fp32_block_step_seed0(tiny0):
    """The tiny configuration exactly as stated: seed 0, one B=4 block."""
    tokens, st = tiny0.gpu(dv.MODE_THRESHOLD, 4, 0.9, 4)
    tr, m = tiny0.oracle(dv.MODE_THRESHOLD, 4, 0.9, 4)
    _compare(tokens, st, tr, dv.MODE_THRESHOLD)
    # the exact KV cache after the block (prefill + causal append) within 1e-4
    L = m.L
    kc = f64(tiny0.kc[0, 0, :, :L])
    vc = f64(tiny0.vc[0, 0, :, :, :L]).transpose(0, 2, 1)
    if tokens == tr.tokens:
        assert max_abs(kc, m.K[0][:, :L]) < 1e-4
        assert max_abs(vc, m.V[0][:, :L]) < 1e-4


@pytest.mark.parametrize("mode", [dv.MODE_THRESHOLD, dv.MODE_SPEC_LINEAR, dv.MODE_AR])
def test_tiny_fp32_modes_seed4(tiny4, mode):
    tokens, st = tiny4.gpu(mode, 4, 0.9, 16)
    tr, m = tiny4.oracle(mode, 4, 0.9, 16)
    assert tr.min_margin >= MARGIN  # chosen seed: well-conditioned trajectory
    _compare(tokens, st, tr, mode)


def test_tiny_fp32_graphs_match_eager(tiny4):
    a, sa = tiny4.gpu(dv.MODE_THRESHOLD, 4, 0.9, 16, use_graphs=1)
    b, sb = tiny4.gpu(dv.MODE_THRESHOLD, 4, 0.9, 16, use_graphs=0)
    assert a == b and sa.nfe == sb.nfe


@pytest.mark.parametrize("seed,mode", [(6, dv.MODE_SPEC_LINEAR)])
def test_bf16_reduced_model_matches_oracle(cuda, seed, mode):
    """2 layers, hidden 1024, 8/1 heads of 128, SwiGLU 1024, vocab 4096;
    48-token context (32 vision + 16 prompt), B=16, 32 tokens, speculative."""
    s = Setup(SMALL_BF16, seed, cuda, 32, 16, 0)
    tokens, st = s.gpu(mode, 16, 0.9, 32)
    tr, m = s.oracle(mode, 16, 0.9, 32)
    assert tr.min_margin >= MARGIN
    _compare(tokens, st, tr, mode)
    s.eng.close()


@pytest.mark.parametrize("seed", [1, 3])
def test_bf16_reduced_model_threshold_teacher_forced(cuda, seed):
    """Threshold decoding (B=16, tau 0.9, 32 tokens) of the reduced bf16 model:
    each noisy forward of the oracle's trajectory replayed on the GPU (engine
    forward over the same cache, then the fused LM head with the final
    RMSNorm), finished blocks appended causally on both sides."""
    s = Setup(SMALL_BF16, seed, cuda, 32, 16, 0)
    eng, d, dev = s.eng, SMALL_BF16, cuda
    B, tau = 16, 0.9
    eng.prefill(s.vis_t.to(dev), 32, torch.from_numpy(s.ids).to(dev), 16)
    _, seed_gpu = eng.position()
    lw = ws_tensor(dv.lmhead_workspace_size(B, d.vocab, d.hidden, dv.DVLM_BF16), dev)
    x = torch.zeros((B, d.hidden), dtype=torch.bfloat16, device=dev)
    counts = {"iters": 0, "top1": 0, "commit": 0}

    def on_iter(L, toks, masked, p1o, topo, p2o):
        assert eng.position()[0] == L
        eng.forward(B, 0, d.n_layers, tokens=torch.tensor(toks, dtype=torch.int32, device=dev), x_out=x)
        top = torch.zeros(B, dtype=torch.int32, device=dev)
        p1 = torch.zeros(B, dtype=torch.float32, device=dev)
        st = status(dev)
        dv.lmhead_conf_commit(x, s.dm.lm_head, R=B, H=d.hidden, V=d.vocab, dtype=dv.DVLM_BF16, apply_rmsnorm=1,
                              top1_id=top, top1_prob=p1, workspace=lw, status=st)
        assert_ok(st)
        p1g, topg = p1.cpu().numpy(), top.cpu().numpy()
        counts["iters"] += 1
        for j in range(1, B):  # position j is scored by row j - 1
            if not masked[j]:
                continue
            r = j - 1
            assert abs(p1g[r] - p1o[j]) <= DELTA
            if p1o[j] - p2o[j] >= DELTA:
                assert topg[r] == topo[j]
                counts["top1"] += 1
            if abs(p1o[j] - tau) >= DELTA:
                assert (p1g[r] >= tau) == (p1o[j] >= tau)
                counts["commit"] += 1

    def on_block(L, toks):
        eng.forward(B, B, d.n_layers, tokens=torch.tensor(toks, dtype=torch.int32, device=dev), advance=True)

    m = O.OracleModel(s.od, weights=s.w, bf16=True, Lmax=s.Lmax)
    seed_o = O.prefill(m, s.vis.astype(np.float64), s.ids)
    assert seed_o == seed_gpu
    tr = O.decode_threshold(m, seed_o, B, tau, 32, on_iter=on_iter, on_block=on_block)
    eng.check()
    # the comparison covered the whole trajectory and most of its decisions
    assert counts["iters"] == tr.nfe - len(tr.tokens) // B
    assert counts["top1"] > 0 and counts["commit"] > 0
    s.eng.close()


@pytest.mark.parametrize("seed", [6, 2])
def test_bf16_reduced_model_spec_teacher_forced(cuda, seed):
    """Linear self-speculative decoding (B=16, 32 tokens) of the reduced bf16
    model, per round and teacher-forced: the oracle's draft pass ([seed,
    MASK...], noisy) and verify pass (its draft, causal) are replayed on the
    GPU over the same cache, top-1 ids compared wherever the oracle's margin
    is at least DELTA and p1 within DELTA, then the cache length and seed are
    set to the oracle's accepted prefix."""
    s = Setup(SMALL_BF16, seed, cuda, 32, 16, 0)
    eng, d, dev = s.eng, SMALL_BF16, cuda
    B = 16
    eng.prefill(s.vis_t.to(dev), 32, torch.from_numpy(s.ids).to(dev), 16)
    _, seed_gpu = eng.position()
    lw = ws_tensor(dv.lmhead_workspace_size(B, d.vocab, d.hidden, dv.DVLM_BF16), dev)
    x = torch.zeros((B, d.hidden), dtype=torch.bfloat16, device=dev)
    counts = {"rounds": 0, "draft": 0, "verify": 0}

    def gpu_rows(toks, n_clean):
        eng.forward(B, n_clean, d.n_layers, tokens=torch.tensor(toks, dtype=torch.int32, device=dev), x_out=x)
        top = torch.zeros(B, dtype=torch.int32, device=dev)
        p1 = torch.zeros(B, dtype=torch.float32, device=dev)
        st = status(dev)
        dv.lmhead_conf_commit(x, s.dm.lm_head, R=B, H=d.hidden, V=d.vocab, dtype=dv.DVLM_BF16, apply_rmsnorm=1,
                              top1_id=top, top1_prob=p1, workspace=lw, status=st)
        assert_ok(st)
        return top.cpu().numpy(), p1.cpu().numpy()

    def check(rows, conf, top, p1, key):
        for r in range(rows):
            assert abs(p1[r] - conf.p1[r]) <= DELTA, (key, r, p1[r], conf.p1[r])
            if conf.p1[r] - conf.p2[r] >= DELTA:
                assert top[r] == conf.top1[r], (key, r)
                counts[key] += 1

    def on_round(L, toks, c, draft, g, k, nxt):
        assert eng.position()[0] == L
        top, p1 = gpu_rows(toks, 0)
        check(B - 1, c, top, p1, "draft")        # row r drafts position r + 1
        top, p1 = gpu_rows(draft, B)
        check(B, g, top, p1, "verify")
        eng.set_position(L + k, nxt)
        counts["rounds"] += 1

    m = O.OracleModel(s.od, weights=s.w, bf16=True, Lmax=s.Lmax)
    seed_o = O.prefill(m, s.vis.astype(np.float64), s.ids)
    assert seed_o == seed_gpu
    tr = O.decode_spec_linear(m, seed_o, B, 32, on_round=on_round)
    eng.check()
    assert counts["rounds"] == len(tr.accept_lens)
    assert counts["draft"] > 0 and counts["verify"] > 0
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
