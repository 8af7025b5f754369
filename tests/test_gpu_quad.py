"""Quadratic self-speculative decoding on the GPU [Fast-dVLM technical
overview (ocdem.com), section 2.3.1: draft and verify in one forward at
O(B^2) cost] against the oracle's forward_quadratic / decode_spec_quadratic.

* The fused forward alone (dvlm_forward_quad): all B + B*B final hidden rows
  (verify rows, then every candidate block) and the verify rows' K/V in the
  cache, against the oracle's fused forward within the bf16 bar (2e-2 plus
  one storage ulp), for B = 4 and B = 16 over a 48-slot context, for B = 8
  on a wider model (SwiGLU 4096: the token-major GEMMs split their k range up
  to 16 ways, gate/up tiles included), and after stale NaN-poisoned slots
  past L + B (no candidate block may read them).
* Decoding through the engine's own graph path (mode DVLM_MODE_SPEC_QUAD):
  every forward replayed against the oracle, teacher-forced
  (tests/decode_replay.py): verify and candidate rows within the bf16 bar,
  verify ids, accepted lengths, next-draft ids and seeds bit-exact at the
  1e-3 bar on the rows the LM head read, within DELTA on the oracle's own
  rows.
Reduced model: 2 layers, hidden 1024, 8/1 heads of 128, SwiGLU 1024, vocab
4096 (the per-head shapes of the Qwen2.5-3B decoder)."""
import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import dvlm_gen as gen
import oracle as O
from decode_replay import Replay, parse_trace
from dvlm_gen.device import DeviceModel, kv_buffers
from gpu_util import assert_bf16_close, f64, ws_tensor

pytestmark = pytest.mark.gpu
DELTA = 0.1
SMALL = gen.ModelDims(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=1, head_dim=128, inter=1024, vocab=4096,
                      lm_scale=25.0, dtype="bf16")


# SwiGLU width 4096: the token-major down projection (64 k blocks) splits its
# k range 16 ways over 4 output tiles at B = 8 (72 rows, one token tile), the
# largest split the residual epilogue allows
WIDE = gen.ModelDims(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=1, head_dim=128, inter=4096, vocab=4096,
                     lm_scale=25.0, dtype="bf16")


class Quad:
    def __init__(self, cuda, seed, Lmax=512, max_ctx=320, dims=SMALL):
        self.cuda, self.seed, self.dims = cuda, seed, dims
        self.dm = DeviceModel(dims, seed, device=cuda)
        self.cm = self.dm.c_model()
        self.kc, self.vc = kv_buffers(dims, Lmax, device=cuda)
        self.ws = ws_tensor(dv.engine_workspace_size(self.cm, Lmax, 16, max_ctx), cuda)
        self.eng = dv.Engine(self.cm, self.kc, self.vc, Lmax, 16, max_ctx, self.ws)
        self.vis_t, self.vis, self.ids = gen.decode_context(dims, seed, 32, 16)
        self.Lmax = Lmax

    def prefill(self):
        self.eng.prefill(self.vis_t.to(self.cuda), 32, torch.from_numpy(self.ids).to(self.cuda), 16)
        self.eng.check()
        return self.eng.position()

    def oracle(self):
        m = O.OracleModel(O.dims_from(self.dims), weights=O.weights_from_generator(gen, self.dims, self.seed),
                          bf16=True, Lmax=self.Lmax)
        s = O.prefill(m, self.vis.astype(np.float64), self.ids)
        return m, s


@pytest.mark.parametrize("B,dims", [(4, SMALL), (16, SMALL), (8, WIDE)], ids=["B4", "B16", "B8-wide"])
@pytest.mark.parametrize("poison", [False, True])
def test_fused_forward_matches_oracle(cuda, B, dims, poison):
    q = Quad(cuda, 2, dims=dims)
    L, seed = q.prefill()
    if poison:   # stale slots past the context
        q.kc[:, :, :, L:] = float("nan")
        q.vc[:, :, :, :, L:] = float("nan")
    rng = np.random.default_rng(B)
    draft = [seed] + [int(t) for t in rng.integers(0, dims.vocab - 1, size=B - 1)]
    x = torch.zeros((B + B * B, dims.hidden), dtype=torch.bfloat16, device=cuda)
    q.eng.forward_quad(torch.tensor(draft, dtype=torch.int32, device=cuda), B, x)
    q.eng.check()
    assert q.eng.position()[0] == L
    m, s = q.oracle()
    xo = O.forward_quadratic(m, draft, L)
    assert_bf16_close(f64(x[:B]), xo[:B], 2e-2, "verify rows")
    for i in range(B):
        assert_bf16_close(f64(x[B + i * B:B + (i + 1) * B]), xo[B + i * B:B + (i + 1) * B], 2e-2, f"candidate {i}")
    for l in range(dims.n_layers):
        assert_bf16_close(f64(q.kc[l, 0, :, L:L + B]), m.K[l][:, L:L + B], 2e-2, f"K layer {l}")
        assert_bf16_close(f64(q.vc[l, 0, :, :, L:L + B]).transpose(0, 2, 1), m.V[l][:, L:L + B], 2e-2,
                          f"V layer {l}")
    q.eng.close()


@pytest.mark.parametrize("seed,B", [(6, 16), (2, 16), (1, 4)])
def test_quadratic_decode_engine_path(cuda, seed, B):
    q = Quad(cuda, seed)
    rb = dv.engine_trace_record_bytes(q.cm)
    buf = torch.zeros(256 * rb, dtype=torch.uint8, device=cuda)
    cnt = torch.zeros(4, dtype=torch.int32, device=cuda)
    q.prefill()
    q.eng.set_trace(buf, cnt)
    out = torch.zeros(32, dtype=torch.int32, device=cuda)
    st = dv.Stats()
    q.eng.generate(dv.DecodeCfg(B, 0.9, dv.MODE_SPEC_QUAD, 1, 32, 1), out, st)
    q.eng.check()
    q.eng.set_trace(None, None)
    L, s_end = q.eng.position()
    recs = parse_trace(buf.cpu().numpy(), int(cnt[0].item()), rb, SMALL.hidden, True)
    m, s0 = q.oracle()
    rp = Replay(m, s0, B, 0.9, decide="gpu", hidden_check=lambda a, b, w: assert_bf16_close(a, b, 2e-2, w),
                secondary=DELTA, seed_bar=DELTA)
    got = rp.quadratic(recs, 32, L, s_end)
    assert got == out.cpu().numpy().tolist()
    # one forward per round after the first draft pass
    assert st.nfe == 1 + (len(recs) - 1) // 2 == rp.t.forwards
    assert rp.t.ids_exact > 0 and rp.t.secondary_checked > 0, rp.t
    print(f"quad seed {seed} B {B}: {rp.t}, accepted {list(st.accept_hist)}")
    q.eng.close()
