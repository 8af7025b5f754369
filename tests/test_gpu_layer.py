"""One decoder layer at the full Qwen2.5-3B widths (hidden 2048, 16/2 heads,
head_dim 128, SwiGLU 11008) through the engine's fused kernels vs the oracle
layer: QKV GEMM + RMSNorm factor + RoPE + KV-slot write, block attention,
O-proj + residual, gate/up + SwiGLU, down + residual.  Inputs are generator
draws (cache prefix N(0,1), token embeddings or N(0,1) rows), so nothing
from the CUDA path feeds the oracle.  Bar: max abs error 2e-2 on every bf16
output (residual stream and the K/V written), plus one bf16 storage ulp of the
reference where fp32 and fp64 sums round to neighbouring bf16 values (see
gpu_util.assert_bf16_close)."""
import dataclasses

import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import dvlm_gen as gen
import oracle as O
from dvlm_gen.device import DeviceModel, kv_buffers
from gpu_util import assert_bf16_close, f64, ws_tensor

pytestmark = pytest.mark.gpu
TOL = 2e-2
SEED = 4


@pytest.fixture(scope="module")
def layer_setup(cuda):
    dims = dataclasses.replace(gen.QWEN3B, n_layers=1)
    dm = DeviceModel(dims, SEED, device=cuda)
    Lmax, L = 1312, 1280
    kc, vc = kv_buffers(dims, Lmax, device=cuda)
    kpre_t, kpre = gen.normal_bf16(SEED, "layer.kprefix", (dims.n_kv_heads, L, dims.head_dim))
    vpre_t, vpre = gen.normal_bf16(SEED, "layer.vprefix", (dims.n_kv_heads, L, dims.head_dim))
    cm = dm.c_model()
    ws = ws_tensor(dv.engine_workspace_size(cm, Lmax, 16, 64), cuda)
    eng = dv.Engine(cm, kc, vc, Lmax, 16, 64, ws)
    w = {f"0.{n}": gen.layer_weight(dims, SEED, 0, n)[1].astype(np.float64) for n in gen.layer_weight_names()}
    od = O.dims_from(dims)
    return dict(dims=dims, dm=dm, kc=kc, vc=vc, kpre_t=kpre_t, vpre_t=vpre_t, kpre=kpre, vpre=vpre, eng=eng, w=w,
                od=od, L=L, Lmax=Lmax)


def _run(s, x_in_t, tokens_t, masked_t, n_rows, n_clean, cuda):
    L = s["L"]
    s["kc"].zero_()
    s["vc"].zero_()
    s["kc"][0, 0, :, :L] = s["kpre_t"].to(cuda)
    s["vc"][0, 0, :, :, :L] = s["vpre_t"].to(cuda).transpose(-1, -2)
    eng = s["eng"]
    eng.set_position(L, 0)
    xo = torch.zeros((n_rows, s["dims"].hidden), dtype=torch.bfloat16, device=cuda)
    eng.forward(n_rows, n_clean, 1, x_in=x_in_t, tokens=tokens_t, masked=masked_t, x_out=xo)
    eng.check()
    k_new = f64(s["kc"][0, 0, :, L:L + n_rows])
    v_new = f64(s["vc"][0, 0, :, :, L:L + n_rows]).transpose(0, 2, 1)
    return f64(xo), k_new, v_new


def _oracle(s, x, n_clean):
    m = O.OracleModel(s["od"], weights=s["w"], bf16=True, Lmax=s["Lmax"])
    L = s["L"]
    m.K[0][:, :L] = s["kpre"]
    m.V[0][:, :L] = s["vpre"]
    xo = m.layer(0, x, L, n_clean)
    n = x.shape[0]
    return xo, m.K[0][:, L:L + n], m.V[0][:, L:L + n]


def test_noisy_block_of_tokens(layer_setup, cuda):
    """A noisy block of 16 rows: the AR seed then [MASK] / committed ids."""
    s = layer_setup
    dims = s["dims"]
    ids = gen.uniform_ids(SEED, "layer.ids", 16, dims.vocab - 1)
    masked = np.array([0, 1, 1, 0, 1, 1, 1, 1, 0, 1, 1, 1, 1, 1, 0, 1], dtype=np.uint8)
    E_t = gen.embedding_weight(dims, SEED)[0]
    rows = [dims.mask_id if masked[i] else int(ids[i]) for i in range(16)]
    x = E_t[torch.tensor(rows)].float().numpy().astype(np.float64)
    got = _run(s, None, torch.from_numpy(ids).to(cuda), torch.from_numpy(masked).to(cuda), 16, 0, cuda)
    want = _oracle(s, x, 0)
    for g, w, what in zip(got, want, ("x", "k", "v")):
        assert_bf16_close(g, w, TOL, what)


@pytest.mark.parametrize("n_rows,n_clean", [(16, 16), (9, 9), (16, 6)])
def test_clean_rows_from_hidden_states(layer_setup, cuda, n_rows, n_clean):
    """Causal rows (append / verify / prefill) with N(0,1) inputs, ragged row counts."""
    s = layer_setup
    x_t, x = gen.normal_bf16(SEED + n_rows, "layer.x", (n_rows, s["dims"].hidden))
    got = _run(s, x_t.to(cuda), None, None, n_rows, n_clean, cuda)
    want = _oracle(s, x.astype(np.float64), n_clean)
    for g, w, what in zip(got, want, ("x", "k", "v")):
        assert_bf16_close(g, w, TOL, what)
