"""Full-size decode (Qwen2.5-3B-shaped decoder: 36 layers, hidden 2048, 16/2
heads, SwiGLU 11008, vocab 151936, random init; 1280 vision + 64 prompt
context; B=16) in the launch configuration the benchmark times.  The oracle
cannot run 36 layers over this context in test time, so these tests check
(a) sampled outputs the oracle computes on its own inputs -- the first layer's
K/V over the first 64 context slots -- and (b) properties that hold at any
size: linear self-speculative decoding reproduces greedy AR decoding exactly,
threshold decoding with B=1 is AR decoding, every block of threshold decoding
commits B-1 positions over its iterations, runs are deterministic and graph
replay equals eager launches."""
import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import dvlm_gen as gen
import oracle as O
from dvlm_gen.device import DeviceModel, kv_buffers
from gpu_util import f64, max_abs, ws_tensor

pytestmark = pytest.mark.gpu
SEED = 4          # the full decode configuration is the fifth: seed 4
N_VIS, N_PROMPT = 1280, 64


@pytest.fixture(scope="module")
def full(cuda):
    dims = gen.QWEN3B
    dm = DeviceModel(dims, SEED, device=cuda)
    Lmax = N_VIS + N_PROMPT + 256 + 64
    kc, vc = kv_buffers(dims, Lmax, device=cuda)
    cm = dm.c_model()
    ws = ws_tensor(dv.engine_workspace_size(cm, Lmax, 16, N_VIS + N_PROMPT), cuda)
    eng = dv.Engine(cm, kc, vc, Lmax, 16, N_VIS + N_PROMPT, ws)
    vis_t, vis, ids = gen.decode_context(dims, SEED, N_VIS, N_PROMPT)
    eng.prefill(vis_t.to(cuda), N_VIS, torch.from_numpy(ids).to(cuda), N_PROMPT)
    eng.check()
    L0, seed0 = eng.position()
    assert L0 == N_VIS + N_PROMPT
    yield dict(dims=dims, dm=dm, eng=eng, kc=kc, vc=vc, vis=vis, L0=L0, seed0=seed0, cm=cm, ws=ws)
    eng.close()


def _gen(full, mode, B, n, tau=0.9, graphs=1):
    eng = full["eng"]
    eng.set_position(full["L0"], full["seed0"])
    out = torch.zeros(n, dtype=torch.int32, device="cuda")
    st = dv.Stats()
    eng.generate(dv.DecodeCfg(B, tau, mode, 1, n, graphs), out, st)
    eng.check()
    return out.cpu().numpy().tolist(), st


def test_prefill_first_layer_kv_matches_oracle(full):
    dims = full["dims"]
    n = 64
    w = {f"0.{k}": gen.layer_weight(dims, SEED, 0, k)[1].astype(np.float64) for k in gen.layer_weight_names()}
    m = O.OracleModel(O.dims_from(dims), weights=w, bf16=True, Lmax=n)
    m.layer(0, full["vis"][:n].astype(np.float64), 0, n)
    k = f64(full["kc"][0, 0, :, :n])
    v = f64(full["vc"][0, 0, :, :, :n]).transpose(0, 2, 1)
    assert max_abs(k, m.K[0][:, :n]) < 2e-2
    assert max_abs(v, m.V[0][:, :n]) < 2e-2


def test_spec_linear_equals_greedy_ar(full):
    ar, st_ar = _gen(full, dv.MODE_AR, 16, 48)
    sp, st_sp = _gen(full, dv.MODE_SPEC_LINEAR, 16, 48)
    assert sp == ar
    assert st_ar.nfe == 48
    assert sum(k * c for k, c in enumerate(st_sp.accept_hist)) >= 48


def test_threshold_block1_equals_ar(full):
    ar, _ = _gen(full, dv.MODE_AR, 16, 20)
    th, st = _gen(full, dv.MODE_THRESHOLD, 1, 20)
    assert th == ar and st.nfe == 20


def test_threshold_blocks_deterministic_and_consistent(full):
    n = 64
    a, sa = _gen(full, dv.MODE_THRESHOLD, 16, n)
    b, sb = _gen(full, dv.MODE_THRESHOLD, 16, n, graphs=0)
    assert a == b
    assert sa.nfe == sb.nfe and list(sa.commit_hist) == list(sb.commit_hist)
    blocks = n // 16
    assert sa.n_rounds == blocks
    assert sum(c * h for c, h in enumerate(sa.commit_hist)) == blocks * 15
    assert sa.nfe == sa.n_iters + blocks
    assert all(0 <= t < full["dims"].vocab for t in a)
    # the first token of every block is the AR prediction of its context
    ar, _ = _gen(full, dv.MODE_AR, 16, 1)
    assert a[0] == ar[0]


def test_host_end_to_end_matches_device_path(full):
    """dvlm_generate_host (host buffers in, host tokens out) equals prefill +
    generate on device buffers."""
    dims = full["dims"]
    vis_t, vis, ids = gen.decode_context(dims, SEED, N_VIS, N_PROMPT)
    want, _ = _gen(full, dv.MODE_THRESHOLD, 16, 32)
    out = torch.zeros(32, dtype=torch.int32).pin_memory()
    st = dv.Stats()
    full["eng"].generate_host(dv.DecodeCfg(16, 0.9, dv.MODE_THRESHOLD, 1, 32, 1), vis_t.pin_memory(), N_VIS,
                              torch.from_numpy(ids).pin_memory(), N_PROMPT, out, st)
    full["eng"].check()
    assert out.tolist() == want
