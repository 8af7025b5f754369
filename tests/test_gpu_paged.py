"""Paged KV cache [Fast-dVLM technical overview (ocdem.com), section 2.3.2:
paged KV cache management; reading: 64-slot pages, slot s of a sequence in row
s % 64 of page table[s // 64]].

* dvlm_block_attn_paged over a batch of sequences with ragged lengths, whose
  pages are scattered in a random order among NaN-poisoned unused pages:
  bitwise equal to dvlm_block_attn on each sequence's contiguous cache (the
  same arithmetic chunk by chunk), and within the attention bar (2e-2 plus one
  storage ulp) of the oracle's paged_block_attention; noisy, causal and mixed
  rows.
* A page id outside the page store is reported as DVLM_ERR_BOUNDS.
* An engine switched to a paged cache (dvlm_engine_set_paged) decodes exactly
  the tokens of the same engine on a contiguous cache (threshold and
  speculative modes), and its pages hold bitwise the contiguous cache's K/V."""
import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import dvlm_gen as gen
import oracle as O
from dvlm_gen.device import DeviceModel, kv_buffers
from gpu_util import assert_bf16_close, f64, status, ws_tensor

pytestmark = pytest.mark.gpu
Hq, Hkv, D, B, P = 16, 2, 128, 16, 64


def _scatter_case(cuda, lens, seed=3, n_extra=5):
    rng = np.random.default_rng(seed)
    n_chunks = [(L + B + P - 1) // P for L in lens]
    max_pages = max(n_chunks)
    n_pages = sum(n_chunks) + n_extra
    perm = rng.permutation(n_pages)
    table = np.zeros((len(lens), max_pages), dtype=np.int32)
    kp = np.full((n_pages, Hkv, P, D), np.nan, dtype=np.float32)
    vp = np.full((n_pages, Hkv, P, D), np.nan, dtype=np.float32)
    conts, nxt = [], 0
    for b, L in enumerate(lens):
        n = L + B
        k = gen.normal_bf16(seed + b, "paged.k", (Hkv, n, D))[1]
        v = gen.normal_bf16(seed + b, "paged.v", (Hkv, n, D))[1]
        conts.append((k, v))
        for c in range(n_chunks[b]):
            page = int(perm[nxt])
            nxt += 1
            table[b, c] = page
            m = min(P, n - c * P)
            kp[page, :, :m] = k[:, c * P:c * P + m]
            vp[page, :, :m] = v[:, c * P:c * P + m]
    q = gen.normal_bf16(seed, "paged.q", (len(lens), B, Hq, D))[1]
    return q, kp, vp, table, conts, n_pages, max_pages


@pytest.mark.parametrize("n_clean", [0, 16, 5])
def test_paged_attention_matches_contiguous_and_oracle(cuda, n_clean):
    lens = [100, 700, 1344]
    q, kp, vp, table, conts, n_pages, max_pages = _scatter_case(cuda, lens)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(cuda)
    qd = bf(q)
    kpd = bf(kp)
    vpd = bf(vp.transpose(0, 1, 3, 2))   # V^T pages [n_pages, Hkv, D, 64]
    out = torch.empty_like(qd)
    st = status(cuda)
    dv.block_attn_paged(qd, out, kpd, vpd, torch.from_numpy(table).to(cuda),
                        torch.tensor(lens, dtype=torch.int32, device=cuda), n_batch=len(lens), n_rows=B,
                        n_clean=n_clean, n_pages=n_pages, max_pages=max_pages, Hq=Hq, Hkv=Hkv, D=D,
                        scale=D ** -0.5, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for b, L in enumerate(lens):
        k, v = conts[b]
        Lmax = (L + B + 7) // 8 * 8
        kc = np.zeros((1, Hkv, Lmax, D), dtype=np.float32)
        vc = np.zeros((1, Hkv, Lmax, D), dtype=np.float32)
        kc[0, :, :L + B], vc[0, :, :L + B] = k, v
        o1 = torch.empty((1, B, Hq, D), dtype=torch.bfloat16, device=cuda)
        dv.block_attn(qd[b:b + 1].contiguous(), o1, bf(kc), bf(vc.transpose(0, 1, 3, 2)), n_batch=1, n_rows=B,
                      n_clean=n_clean, L=L, Lmax=Lmax, Hq=Hq, Hkv=Hkv, D=D, scale=D ** -0.5, dtype=dv.DVLM_BF16,
                      status=st)
        torch.cuda.synchronize()
        assert torch.equal(o1[0], out[b]), b
        want = O.paged_block_attention(q[b].astype(np.float64), kp.astype(np.float64), vp.astype(np.float64),
                                       table[b].tolist(), L, n_clean, D ** -0.5)
        assert_bf16_close(f64(out[b]), want, 2e-2, f"sequence {b}")


def test_paged_attention_reports_a_bad_page(cuda):
    lens = [200]
    q, kp, vp, table, conts, n_pages, max_pages = _scatter_case(cuda, lens)
    kp = np.nan_to_num(kp)
    vp = np.nan_to_num(vp)
    table[0, 1] = n_pages + 7
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(cuda)
    qd = bf(q)
    out = torch.empty_like(qd)
    st = status(cuda)
    dv.block_attn_paged(qd, out, bf(kp), bf(vp.transpose(0, 1, 3, 2)), torch.from_numpy(table).to(cuda),
                        torch.tensor(lens, dtype=torch.int32, device=cuda), n_batch=1, n_rows=B, n_clean=0,
                        n_pages=n_pages, max_pages=max_pages, Hq=Hq, Hkv=Hkv, D=D, scale=D ** -0.5, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 8   # DVLM_ERR_BOUNDS


SMALL = gen.ModelDims(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=1, head_dim=128, inter=1024, vocab=4096,
                      lm_scale=25.0, dtype="bf16")


@pytest.mark.parametrize("mode", [dv.MODE_THRESHOLD, dv.MODE_SPEC_LINEAR])
def test_paged_engine_decodes_like_contiguous(cuda, mode):
    seed, Lmax, n_new = 5, 192, 32
    dm = DeviceModel(SMALL, seed, device=cuda)
    cm = dm.c_model()
    vis_t, vis, ids = gen.decode_context(SMALL, seed, 32, 16)
    runs = []
    for paged in (False, True):
        kc, vc = kv_buffers(SMALL, Lmax, device=cuda)
        ws = ws_tensor(dv.engine_workspace_size(cm, Lmax, 16, 64), cuda)
        eng = dv.Engine(cm, kc, vc, Lmax, 16, 64, ws)
        eng.set_option("prefill_gemm", 0)      # both prefill in 16-row forwards
        pages = None
        if paged:
            max_pages = Lmax // 64
            n_pages = max_pages + 3
            perm = np.random.default_rng(1).permutation(n_pages)[:max_pages].astype(np.int32)
            kp = torch.full((SMALL.n_layers, n_pages, SMALL.n_kv_heads, 64, 128), float("nan"),
                            dtype=torch.bfloat16, device=cuda)
            vp = torch.full((SMALL.n_layers, n_pages, SMALL.n_kv_heads, 128, 64), float("nan"),
                            dtype=torch.bfloat16, device=cuda)
            table = torch.from_numpy(perm).to(cuda)
            eng.set_paged(kp, vp, table, n_pages, max_pages)
            pages = (kp, vp, perm)
        eng.prefill(vis_t.to(cuda), 32, torch.from_numpy(ids).to(cuda), 16)
        out = torch.zeros(n_new, dtype=torch.int32, device=cuda)
        st = dv.Stats()
        eng.generate(dv.DecodeCfg(16, 0.9, mode, 1, n_new, 1), out, st)
        eng.check()
        L, _ = eng.position()
        runs.append((out.cpu().numpy().tolist(), st.nfe, L, kc, vc, pages))
        eng.close()
    (ta, na, La, kc, vc, _), (tb, nb, Lb, _, _, (kp, vp, perm)) = runs
    assert ta == tb and na == nb and La == Lb
    for s0 in range(0, La, 64):
        m = min(64, La - s0)
        page = int(perm[s0 // 64])
        assert torch.equal(kp[:, page, :, :m], kc[:, 0, :, s0:s0 + m])
        assert torch.equal(vp[:, page, :, :, :m], vc[:, 0, :, :, s0:s0 + m])
