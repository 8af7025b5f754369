"""The scratch-free fused LM head (dvlm_lmhead_conf_commit_static).

It exists for callers that cannot allocate device memory when they call the
library -- a process whose device memory another framework's caching
allocator reserved up front, or a real-time loop that forbids cudaMalloc
after start-up because an allocation can stall the device.  It keeps its
scratch in one fixed array inside the library instead of a workspace.

Checked here through the C ABI: two calls in a row (different shapes, the
second one after the first left its counters and records in the shared
array) each match the workspace entry point on the same inputs, within the
LM-head tests' bars, the first with certificate anchors taken from the
oracle's top-1 of a related hidden set so that the certified prefix is not
trivially empty; sizes beyond the fixed scratch (too many rows, or a
vocabulary whose scratch layout overflows the array) are refused on the host;
and a call after a warm-up call leaves the device's free memory unchanged.
This file is collected last so that a stop-at-first-failure run has already
run every other test."""
import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import dvlm_gen as gen
import oracle as O
from gpu_util import assert_ok, status, ws_tensor

pytestmark = pytest.mark.gpu
P1_TOL = 2e-4


def _outputs(R, dev):
    return dict(top1_id=torch.full((R,), -1, dtype=torch.int32, device=dev),
                top1_prob=torch.full((R,), -1.0, dtype=torch.float32, device=dev),
                commit=torch.zeros(R, dtype=torch.uint8, device=dev),
                n_commit=torch.zeros(1, dtype=torch.int32, device=dev))


def _compare(a, b):
    assert torch.equal(a["top1_id"], b["top1_id"])
    np.testing.assert_allclose(a["top1_prob"].cpu().numpy(), b["top1_prob"].cpu().numpy(), atol=P1_TOL, rtol=0)
    assert torch.equal(a["commit"], b["commit"])
    assert torch.equal(a["n_commit"], b["n_commit"])


def _case(cuda, seed, R, H, V, apply_rmsnorm, with_commit, with_cert):
    (h_t, h1), (w_t, wv), (h2_t, _) = gen.lmhead_case(seed, R, H, V)
    h, w = h2_t.to(cuda), w_t.to(cuda)
    masked0 = torch.from_numpy((np.arange(R) % 5 != 2).astype(np.uint8)).to(cuda)
    tokens0 = torch.arange(R, dtype=torch.int32, device=cuda) + 7
    kw = {}
    if with_cert:
        # anchors: the oracle's top-1 (id, confidence) of the first hidden set,
        # which the scored set H2 = H1 + 0.5 N(0,1) partly agrees with
        a = O.lm_head_conf(h1.astype(np.float64), wv.astype(np.float64))
        kw = dict(anchor_id=torch.from_numpy(a.top1.astype(np.int32)).to(cuda),
                  anchor_conf=torch.from_numpy(a.p1.astype(np.float32)).to(cuda))
    results = []
    for variant in ("workspace", "static"):
        out = _outputs(R, cuda)
        cert = torch.full((1,), -1, dtype=torch.int32, device=cuda) if with_cert else None
        m = masked0.clone() if with_commit else None
        t = tokens0.clone() if with_commit else None
        st = status(cuda)
        args = dict(R=R, H=H, V=V, apply_rmsnorm=apply_rmsnorm, masked=m, tokens=t, threshold=0.9, status=st,
                    cert_len=cert, **out, **kw)
        if variant == "workspace":
            ws = ws_tensor(dv.lmhead_workspace_size(R, V, H, dv.DVLM_BF16), cuda)
            dv.lmhead_conf_commit(h, w, dtype=dv.DVLM_BF16, workspace=ws, **args)
        else:
            dv.lmhead_conf_commit_static(h, w, **args)
        assert_ok(st)
        results.append((out, cert, m, t))
    (a, ca, ma, ta), (b, cb, mb, tb) = results
    _compare(a, b)
    if with_cert:
        assert int(ca.item()) == int(cb.item())
        # rows masked on entry in descending anchor confidence agree for a while
        assert int(ca.item()) > 0
    if with_commit:
        assert torch.equal(ma, mb) and torch.equal(ta, tb)


def test_static_scratch_matches_workspace_entry_two_calls(cuda):
    # first call: the fused LM-head configuration (R=32, full vocabulary),
    # commit applied in place and the certificate scan
    _case(cuda, 2, 32, 2048, 151936, apply_rmsnorm=0, with_commit=True, with_cert=True)
    # second call straight after, other shape and the final RMSNorm: the
    # shared array still holds the first call's contents
    _case(cuda, 3, 16, 2048, 151936, apply_rmsnorm=1, with_commit=False, with_cert=False)


def test_static_scratch_refuses_sizes_beyond_its_capacity(cuda):
    R, H, V = 64, 256, 1000
    h = torch.zeros((R, H), dtype=torch.bfloat16, device=cuda)
    w = torch.zeros((V, H), dtype=torch.bfloat16, device=cuda)
    with pytest.raises(dv.DvlmError) as ei:
        dv.lmhead_conf_commit_static(h, w, R=R, H=H, V=V, top1_id=torch.zeros(R, dtype=torch.int32, device=cuda))
    assert ei.value.status == 7  # DVLM_ERR_WORKSPACE
    # R <= 32 but a vocabulary of 2^28 rows: its counters alone (4 bytes per
    # 128 rows, 8 MiB) overflow the 6 MiB array on any device.  The weight
    # tensor is real (34 GB, never read: the call is refused on the host
    # before any launch).
    R, H, V = 16, 64, 1 << 28
    h = torch.zeros((R, H), dtype=torch.bfloat16, device=cuda)
    w = torch.empty((V, H), dtype=torch.bfloat16, device=cuda)
    with pytest.raises(dv.DvlmError) as ei:
        dv.lmhead_conf_commit_static(h, w, R=R, H=H, V=V, top1_id=torch.zeros(R, dtype=torch.int32, device=cuda))
    assert ei.value.status == 7
    del w
    torch.cuda.empty_cache()


def test_static_scratch_call_leaves_free_memory_unchanged(cuda):
    R, H, V = 16, 2048, 151936
    (h_t, _), (w_t, _), _ = gen.lmhead_case(5, R, H, V)
    h, w = h_t.to(cuda), w_t.to(cuda)
    out = _outputs(R, cuda)
    st = status(cuda)
    dv.lmhead_conf_commit_static(h, w, R=R, H=H, V=V, status=st, **out)   # warm-up
    assert_ok(st)
    free0, _ = torch.cuda.mem_get_info()
    dv.lmhead_conf_commit_static(h, w, R=R, H=H, V=V, status=st, **out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert_ok(st)
    assert free1 == free0
