"""GPU checks whose logic can run on the CPU against stand-ins.

The teacher-forced routing checks run against a stand-in engine: a copy of
the oracle whose stored bf16 values are perturbed by about 5e-7 relative
before rounding (the CPU model of the GPU's fp32-sum differences), behind the
same calls the checks make (prefill, position, forward with x_out / advance,
TEXT-ONLY forward, set_position, the fused LM head).  This runs the checks'
own logic -- call order, row-to-position mapping, tolerances -- before any
GPU does.  (The threshold and speculative decode checks replay the engine's
own trace; tests/test_decode_replay_logic.py covers their logic.)  The TEXT-ONLY attention
check runs against a stand-in that addresses memory as the kernel does, from
the base pointers it is given, so the offset cache views are shown to reach
exactly the intended slots and to stay inside their buffers."""
import numpy as np
import pytest
import torch

import block_diffusion_vlm_b200 as dv
import dvlm_gen as gen
import dvlm_gen.device as gdev
import oracle as O
import test_gpu_decode as T


class _Dims:
    def __init__(self, dims, seed):
        self.dims, self.seed = dims, seed


class _DeviceModel:
    def __init__(self, dims, seed, device=None):
        self.dims, self.seed = dims, seed
        self.lm_head = ("lm_head", dims, seed)

    def c_model(self):
        return _Dims(self.dims, self.seed)


_WEIGHTS = {}


def _weights(dims, seed):
    if (dims, seed) not in _WEIGHTS:
        _WEIGHTS[(dims, seed)] = O.weights_from_generator(gen, dims, seed)
    return _WEIGHTS[(dims, seed)]


class _Engine:
    def __init__(self, cm, kc, vc, Lmax, max_block, max_ctx, ws, stream=None):
        self.d = cm.dims
        self.m = O.OracleModel(O.dims_from(cm.dims), weights=_weights(cm.dims, cm.seed), bf16=True, Lmax=Lmax)
        rng = np.random.default_rng(1000 + cm.seed)
        self.m.rnd = lambda x: O.bf16_round(np.asarray(x) * (1 + 2.0 ** -21 * rng.standard_normal(np.shape(x))))
        self.seed = None

    def prefill(self, vis, n_vis, ids, n_ids, stream=None):
        self.seed = O.prefill(self.m, vis.float().numpy().astype(np.float64), ids.numpy())

    def position(self, stream=None):
        return self.m.L, self.seed

    def set_position(self, L, seed, stream=None):
        self.m.L, self.seed = L, seed

    def forward(self, n_rows, n_clean, n_layers, *, tokens=None, x_out=None, advance=False, **kw):
        assert n_layers == self.d.n_layers and tokens is not None
        x = self.m.forward(self.m.embed(tokens.numpy()), self.m.L, n_clean=n_clean)
        if x_out is not None:
            x_out[:n_rows] = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
        if advance:
            self.m.L += n_rows

    def forward_text_only(self, n_rows, n_hidden, *, tokens=None, x_out=None, **kw):
        assert tokens is not None and n_hidden % 8 == 0 and n_hidden <= self.m.L
        x = self.m.forward(self.m.embed(tokens.numpy()), self.m.L, n_clean=0, hide=n_hidden)
        if x_out is not None:
            x_out[:n_rows] = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)

    def check(self, stream=None):
        pass

    def close(self):
        pass


def _lmhead(h, w, *, R, H, V, dtype, apply_rmsnorm=0, top1_id=None, top1_prob=None, workspace=None, status=None,
            **kw):
    _, dims, seed = w
    x = h[:R].float().numpy().astype(np.float64)
    c = O.lm_head_conf(x, _weights(dims, seed)["lm_head"], O.rms_factor(x)[:, 0] if apply_rmsnorm else None)
    top1_id[:R] = torch.from_numpy(c.top1.astype(np.int32))
    top1_prob[:R] = torch.from_numpy(c.p1.astype(np.float32))


@pytest.fixture()
def standin(monkeypatch):
    real_device = torch.device
    monkeypatch.setattr(torch, "device", lambda *a, **k: real_device("cpu"))
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(T, "DeviceModel", _DeviceModel)
    monkeypatch.setattr(gdev, "DeviceModel", _DeviceModel)
    monkeypatch.setattr(T, "kv_buffers", lambda *a, **k: (None, None))
    monkeypatch.setattr(dv, "Engine", _Engine)
    monkeypatch.setattr(dv, "engine_workspace_size", lambda *a: 64)
    monkeypatch.setattr(dv, "lmhead_workspace_size", lambda *a: 64)
    monkeypatch.setattr(dv, "lmhead_conf_commit", _lmhead)
    return torch.device("cpu")


def _attn_by_kernel_addressing(q, out, k, v, *, n_batch, n_rows, n_clean, L, Lmax, Hq, Hkv, D, scale, dtype,
                               status=None, **kw):
    """Block attention computed from raw storage with the kernel's
    addressing: K row (b*Hkv + g)*Lmax + key from the K base pointer, V^T
    element ((b*Hkv + g)*D + d)*Lmax + key from the V base pointer, keys
    0..L+n_rows-1, every 64-key box the kernel requests inside the storage."""
    kflat = torch.empty(0, dtype=k.dtype).set_(k.untyped_storage()).float()
    vflat = torch.empty(0, dtype=v.dtype).set_(v.untyped_storage()).float()
    ko, vo = k.storage_offset(), v.storage_offset()
    n_keys = L + n_rows
    boxed = -(-n_keys // 64) * 64
    qn = q.float().numpy().astype(np.float64)
    res = np.zeros(qn.shape)
    for b in range(n_batch):
        for g in range(Hkv):
            row0 = (b * Hkv + g) * Lmax
            assert ko + (row0 + boxed) * D <= kflat.numel()
            assert vo + ((b * Hkv + g) * D + D - 1) * Lmax + boxed <= vflat.numel()
            K = kflat[ko + row0 * D: ko + (row0 + n_keys) * D].reshape(n_keys, D).numpy().astype(np.float64)
            base = vo + (b * Hkv + g) * D * Lmax
            V = np.stack([vflat[base + d * Lmax: base + d * Lmax + n_keys].numpy() for d in range(D)],
                         axis=1).astype(np.float64)
            heads = slice(g * (Hq // Hkv), (g + 1) * (Hq // Hkv))
            res[b][:, heads] = O.block_attention(qn[b][:, heads], K[None], V[None], L, n_clean, scale)
    out.copy_(torch.from_numpy(res.astype(np.float32)).to(out.dtype))


@pytest.mark.parametrize("case", [(1280, 1344, 16, 0, 1), (64, 300, 16, 0, 2), (8, 100, 4, 0, 1),
                                  (64, 64, 16, 0, 1), (128, 500, 12, 5, 1)])
def test_text_only_offset_views_reach_the_intended_slots(standin, monkeypatch, case):
    import test_gpu_attn as TA
    monkeypatch.setattr(dv, "block_attn", _attn_by_kernel_addressing)
    monkeypatch.setattr(TA, "assert_ok", lambda st: None)
    TA.test_text_only_pass_through_offset_cache_views(standin, *case)


def test_text_only_check_catches_unhidden_vision_slots(standin, monkeypatch):
    """Reading from the cache's own base (the vision slots not hidden) fails
    the TEXT-ONLY check."""
    import test_gpu_attn as TA

    def from_base(q, out, k, v, **kw):
        full_k = torch.empty(0, dtype=k.dtype).set_(k.untyped_storage())
        full_v = torch.empty(0, dtype=v.dtype).set_(v.untyped_storage())
        n_vis = k.storage_offset() // kw["D"]
        kw["L"] += n_vis
        _attn_by_kernel_addressing(q, out, full_k, full_v, **kw)

    monkeypatch.setattr(dv, "block_attn", from_base)
    monkeypatch.setattr(TA, "assert_ok", lambda st: None)
    with pytest.raises(AssertionError):
        TA.test_text_only_pass_through_offset_cache_views(standin, 64, 300, 16, 0, 1)


def _lmhead_full(h, w, *, R, H, V, dtype, masked=None, tokens=None, threshold=0.9, top1_id=None, top1_prob=None,
                 anchor_id=None, anchor_conf=None, cert_len=None, workspace=None, status=None, **kw):
    """Fused LM head stand-in with the header's contract: outputs, in-place
    commit only when tokens is given, certificate over the rows masked on
    entry."""
    x = h[:R].float().numpy().astype(np.float64)
    c = O.lm_head_conf(x, w.float().numpy().astype(np.float64))
    p1 = c.p1.astype(np.float32)
    if top1_id is not None:
        top1_id[:R] = torch.from_numpy(c.top1.astype(np.int32))
    if top1_prob is not None:
        top1_prob[:R] = torch.from_numpy(p1)
    part = masked.numpy().astype(bool) if masked is not None else np.ones(R, dtype=bool)
    if cert_len is not None:
        cert_len[0] = O.certificate_scan(anchor_id.numpy(), anchor_conf.numpy().astype(np.float64), c.top1, part)
    if tokens is not None:
        for r in O.threshold_commit(p1.astype(np.float64), part, threshold):
            tokens[r], masked[r] = int(c.top1[r]), 0


def _commit_standin(order_fn):
    def run(p, ids, *rest, R, k, commit=None, n_commit=None, status=None, **kw):
        other = rest[0] if len(rest) == 3 else None
        masked, tokens = rest[-2], rest[-1]
        part = masked.numpy().astype(bool)
        rows = order_fn(p.numpy().astype(np.float64), ids.numpy(), None if other is None else other.numpy(), part, k)
        for r in rows:
            tokens[r], masked[r] = int(ids[r]), 0
    return run


def test_routing_step_check_logic(standin, monkeypatch):
    import test_gpu_topk as TK
    monkeypatch.setattr(dv, "lmhead_conf_commit", _lmhead_full)
    monkeypatch.setattr(dv, "topk_commit", _commit_standin(lambda p, ids, other, part, k: O.topk_commit(p, part, k)))
    monkeypatch.setattr(dv, "divergence_first_commit", _commit_standin(
        lambda p, ids, other, part, k: O.divergence_first_order(ids, p, other, part)[:k]))
    monkeypatch.setattr(TK, "assert_ok", lambda st: None)
    TK.test_routing_step_decisions_on_the_lm_head_outputs(standin)


def test_routing_decode_check_logic(standin):
    T.test_bf16_reduced_model_routing_teacher_forced(standin)


def test_routing_decode_check_catches_a_text_pass_that_sees_the_vision_rows(standin, monkeypatch):
    monkeypatch.setattr(_Engine, "forward_text_only",
                        lambda self, n_rows, n_hidden, **kw: _Engine.forward(self, n_rows, 0, self.d.n_layers, **kw))
    with pytest.raises(AssertionError):
        T.test_bf16_reduced_model_routing_teacher_forced(standin)
