"""The teacher-forced GPU decode checks, run on the CPU against a stand-in
engine: a copy of the oracle whose stored bf16 values are perturbed by about
5e-7 relative before rounding (the CPU model of the GPU's fp32-sum
differences), behind the same calls the checks make (prefill, position,
forward with x_out / advance, set_position, the fused LM head).  This runs
the checks' own logic -- call order, row-to-position mapping, accepted-prefix
bookkeeping, tolerances -- before any GPU does."""
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


@pytest.mark.parametrize("seed", [1, 3])
def test_threshold_check_logic(standin, seed):
    T.test_bf16_reduced_model_threshold_teacher_forced(standin, seed)


@pytest.mark.parametrize("seed", [6, 2])
def test_speculative_check_logic(standin, seed):
    T.test_bf16_reduced_model_spec_teacher_forced(standin, seed)


def test_speculative_check_catches_a_stale_cache_length(standin, monkeypatch):
    """An engine that ignores the accepted-prefix update (keeps L after a
    round) fails the check: its next round runs over the wrong cache slots."""
    monkeypatch.setattr(_Engine, "set_position", lambda self, L, seed, stream=None: None)
    with pytest.raises(AssertionError):
        T.test_bf16_reduced_model_spec_teacher_forced(standin, 6)


def test_threshold_check_catches_a_swapped_row_mapping(standin, monkeypatch):
    """A fused LM head that reports row r's result for position r (no shift)
    fails the threshold check."""
    def unshifted(h, w, **kw):
        _lmhead(h, w, **kw)
        kw["top1_id"][:] = torch.roll(kw["top1_id"], 1)
        kw["top1_prob"][:] = torch.roll(kw["top1_prob"], 1)

    monkeypatch.setattr(dv, "lmhead_conf_commit", unshifted)
    with pytest.raises(AssertionError):
        T.test_bf16_reduced_model_threshold_teacher_forced(standin, 1)
