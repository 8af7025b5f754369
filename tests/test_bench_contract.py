"""bench.py's own arm assembles the benchmark's JSON line from measured
values; here the measuring parts (CUDA, the engine, the device model) are
replaced by stand-ins with fixed timings, so that the line's assembly runs on
the CPU and its contract keys are checked before any GPU run."""
import importlib
import json
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class _Event:
    def __init__(self, enable_timing=False):
        pass

    def record(self, stream=None):
        pass

    def elapsed_time(self, other):
        return 100.0                                   # ms between any two events


class _Stream:
    cuda_stream = 0

    def __init__(self, device=None):
        pass


class _FakeEngine:
    def __init__(self, *a, **k):
        pass

    def prefill(self, *a, **k):
        pass

    def check(self, stream=None):
        pass

    def position(self, stream=None):
        return 1344, 7

    def set_position(self, L, seed, stream=None):
        pass

    def generate(self, cfg, out, st=None, stream=None):
        if st is not None:
            st.nfe, st.n_tokens, st.n_launches = 71, 256, 12954
            st.commit_hist[1], st.commit_hist[15] = 70, 1

    def generate_host(self, *a, **k):
        pass

    def profile_forward(self, *a, **k):
        ms = {"embed": 0.01, "qkv_gemm": 0.47, "attention": 0.56, "oproj_gemm": 0.43, "gateup_gemm": 0.90,
              "down_gemm": 0.68, "lm_head": 0.107}
        return {k: (v, 1 if k in ("embed", "lm_head") else 36) for k, v in ms.items()}

    def close(self):
        pass


class _FakeDeviceModel:
    def __init__(self, *a, **k):
        pass

    def c_model(self):
        return None


def test_default_arm_line_has_the_contract_keys(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    import block_diffusion_vlm_b200 as dv
    import dvlm_gen as gen
    import dvlm_gen.device as gdev
    real_device = torch.device
    monkeypatch.setattr(torch, "device", lambda *a, **k: real_device("cpu"))
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "Stream", _Stream)
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(dv, "Engine", _FakeEngine)
    monkeypatch.setattr(dv, "engine_workspace_size", lambda *a: 64)
    monkeypatch.setattr(gdev, "DeviceModel", _FakeDeviceModel)
    monkeypatch.setattr(gdev, "kv_buffers", lambda *a, **k: (None, None))
    monkeypatch.setattr(bench, "gpu_uuid", lambda: None)
    args = bench.argparse.Namespace(steps=5, warmup=3, mode="threshold", quick=True, no_cpu_baseline=True,
                                    layers=36, profile_forwards=0, impl="ours", gpus=1, sweep=None, weights="bf16", option=None)
    bench.run_ours(args, 0, 1, 0, None)
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["value"] == pytest.approx(256 * 5 / 0.1) and d["ms_per_step"] == pytest.approx(20.0)
    assert d["n_gpus"] == 1 and d["dtype"] == "bf16" and d["higher_is_better"] is True
    assert "workload" in d["config"] and d["gpu_launches"] == 5 * 12954
    r = d["roofline"]
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(r) and r["kernel"] == "gateup_gemm"
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"]) and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(bench.algorithmic_bytes("gateup_gemm", gen.QWEN3B, 1344) /
                                          (0.90 / 36 * 1e-3) / 1e9)
    assert d["lmhead"]["kernel"] == "lm_head"
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 1280 * 2048 * 2 + 64 * 4 and e["d2h_bytes_per_step"] == 256 * 4
    dec = d["decode"]
    assert dec["nfe_per_step"] == 71
    assert dec["forward_gbs"] == pytest.approx(6_171_394_048 / (0.1 / 5 / 71) / 1e9)
    assert isinstance(d["clocks"], dict) and "reasons" in d["clocks"]


class _Graph:
    def replay(self):
        pass


class _GraphCtx:
    def __init__(self, g):
        pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def test_sweep_prints_one_line_per_case(monkeypatch, capsys):
    """`bench.py --sweep all` with the entry points, CUDA graphs and large
    draws replaced by stand-ins: the attention cases (12 shapes, one cache
    and 36 caches per launch, plus the TEXT-ONLY pair), the four LM-head
    row counts and the speculative accept at b = 1 and 8 each print one line
    with their bytes, GB/s and fraction; the tiny step prints its block time."""
    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    import block_diffusion_vlm_b200 as dv
    import dvlm_gen as gen
    real_device = torch.device
    monkeypatch.setattr(torch, "device", lambda *a, **k: real_device("cpu"))
    for name, fake in [("set_device", lambda *a, **k: None), ("synchronize", lambda *a, **k: None),
                       ("Stream", _Stream), ("Event", _Event), ("CUDAGraph", _Graph), ("graph", _GraphCtx),
                       ("current_stream", lambda *a, **k: _Stream()), ("stream", lambda s: _GraphCtx(s))]:
        monkeypatch.setattr(torch.cuda, name, fake)
    monkeypatch.setattr(_Stream, "wait_stream", lambda self, other: None, raising=False)
    calls = {"attn": [], "lm": []}
    monkeypatch.setattr(dv, "block_attn", lambda q, out, k, v, **kw: calls["attn"].append(kw))
    monkeypatch.setattr(dv, "block_attn_split", lambda q, out, k, v, **kw: calls["attn"].append(kw))
    monkeypatch.setattr(dv, "block_attn_split_workspace_size", lambda *a: 64)
    monkeypatch.setattr(dv, "lmhead_conf_commit", lambda h, w, **kw: calls["lm"].append(kw["R"]))
    monkeypatch.setattr(dv, "lmhead_workspace_size", lambda *a: 64)
    monkeypatch.setattr(dv, "topk_commit", lambda *a, **kw: calls["lm"].append(("topk", kw["R"], kw["k"])))
    small = torch.zeros(2, 2, 2, 2, dtype=torch.bfloat16)
    monkeypatch.setattr(gen, "attn_case", lambda *a, **k: ((small, None),) * 3)
    monkeypatch.setattr(gen, "lmhead_case", lambda *a, **k: ((small, None), (small, None)))
    monkeypatch.setattr(gen, "normal_bf16", lambda *a, **k: (small, None))
    import numpy as np
    import dvlm_gen.device as gdev
    monkeypatch.setattr(gen, "spec_case", lambda *a, **k: (small, None, None, np.zeros((1, 16), np.int32), None))
    monkeypatch.setattr(dv, "spec_verify_accept", lambda **kw: calls["spec"].append(kw["b"]))
    monkeypatch.setattr(dv, "spec_workspace_size", lambda *a: 64)
    monkeypatch.setattr(gdev, "DeviceModel", _FakeDeviceModel)
    monkeypatch.setattr(gdev, "kv_buffers", lambda *a, **k: (None, None))
    monkeypatch.setattr(gen, "decode_context", lambda *a, **k: (small, None, np.zeros(16, np.int32)))
    monkeypatch.setattr(dv, "Engine", _FakeEngine)
    monkeypatch.setattr(dv, "engine_workspace_size", lambda *a: 64)
    calls["spec"] = []
    args = bench.argparse.Namespace(sweep="all")
    bench.run_sweep(args, 0)
    lines = [json.loads(ln) for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    attn = [d for d in lines if d["sweep"] == "attention"]
    assert len(attn) == 4 * 3 * 2 * 2
    for kern in ("cluster", "split"):
        assert {(d["B"], d["L"], d["caches_per_launch"]) for d in attn if d["kernel"] == kern} == \
            {(B, L, nb) for B in (4, 8, 16, 32) for L in (256, 1024, 4096) for nb in (1, 36)}
    for d in attn:
        assert d["bytes_per_launch"] == d["caches_per_launch"] * bench.algorithmic_bytes("attention", gen.QWEN3B,
                                                                                         d["L"], rows=d["B"])
        assert d["frac"] == pytest.approx(d["gbs"] / d["peak"]) and d["timing"] == "graph"
    text = {d["sweep"]: d for d in lines if d["sweep"].startswith("attention_")}
    assert set(text) == {"attention_full", "attention_text_only"}
    assert text["attention_text_only"]["hidden_slots"] == 1280 and text["attention_full"]["hidden_slots"] == 0
    hidden = [kw for kw in calls["attn"] if kw["L"] == 1344 - 1280]
    assert hidden and all(kw["Lmax"] >= 1344 + 16 + 64 and kw["n_batch"] == 36 for kw in hidden)
    lm = [d for d in lines if d["sweep"] == "lm_head"]
    assert [d["R"] for d in lm] == [1, 16, 32, 128]
    assert all(d["bytes_per_launch"] == bench.algorithmic_bytes("lm_head", gen.QWEN3B, 0, rows=d["R"]) for d in lm)
    tk = [d for d in lines if d["sweep"] == "topk_commit"]
    assert len(tk) == 1 and tk[0]["R"] == 16 and tk[0]["us_per_launch"] > 0
    sp = [d for d in lines if d["sweep"] == "spec_accept"]
    assert [d["b"] for d in sp] == [1, 8] and set(calls["spec"]) == {1, 8}
    assert all(d["bytes_per_launch"] == d["b"] * 16 * 151936 * 2 + 2 * d["b"] * 16 * 4 for d in sp)
    tiny = [d for d in lines if d["sweep"] == "tiny_step"]
    assert len(tiny) == 1 and tiny[0]["B"] == 4 and tiny[0]["ms_per_block"] > 0


def test_full_line_carries_modes_and_compact_sweep(monkeypatch, capsys):
    """Without --quick the decode line also times the speculative modes and
    routing on the same engine, and carries the compact single-kernel set
    (run_sweep in collecting mode, here a stand-in)."""
    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    import block_diffusion_vlm_b200 as dv
    import dvlm_gen.device as gdev
    real_device = torch.device
    monkeypatch.setattr(torch, "device", lambda *a, **k: real_device("cpu"))
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "Stream", _Stream)
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(dv, "Engine", _FakeEngine)
    monkeypatch.setattr(dv, "engine_workspace_size", lambda *a: 64)
    monkeypatch.setattr(gdev, "DeviceModel", _FakeDeviceModel)
    monkeypatch.setattr(gdev, "kv_buffers", lambda *a, **k: (None, None))
    monkeypatch.setattr(bench, "gpu_uuid", lambda: None)
    seen = []

    def fake_sweep(a, local, sink=None):
        seen.append(a.sweep)
        sink({"sweep": "lm_head", "R": 16, "us_per_launch": 100.0, "peak": 1.0, "timing": "eager"})

    monkeypatch.setattr(bench, "run_sweep", fake_sweep)
    args = bench.argparse.Namespace(steps=5, warmup=3, mode="threshold", quick=False, no_cpu_baseline=True,
                                    layers=36, profile_forwards=0, impl="ours", gpus=1, sweep=None, weights="bf16",
                                    option=None)
    bench.run_ours(args, 0, 1, 0, None)
    d = json.loads([ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")][0])
    assert seen == ["compact"]
    assert d["sweep"] == [{"sweep": "lm_head", "R": 16, "us_per_launch": 100.0}]
    for key in ("spec_linear", "spec_quadratic", "route"):
        assert d[key]["nfe"] == 71 and d[key]["tokens_per_s"] > 0
    assert d["route"]["route_k"] == bench.ROUTE_K and d["route"]["hidden_vision_slots"] == 1280


def test_attention_auto_splits_fill_one_wave():
    """The sweep's split count for the split-form attention: one wave of CTAs
    (groups x S <= 148 whenever a split of 1 fits), no CTA without a 128-key
    chunk, and the largest such S."""
    import importlib
    bench = importlib.import_module("bench")
    for B in (4, 8, 16, 32):
        for L in (256, 1024, 1344, 4096):
            for nb in (1, 36):
                S = bench.attn_auto_splits(B, L, nb, 2)
                groups = nb * ((B + 15) // 16) * 2
                n_chunks = (L + B + 127) // 128
                assert 1 <= S <= min(32, n_chunks) or (S == 1 and n_chunks >= 1)
                if groups <= 148:
                    assert groups * S <= 148
                    assert S == min(32, n_chunks) or groups * (S + 1) > 148
    assert bench.attn_auto_splits(16, 4096, 36, 2) == 2   # the bandwidth case: 144 CTAs
    assert bench.attn_auto_splits(16, 1344, 1, 2) == 11   # the decode shape: one CTA per chunk
