#!/usr/bin/env python
"""Block-decode tokens/s at batch 1 (B=16) on the Qwen2.5-3B-shaped synthetic
decoder (36 layers, hidden 2048, 16/2 heads of 128, SwiGLU 11008, vocab
151936, random init, LM head x25), context 1280 vision + 64 prompt, 256 new
tokens, threshold 0.9; plus the fused LM-head's HBM GB/s against the measured
peak.

One step = one generation of 256 tokens from the prefilled context (the KV
prefix and weights are resident in HBM; the cache length is rewound before
each step).  Weights (6.2 GB) exceed the 126 MB L2, so no flush is needed
between steps.  Multi-GPU runs are independent replicas (one request per GPU;
the decode step has no data-path collective): value = all ranks' tokens / the
slowest rank's time.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-decode tokens/sec at batch 1 (B=16); fused LM-head+commit HBM GB/s vs peak"
N_VIS, N_PROMPT, N_NEW, BLOCK, TAU, SEED = 1280, 64, 256, 16, 0.9, 4
ROUTE_K = 2   # certificate-guided routing: positions unmasked per step
WORKLOAD = "qwen2.5-3b-shaped block-diffusion decode: 36L h2048 16/2x128 ffn11008 V151936, ctx 1280 vision + 64 prompt, 256 new, B=16, tau 0.9"
PROFILE_DIR = os.path.join(ROOT, "profiles")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # the part's nominal HBM3e bandwidth (context beside the measured copy figure)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", FALLBACK_HBM_GBS), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------- ranks
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return rank, world, local, pg


def barrier(pg):
    if pg is not None:
        pg.barrier()


def max_over_ranks(pg, value: float) -> float:
    """Max of a per-rank float over all ranks (the job's time is the slowest rank's)."""
    if pg is None:
        return value
    import torch
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(tokens_per_rank: int, world: int, max_seconds: float) -> float:
    return tokens_per_rank * world / max_seconds


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if gpu_id:
            cmd += ["-i", gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        sms, maxs, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.file.read().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sms.append(float(f[1]))
                maxs.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.file.name)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s in sms if s > 0.5 * max(sms)] or sms
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(maxs), "reasons": sorted(reasons),
                "power_w_max": max(power), "samples": len(sms)}


def gpu_uuid():
    try:
        import torch
        u = torch.cuda.get_device_properties(torch.cuda.current_device()).uuid
        return f"GPU-{u}"
    except Exception:
        return None


# ----------------------------------------------------------------- algorithmic bytes
def algorithmic_bytes(kind: str, dims, L: int, rows: int = 16, fp8: bool = False) -> float:
    """Bytes a kernel must move per launch: its weights once, its inputs and
    outputs once (bf16 activations).  fp8: the decoder projections' weights
    are E4M3 codes (1 byte each) plus one fp32 scale per weight row."""
    H, I, D, Hq, Hkv, V = dims.hidden, dims.inter, dims.head_dim, dims.n_q_heads, dims.n_kv_heads, dims.vocab
    qkv = (Hq + 2 * Hkv) * D

    def w(n_out, n_in):
        return n_out * n_in + 4 * n_out if fp8 else 2 * n_out * n_in
    if kind == "qkv_gemm":
        return w(qkv, H) + 2 * (rows * H + rows * qkv)
    if kind == "oproj_gemm":
        return w(H, Hq * D) + 2 * (rows * Hq * D + 2 * rows * H)
    if kind == "gateup_gemm":
        return 2 * w(I, H) + 2 * (rows * H + rows * I)
    if kind == "down_gemm":
        return w(H, I) + 2 * (rows * I + 2 * rows * H)
    if kind == "persistent_forward":   # every decoder layer of a forward in one launch
        return dims.n_layers * sum(algorithmic_bytes(k, dims, L, rows, fp8)
                                   for k in ("qkv_gemm", "attention", "oproj_gemm", "gateup_gemm", "down_gemm"))
    if kind == "lm_head":
        return 2 * (V * H + rows * H)
    if kind == "attention":
        return 2 * (2 * Hkv * (L + rows) * D + 2 * rows * Hq * D)
    return 0.0


# Kernel sources (under block_diffusion_vlm_b200/csrc) each recorded DRAM
# traffic depends on: the kernel's own file, the shared device headers and the
# tensor-map setup that fixes its tile boxes (host orchestration in the engine
# does not change what one launch reads and writes).
_COMMON_SOURCES = ["ptx.cuh", "mainloop.cuh", "kernels.h", "tmap.cu"]
TRAFFIC_SOURCES = {
    "qkv_gemm": _COMMON_SOURCES + ["gemm_ws.cu"],
    "oproj_gemm": _COMMON_SOURCES + ["gemm_ws.cu"],
    "gateup_gemm": _COMMON_SOURCES + ["gemm_ws.cu"],
    "down_gemm": _COMMON_SOURCES + ["gemm_ws.cu"],
    "persistent_forward": _COMMON_SOURCES + ["gemm_ws.cu"],
    "lm_head": _COMMON_SOURCES + ["lmhead.cu", "finalize.cuh"],
    "attention": _COMMON_SOURCES + ["attn_split.cu"],
}


def load_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, when it was taken
    on the kernel's current sources; else None."""
    p = os.path.join(PROFILE_DIR, "traffic.json")
    if not os.path.exists(p) or kernel not in TRAFFIC_SOURCES:
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(kernel)
    if not ent:
        return None
    if ent.get("source_hash") != source_hash(TRAFFIC_SOURCES[kernel]):
        return None
    return ent.get("dram_bytes_per_launch")


def source_hash(files=None) -> str:
    """Hash of kernel sources (all of csrc, or the listed files) with comments
    and white space removed: the recorded DRAM traffic stays attached to the
    code it was measured on, and a comment-only edit does not detach it."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_diffusion_vlm_b200", "csrc")
    for n in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, n), encoding="utf-8") as f:
            txt = f.read()
        txt = re.sub(r"/\*.*?\*/", " ", txt, flags=re.S)
        txt = re.sub(r"//[^\n]*", " ", txt)
        txt = re.sub(r"\s+", " ", txt).strip()
        h.update(n.encode())
        h.update(txt.encode())
    return h.hexdigest()[:16]


# ----------------------------------------------------------------- oracle CPU baseline
def cpu_baseline(nfe_per_step: float, layers_timed: int = 4) -> dict:
    """The oracle (fp64 numpy, as it stands) on a bounded sample of the
    workload: one 16-row noisy-block forward at L=1344 through `layers_timed`
    of the 36 decoder layers plus the LM head, with a generator-drawn KV
    prefix; scaled to 36 layers and to the run's NFE per 256 tokens."""
    import numpy as np
    import dvlm_gen as gen
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    dims = gen.QWEN3B
    od = O.dims_from(dims)
    L, n = N_VIS + N_PROMPT, BLOCK
    x = gen.normal(SEED, "cpu.x", (n, dims.hidden), 0.02).astype(np.float64)
    t_layers = []
    for l in range(layers_timed):
        w = {f"{l}.{k}": gen.layer_weight(dims, SEED, l, k)[1].astype(np.float64) for k in gen.layer_weight_names()}
        m = O.OracleModel(od, weights=w, bf16=True, Lmax=L + n)
        m.K[l][:, :L] = gen.normal(SEED, f"cpu.k{l}", (dims.n_kv_heads, L, dims.head_dim))
        m.V[l][:, :L] = gen.normal(SEED, f"cpu.v{l}", (dims.n_kv_heads, L, dims.head_dim))
        t0 = time.perf_counter()
        x = m.layer(l, x, L, 0)
        t_layers.append(time.perf_counter() - t0)
        del w, m
    W = gen.lm_head_weight(dims, SEED)[1].astype(np.float64)
    t0 = time.perf_counter()
    O.lm_head_conf(x, W, O.rms_factor(x)[:, 0])
    t_lm = time.perf_counter() - t0
    del W
    t_fwd = statistics.mean(t_layers) * dims.n_layers + t_lm
    t_step = t_fwd * nfe_per_step
    return {"value": N_NEW / t_step, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{layers_timed} of 36 decoder layers + LM head of one 16-row noisy forward at L=1344 "
                      f"(fp64 numpy), scaled to 36 layers x {nfe_per_step:.1f} forwards per 256 tokens",
            "forward_s": t_fwd}


def workload_nfe() -> float | None:
    p = os.path.join(PROFILE_DIR, "decode_workload.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f).get("nfe_per_256_threshold")
    return None


def forward_bytes(dims, fp8: bool) -> float:
    """Bytes one decode forward streams: every decoder matrix and the LM head
    (the embedding table is only gathered by row); fp8: E4M3 projection codes
    plus their per-row fp32 scales, bf16 LM head."""
    if not fp8:
        return dims.streamed_params() * 2
    H, I, D, Hq = dims.hidden, dims.inter, dims.head_dim, dims.n_q_heads
    per_layer_params = dims.qkv_rows * H + H * Hq * D + 3 * I * H
    per_layer_rows = dims.qkv_rows + H + 2 * I + H
    return dims.n_layers * (per_layer_params + 4 * per_layer_rows) + 2 * dims.vocab * H


def workload_config(args, world: int) -> dict:
    """The `config` object both arms report (same workload, same keys)."""
    c = {"workload": WORKLOAD, "global_batch": world, "seq_len": N_VIS + N_PROMPT + N_NEW,
         "parallelism": f"replicas x{world}", "mode": args.mode,
         "l2": "inputs larger than L2 (6.2 GB of weights streamed per forward)"}
    if getattr(args, "block", BLOCK) != BLOCK:
        c["block"] = args.block
    if getattr(args, "weights", "bf16") != "bf16":
        c["weights"] = "fp8-w8a8 (E4M3 projections, per-row / per-token scales; bf16 LM head)"
    return c


# ----------------------------------------------------------------- arms
def run_reference(args, rank, world):
    if rank != 0:
        return
    nfe = workload_nfe() or float(N_NEW)
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state; warm-up steps are not timed work
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(cpu_baseline(nfe, layers_timed=1))
    elapsed = time.perf_counter() - t0
    v = statistics.mean(c["value"] for c in vals)
    cb = dict(vals[-1])
    cb["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * elapsed / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args, world),
            "cpu_baseline": cb, "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local, pg):
    import torch
    import block_diffusion_vlm_b200 as dv
    import dvlm_gen as gen
    from dvlm_gen.device import DeviceModel, kv_buffers

    import dataclasses
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dims = gen.QWEN3B if args.layers == 36 else dataclasses.replace(gen.QWEN3B, n_layers=args.layers)
    dm = DeviceModel(dims, SEED, device=dev)
    Lmax = N_VIS + N_PROMPT + N_NEW + 32
    kc, vc = kv_buffers(dims, Lmax, device=dev)
    fp8 = args.weights == "fp8"
    cm = dm.fp8_c_model() if fp8 else dm.c_model()
    ws = torch.zeros((dv.engine_workspace_size(cm, Lmax, BLOCK, N_VIS + N_PROMPT) + 3) // 4, dtype=torch.int32,
                     device=dev)
    stream = torch.cuda.Stream(device=dev)
    eng = dv.Engine(cm, kc, vc, Lmax, BLOCK, N_VIS + N_PROMPT, ws, stream=stream)
    for opt in args.option or []:
        name, val = opt.split("=")
        eng.set_option(name, int(val))
    vis_t, vis, ids = gen.decode_context(dims, SEED, N_VIS, N_PROMPT)
    vis_d, ids_d = vis_t.to(dev), torch.from_numpy(ids).to(dev)
    eng.prefill(vis_d, N_VIS, ids_d, N_PROMPT, stream=stream)
    eng.check(stream=stream)
    L0, seed0 = eng.position(stream=stream)
    if args.profile_forwards:
        # profiling case for ncu: eager noisy-block forwards only
        toks = torch.full((BLOCK,), dims.mask_id, dtype=torch.int32, device=dev)
        for _ in range(args.profile_forwards):
            eng.profile_forward(toks, BLOCK, 0, stream=stream)
        eng.check(stream=stream)
        eng.close()
        if rank == 0:
            print(json.dumps({"profile_forwards": args.profile_forwards, "layers": dims.n_layers}), flush=True)
        return
    mode = {"threshold": dv.MODE_THRESHOLD, "spec": dv.MODE_SPEC_LINEAR, "ar": dv.MODE_AR,
            "quad": dv.MODE_SPEC_QUAD, "route": dv.MODE_ROUTE}[args.mode]
    # routing: k = ROUTE_K positions unmasked per step, the 1280 vision rows
    # hidden in TEXT-ONLY passes
    block = getattr(args, "block", BLOCK)
    cfg = dv.DecodeCfg(block, TAU, mode, 1, N_NEW, 1, ROUTE_K, N_VIS)
    out = torch.zeros(N_NEW, dtype=torch.int32, device=dev)

    def step(c=cfg):
        eng.set_position(L0, seed0, stream=stream)
        st = dv.Stats()
        eng.generate(c, out, st, stream=stream)
        return st

    for _ in range(args.warmup):
        step()
    eng.check(stream=stream)
    clocks = ClockSampler(gpu_uuid()) if rank == 0 else None
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(pg)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    stats = [step() for _ in range(args.steps)]
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(pg)
    clk = clocks.stop() if clocks else None
    eng.check(stream=stream)
    secs = max_over_ranks(pg, ev0.elapsed_time(ev1) / 1000.0)
    value = aggregate_throughput(N_NEW * args.steps, world, secs)
    nfe = statistics.mean(s.nfe for s in stats)
    launches = sum(s.n_launches for s in stats)
    hist = [sum(s.commit_hist[i] for s in stats) for i in range(dv.binding.HIST)]

    # end to end through the C ABI from pinned host buffers (prefill included)
    vis_h, ids_h = vis_t.pin_memory(), torch.from_numpy(ids).pin_memory()
    out_h = torch.zeros(N_NEW, dtype=torch.int32).pin_memory()
    e2e_steps = max(1, min(args.steps, 3))
    eng.generate_host(cfg, vis_h, N_VIS, ids_h, N_PROMPT, out_h, stream=stream)
    barrier(pg)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(e2e_steps):
        eng.generate_host(cfg, vis_h, N_VIS, ids_h, N_PROMPT, out_h, stream=stream)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_secs = max_over_ranks(pg, ev0.elapsed_time(ev1) / 1000.0)
    e2e = {"value": aggregate_throughput(N_NEW * e2e_steps, world, e2e_secs), "unit": "tokens/s",
           "h2d_bytes_per_step": N_VIS * dims.hidden * 2 + N_PROMPT * 4, "d2h_bytes_per_step": N_NEW * 4,
           "includes": "H2D of vision+prompt, prefill of 1344 slots, 256-token decode, D2H of tokens"}

    # live per-kernel timing (CUDA events around each launch of one eager forward)
    eng.set_position(L0, seed0, stream=stream)
    toks = torch.full((BLOCK,), dims.mask_id, dtype=torch.int32, device=dev)
    prof = None
    for _ in range(3):
        prof = eng.profile_forward(toks, BLOCK, 0, stream=stream)
    hbm_peak, peak_kind = peaks()
    per = {}
    for k, (ms, cnt) in prof.items():
        if cnt:
            b = algorithmic_bytes(k, dims, L0, fp8=fp8)
            per[k] = {"ms_per_launch": ms / cnt, "launches": cnt, "gbs": b / (ms / cnt * 1e-3) / 1e9,
                      "bytes_per_launch": b}
    dom = max((k for k in per if k != "embed"), key=lambda k: per[k]["ms_per_launch"] * per[k]["launches"])

    def roof(k):
        return {"bound": "hbm", "achieved": per[k]["gbs"], "peak": hbm_peak, "unit": "GB/s",
                "frac": per[k]["gbs"] / hbm_peak, "traffic": load_traffic(k), "kernel": k,
                "peak_source": f"{peak_kind} copy bandwidth", "bytes_per_launch": per[k]["bytes_per_launch"],
                "ms_per_launch": per[k]["ms_per_launch"], "frac_of_nominal": per[k]["gbs"] / NOMINAL_HBM_GBS,
                "nominal_peak": NOMINAL_HBM_GBS}

    fwd_ms = sum(v["ms_per_launch"] * v["launches"] for v in per.values())
    fwd_bytes = forward_bytes(dims, fp8)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000 * secs / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp8-e4m3+bf16" if fp8 else "bf16", "data": "synthetic",
            "config": dict(workload_config(args, world), **({"options": args.option} if args.option else {})),
            "roofline": roof(dom), "lmhead": roof("lm_head") if "lm_head" in per else None,
            "gpu_launches": launches, "clocks": clk, "e2e": e2e,
            "decode": {"nfe_per_step": nfe, "tokens_per_nfe": N_NEW / nfe, "commit_hist": hist,
                       "ms_per_forward": 1000 * secs / args.steps / nfe,
                       "forward_gbs": fwd_bytes / (secs / args.steps / nfe) / 1e9,
                       "forward_frac": fwd_bytes / (secs / args.steps / nfe) / 1e9 / hbm_peak,
                       "forward_frac_of_nominal": fwd_bytes / (secs / args.steps / nfe) / 1e9 / NOMINAL_HBM_GBS},
            "kernels": per, "eager_forward_ms": fwd_ms}

    # short runs of the speculative modes for context (same model and context)
    if args.mode == "threshold" and not args.quick:
        for key, md in (("spec_linear", dv.MODE_SPEC_LINEAR), ("spec_quadratic", dv.MODE_SPEC_QUAD),
                        ("route", dv.MODE_ROUTE)):
            sc = dv.DecodeCfg(BLOCK, TAU, md, 1, N_NEW, 1, ROUTE_K, N_VIS)
            step(sc)
            ev0.record(stream)
            st = step(sc)
            ev1.record(stream)
            torch.cuda.synchronize(dev)
            secs_sc = ev0.elapsed_time(ev1) / 1000.0
            line[key] = {"tokens_per_s": N_NEW / secs_sc, "nfe": st.nfe, "ms_per_forward": 1000 * secs_sc / st.nfe,
                         "accept_hist": list(st.accept_hist)}
            if md == dv.MODE_ROUTE:
                line[key].update(route_k=ROUTE_K, hidden_vision_slots=N_VIS, text_only_passes=st.n_text_passes)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not fp8:
        line["cpu_baseline"] = cpu_baseline(nfe)
    eng.close()
    # compact single-kernel set (decode-shape and long-cache attention, LM
    # head rows, speculative accept) on the same GPU, after the decode
    if rank == 0 and world == 1 and args.mode == "threshold" and not args.quick:
        cases = []
        run_sweep(argparse.Namespace(sweep="compact"), local, sink=cases.append)
        line["sweep"] = [{k: v for k, v in d.items() if k not in ("peak", "peak_source", "timing", "working_set_mb")}
                         for d in cases]
    if rank == 0:
        print(json.dumps(line), flush=True)


def _device_ms_per_call(fn, reps, dev):
    """Device time per call of `fn` (launches on the current stream), from CUDA
    events around a CUDA graph of `reps` calls; eager launches if the capture
    is refused.  Returns (ms, "graph" | "eager")."""
    import torch
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _ in range(3):          # warm-up outside the capture (one-time setup)
            fn()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    mode = "graph"
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        run = g.replay
    except RuntimeError:
        mode = "eager"

        def run():
            for _ in range(reps):
                fn()
    run()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    run()
    e1.record()
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) / reps, mode


def attn_auto_splits(B: int, L: int, nb: int, Hkv: int, sms: int = 148) -> int:
    """Split count of the split-form attention on nb caches of L slots with B
    rows: as many CTAs as fit in one wave on the SMs (one CTA per SM), at most
    one CTA per 128-key chunk and 32 per group, at least 1."""
    n_chunks = (L + B + 127) // 128
    groups = nb * ((B + 15) // 16) * Hkv
    return max(1, min(n_chunks, 32, sms // groups))


def run_sweep(args, local, sink=None):
    """Timings of the single-kernel configurations, one JSON line per case:
    block attention for B in {4, 8, 16, 32} x L in {256, 1024, 4096}, both one
    cache per call (L2-resident after the first call) and 36 distinct caches
    in one batched launch (one per decoder layer; the working set exceeds L2
    at L = 4096); the fused LM head + commit for R in {1, 16, 32, 128} rows
    (its 622 MB of weights exceed L2 on every call).  `sink`: a callable that
    receives each case's dict instead of printing it (the compact set that the
    decode line carries)."""
    import torch
    import block_diffusion_vlm_b200 as dv
    import dvlm_gen as gen
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dims = gen.QWEN3B
    hbm_peak, peak_kind = peaks()
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    def emit(d):
        d.update(peak=hbm_peak, peak_source=f"{peak_kind} copy bandwidth")
        if sink is not None:
            sink(d)
        else:
            print(json.dumps(d), flush=True)

    D, Hq, Hkv = dims.head_dim, dims.n_q_heads, dims.n_kv_heads

    def attn_case(B, L, nb, split_list):
        """Times the attention kernel's cluster form (the decode path) and its
        split form (each S in split_list) on one shape; prints one line per
        configuration."""
        Lmax = (L + B + 7) // 8 * 8
        q, k, v = (t for t, _ in gen.attn_case(1, B, L, Lmax=Lmax, n_batch=nb))
        qd, kd = q.to(dev).contiguous(), k.to(dev).contiguous()
        vt = v.transpose(-1, -2).contiguous().to(dev)
        out = torch.empty_like(qd)
        b = nb * algorithmic_bytes("attention", dims, L, rows=B)
        reps = 20 if nb > 1 else 200

        def call():
            dv.block_attn(qd, out, kd, vt, n_batch=nb, n_rows=B, n_clean=0, L=L, Lmax=Lmax, Hq=Hq,
                          Hkv=Hkv, D=D, scale=1.0 / D ** 0.5, dtype=dv.DVLM_BF16, status=st)

        ms, mode = _device_ms_per_call(call, reps, dev)
        emit({"sweep": "attention", "kernel": "cluster", "B": B, "L": L, "caches_per_launch": nb,
              "us_per_launch": 1000 * ms, "us_per_cache": 1000 * ms / nb,
              "bytes_per_launch": b, "gbs": b / (ms * 1e-3) / 1e9,
              "frac": b / (ms * 1e-3) / 1e9 / hbm_peak,
              "working_set_mb": (kd.numel() + vt.numel()) * 2 / 1e6, "timing": mode})
        for splits in split_list:
            ws = torch.zeros((dv.block_attn_split_workspace_size(nb, B, Hkv, splits) + 3) // 4,
                             dtype=torch.int32, device=dev)

            def call_split():
                dv.block_attn_split(qd, out, kd, vt, n_batch=nb, n_rows=B, n_clean=0, L=L, Lmax=Lmax, Hq=Hq,
                                    Hkv=Hkv, D=D, scale=1.0 / D ** 0.5, splits=splits, workspace=ws,
                                    status=st)

            ms, mode = _device_ms_per_call(call_split, reps, dev)
            emit({"sweep": "attention", "kernel": "split", "splits": splits, "B": B, "L": L,
                  "caches_per_launch": nb, "us_per_launch": 1000 * ms, "us_per_cache": 1000 * ms / nb,
                  "bytes_per_launch": b, "gbs": b / (ms * 1e-3) / 1e9,
                  "frac": b / (ms * 1e-3) / 1e9 / hbm_peak, "timing": mode})
            del ws
        del qd, kd, vt, out

    def auto_splits(B, L, nb):
        return attn_auto_splits(B, L, nb, Hkv)

    if args.sweep == "compact":
        # the decode shape and the bandwidth case, one line each per kernel
        attn_case(BLOCK, N_VIS + N_PROMPT, 1, [4])
        attn_case(BLOCK, 4096, dims.n_layers, [2])
    if args.sweep == "attn_long":
        # the bandwidth case alone: 36 caches of 4096 slots in one launch
        attn_case(BLOCK, 4096, dims.n_layers, [2])
    if args.sweep == "attn_decode":
        # the decode shape (one cache per launch) and the long batched case,
        # split counts around the automatic choice
        attn_case(BLOCK, N_VIS + N_PROMPT, 1, [2, 4, 8, 16])
        attn_case(BLOCK, 4096, dims.n_layers, [1, 2, 3, 4])
    if args.sweep in ("attention", "all"):
        for B in (4, 8, 16, 32):
            for L in (256, 1024, 4096):
                for nb in (1, dims.n_layers):
                    attn_case(B, L, nb, [auto_splits(B, L, nb)])
        # TEXT-ONLY pass of certificate-guided routing at the decode shape: the
        # 1280 vision slots hidden by viewing the cache from slot 1280 (64 spare
        # slots keep the last key chunk inside each head's rows)
        B, L, n_vis = BLOCK, N_VIS + N_PROMPT, N_VIS
        Lmax = (L + B + 7) // 8 * 8 + 64
        q, k, v = (t for t, _ in gen.attn_case(1, B, L, Lmax=Lmax, n_batch=dims.n_layers))
        qd, kd = q.to(dev).contiguous(), k.to(dev).contiguous()
        vt = v.transpose(-1, -2).contiguous().to(dev)
        out = torch.empty_like(qd)
        for hide in (0, n_vis):
            def call():
                dv.block_attn(qd, out, kd[:, :, hide:, :], vt[:, :, :, hide:], n_batch=dims.n_layers, n_rows=B,
                              n_clean=0, L=L - hide, Lmax=Lmax, Hq=Hq, Hkv=Hkv, D=D, scale=1.0 / D ** 0.5,
                              dtype=dv.DVLM_BF16, status=st)

            ms, mode = _device_ms_per_call(call, 20, dev)
            emit({"sweep": "attention_text_only" if hide else "attention_full", "B": B, "L": L, "hidden_slots": hide,
                  "caches_per_launch": dims.n_layers, "us_per_launch": 1000 * ms,
                  "us_per_cache": 1000 * ms / dims.n_layers, "timing": mode})
        del qd, kd, vt, out
    if args.sweep in ("lmhead", "all", "compact"):
        H, V = dims.hidden, dims.vocab
        _, (w_t, _) = gen.lmhead_case(2, 1, H, V, second_set=False)
        wd = w_t.to(dev)
        for R in (1, 16, 32, 128):
            hd = gen.normal_bf16(2, "lm.h1", (R, H))[0].to(dev)
            o = dict(top1_id=torch.empty(R, dtype=torch.int32, device=dev),
                     top1_prob=torch.empty(R, dtype=torch.float32, device=dev),
                     commit=torch.empty(R, dtype=torch.uint8, device=dev),
                     n_commit=torch.empty(1, dtype=torch.int32, device=dev))
            ws = torch.zeros((dv.lmhead_workspace_size(R, V, H, dv.DVLM_BF16) + 3) // 4 + 1, dtype=torch.int32,
                             device=dev)

            def call():
                dv.lmhead_conf_commit(hd, wd, R=R, H=H, V=V, dtype=dv.DVLM_BF16, threshold=TAU, workspace=ws,
                                      status=st, **o)

            for _ in range(3):
                call()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 20
            e0.record()
            for _ in range(reps):
                call()
            e1.record()
            torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1) / reps
            b = algorithmic_bytes("lm_head", dims, 0, rows=R)
            emit({"sweep": "lm_head", "R": R, "us_per_launch": 1000 * ms, "bytes_per_launch": b,
                  "gbs": b / (ms * 1e-3) / 1e9, "frac": b / (ms * 1e-3) / 1e9 / hbm_peak, "timing": "eager"})
        # top-k commit on the LM head's per-row outputs (a latency-bound launch)
        R, k = BLOCK, 4
        p1 = torch.rand(R, device=dev)
        top = torch.zeros(R, dtype=torch.int32, device=dev)
        masked = torch.ones(R, dtype=torch.uint8, device=dev)
        tokens = torch.zeros(R, dtype=torch.int32, device=dev)

        def call():
            dv.topk_commit(p1, top, masked, tokens, R=R, k=k, status=st)

        ms, mode = _device_ms_per_call(call, 200, dev)
        emit({"sweep": "topk_commit", "R": R, "k": k, "us_per_launch": 1000 * ms, "timing": mode})
    if args.sweep in ("spec", "all", "compact"):
        # speculative verify + accept on bf16 logits [b, 16, 151936] (cache
        # lengths updated in place); four input sets in turn, so that b = 8
        # (4 x 38.9 MB) does not run from L2
        V = dims.vocab
        for b in (1, 8):
            sets = []
            for i in range(4):
                logits_t, _, _, draft, _ = gen.spec_case(4 + i, b, BLOCK, V)
                sets.append((logits_t.to(dev), torch.from_numpy(draft).to(dev)))
            acc = torch.zeros(b, dtype=torch.int32, device=dev)
            cl = torch.full((b,), 1 << 30, dtype=torch.int32, device=dev)
            ws = torch.zeros((dv.spec_workspace_size(b, BLOCK, V) + 3) // 4 + 1, dtype=torch.int32, device=dev)
            calls = [0]

            def call():
                lg, dr = sets[calls[0] % 4]
                calls[0] += 1
                dv.spec_verify_accept(draft_ids=dr, b=b, B=BLOCK, V=V, accept_len=acc, verify_logits=lg,
                                      cache_len=cl, workspace=ws, status=st)

            for _ in range(4):
                call()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 64
            e0.record()
            for _ in range(reps):
                call()
            e1.record()
            torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1) / reps
            nbytes = b * BLOCK * V * 2 + 2 * b * BLOCK * 4
            emit({"sweep": "spec_accept", "b": b, "B": BLOCK, "V": V, "us_per_launch": 1000 * ms,
                  "bytes_per_launch": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9,
                  "frac": nbytes / (ms * 1e-3) / 1e9 / hbm_peak, "timing": "eager", "input_sets": 4})
            del sets, ws
    if args.sweep in ("tiny", "all"):
        # the tiny fp32 configuration: 1 layer, hidden 32, 64 context slots,
        # one block of B = 4 to completion (threshold 0.9), graph-driven
        from dvlm_gen.device import DeviceModel, kv_buffers
        td = gen.TINY
        dm = DeviceModel(td, 0, device=dev)
        Lmax = 128
        kc, vc = kv_buffers(td, Lmax, device=dev)
        cm = dm.c_model()
        ws = torch.zeros(dv.engine_workspace_size(cm, Lmax, 16, 128) // 4 + 1, dtype=torch.int32, device=dev)
        eng = dv.Engine(cm, kc, vc, Lmax, 16, 128, ws)
        vis_t, _, ids = gen.decode_context(td, 0, 32, 16, 16)
        eng.prefill(vis_t.to(dev), 32, torch.from_numpy(ids).to(dev), len(ids))
        eng.check()
        L0, seed0 = eng.position()
        cfg = dv.DecodeCfg(4, TAU, dv.MODE_THRESHOLD, 1, 4, 1)
        out = torch.zeros(4, dtype=torch.int32, device=dev)
        for _ in range(3):
            eng.set_position(L0, seed0)
            eng.generate(cfg, out)
        torch.cuda.synchronize(dev)
        reps = 50
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        total = 0.0
        for _ in range(reps):
            stt = dv.Stats()
            eng.set_position(L0, seed0)
            e0.record()
            eng.generate(cfg, out, stt)
            e1.record()
            torch.cuda.synchronize(dev)
            total += e0.elapsed_time(e1)
        eng.check()
        ms = total / reps
        emit({"sweep": "tiny_step", "B": 4, "context": L0, "nfe": stt.nfe, "ms_per_block": ms,
              "us_per_forward": 1000 * ms / max(stt.nfe, 1), "tokens_per_s": 4 / (ms * 1e-3),
              "timing": "graph replay per forward, host-driven block loop"})
        eng.close()
    torch.cuda.synchronize(dev)
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} after the sweep")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--mode", choices=["threshold", "spec", "ar", "quad", "route"], default="threshold")
    ap.add_argument("--block", type=int, default=BLOCK,
                    help="block size B of the timed decode (the benchmarked configuration: 16)")
    ap.add_argument("--option", action="append", default=None, metavar="NAME=VALUE",
                    help="engine launch knob (dvlm_engine_set_option), e.g. attn_split=8; repeatable")
    ap.add_argument("--weights", choices=["bf16", "fp8"], default="bf16",
                    help="fp8: the W8A8 decoder (E4M3 projections quantised from the same bf16 weights)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true", help="skip the extra speculative-mode run")
    ap.add_argument("--layers", type=int, default=36, help="decoder depth (36 = the benchmarked model)")
    ap.add_argument("--profile-forwards", type=int, default=0,
                    help="profiling case: run this many eager forwards after prefill and exit")
    ap.add_argument("--sweep", choices=["attention", "attn_decode", "attn_long", "compact", "lmhead", "spec", "tiny", "all"], default=None,
                    help="time the single-kernel configurations (one JSON line per case) instead of the decode")
    args = ap.parse_args()
    rank, world, local, pg = dist_setup()
    try:
        if args.sweep:
            if rank == 0:
                run_sweep(args, local)
        elif args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local, pg)
    finally:
        if pg is not None:
            pg.destroy_process_group()


if __name__ == "__main__":
    main()
