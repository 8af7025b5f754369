"""Upload generator-drawn synthetic models and caches to a torch device in
the C ABI's layouts (stacked per-layer weights, value cache transposed).

Pure data movement: draws come from ``dvlm_gen``; nothing here computes any
part of the decoding method.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (ModelDims, embedding_weight, layer_weight, lm_head_weight)


def torch_dtype(dims: ModelDims):
    return torch.bfloat16 if dims.dtype == "bf16" else torch.float32


class DeviceModel:
    """Device weights of a synthetic model plus the dims they were drawn with."""

    def __init__(self, dims: ModelDims, seed: int, device="cuda", layers=None):
        self.dims = dims
        self.seed = seed
        dt = torch_dtype(dims)
        nl = dims.n_layers
        H, I, D = dims.hidden, dims.inter, dims.head_dim
        HD = dims.n_q_heads * D
        self.embed = embedding_weight(dims, seed)[0].to(device)
        self.lm_head = lm_head_weight(dims, seed)[0].to(device)
        self.wqkv = torch.empty((nl, dims.qkv_rows, H), dtype=dt, device=device)
        self.wo = torch.empty((nl, H, HD), dtype=dt, device=device)
        self.wgate = torch.empty((nl, I, H), dtype=dt, device=device)
        self.wup = torch.empty((nl, I, H), dtype=dt, device=device)
        self.wdown = torch.empty((nl, H, I), dtype=dt, device=device)
        for l in range(nl) if layers is None else layers:
            q, k, v = (layer_weight(dims, seed, l, n)[0] for n in ("wq", "wk", "wv"))
            self.wqkv[l].copy_(torch.cat([q, k, v], dim=0))
            self.wo[l].copy_(layer_weight(dims, seed, l, "wo")[0])
            self.wgate[l].copy_(layer_weight(dims, seed, l, "wg")[0])
            self.wup[l].copy_(layer_weight(dims, seed, l, "wu")[0])
            self.wdown[l].copy_(layer_weight(dims, seed, l, "wd")[0])

    def c_model(self):
        from block_diffusion_vlm_b200 import DVLM_BF16, DVLM_FP32, make_model
        return make_model(self.dims, embed=self.embed, wqkv=self.wqkv, wo=self.wo, wgate=self.wgate,
                          wup=self.wup, wdown=self.wdown, lm_head=self.lm_head,
                          dtype=DVLM_BF16 if self.dims.dtype == "bf16" else DVLM_FP32)


    def fp8_c_model(self):
        """The W8A8 version of this model: each projection's E4M3 codes and
        per-row scales, quantised from these bf16 weights on the device by the
        library (dvlm_quantize_rows_e4m3); embedding and LM head stay bf16."""
        from block_diffusion_vlm_b200 import DVLM_FP8_W8A8, make_model, quantize_rows_e4m3
        q = {}
        for name in ("wqkv", "wo", "wgate", "wup", "wdown"):
            w = getattr(self, name)
            codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
            scales = torch.empty(w.shape[:2], dtype=torch.float32, device=w.device)
            quantize_rows_e4m3(w, codes, scales, rows=w.shape[0] * w.shape[1], K=w.shape[2])
            q[name] = (codes, scales)
        self.fp8 = q
        return make_model(self.dims, embed=self.embed, wqkv=q["wqkv"][0], wo=q["wo"][0], wgate=q["wgate"][0],
                          wup=q["wup"][0], wdown=q["wdown"][0], lm_head=self.lm_head, dtype=DVLM_FP8_W8A8,
                          scales=tuple(q[n][1] for n in ("wqkv", "wo", "wgate", "wup", "wdown")))


def kv_buffers(dims: ModelDims, Lmax: int, device="cuda", n_batch: int = 1):
    """Zeroed K cache [n_layers, n_batch, Hkv, Lmax, D] and transposed V cache
    [n_layers, n_batch, Hkv, D, Lmax]."""
    dt = torch_dtype(dims)
    k = torch.zeros((dims.n_layers, n_batch, dims.n_kv_heads, Lmax, dims.head_dim), dtype=dt, device=device)
    v = torch.zeros((dims.n_layers, n_batch, dims.n_kv_heads, dims.head_dim, Lmax), dtype=dt, device=device)
    return k, v


def as_f64(t) -> np.ndarray:
    """Exact float64 copy of a (bf16 / fp32) tensor."""
    return t.detach().float().cpu().numpy().astype(np.float64)
