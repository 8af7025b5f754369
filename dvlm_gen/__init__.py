"""Seeded synthetic inputs for the block-diffusion decode step.

This module is the one piece shared by the CPU oracle and the CUDA path.  It
holds random draws and the model/workload shapes only -- none of the decoding
method's arithmetic (no norms, products, softmax, argmax, masks or commits).

Every tensor is drawn from its own stream: numpy's PCG64 seeded with
``SeedSequence([seed, crc32(name)])``, so any tensor can be regenerated alone
(the oracle regenerates one layer at a time; the GPU side uploads layer by
layer).  bf16 tensors are drawn in fp32 and converted with PyTorch's
round-to-nearest-even cast; the returned fp32 array holds exactly the bf16
values, so the oracle (fp64) and the kernels (bf16) see identical inputs.

Workload recipes follow the five synthetic configurations of the method's
decode step (tiny fp32 step, block attention, fused LM head + commit,
speculative accept, full Qwen2.5-3B-shaped decode).
"""
from __future__ import annotations

import dataclasses
import zlib

import numpy as np

__all__ = [
    "ModelDims", "TINY", "QWEN3B", "stream", "normal", "normal_bf16",
    "uniform_ids", "layer_weight_names", "layer_weight", "lm_head_weight",
    "embedding_weight", "decode_context", "attn_case", "lmhead_case",
    "spec_case", "bf16_tensor",
]


@dataclasses.dataclass(frozen=True)
class ModelDims:
    """Decoder shape. Weight matrices are [out, in] row-major."""
    n_layers: int
    hidden: int          # H
    n_q_heads: int       # Hq
    n_kv_heads: int      # Hkv
    head_dim: int        # D
    inter: int           # I (SwiGLU width)
    vocab: int           # V
    rope_base: float = 10000.0
    eps: float = 1e-6
    w_std: float = 0.02
    lm_scale: float = 25.0
    dtype: str = "bf16"  # storage dtype of weights/activations: "bf16" or "f32"

    @property
    def mask_id(self) -> int:
        """[MASK] is the last vocabulary id (it stays predictable)."""
        return self.vocab - 1

    @property
    def qkv_rows(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    def n_params(self) -> int:
        H, I, V = self.hidden, self.inter, self.vocab
        per_layer = self.qkv_rows * H + H * self.n_q_heads * self.head_dim + 3 * I * H
        return self.n_layers * per_layer + 2 * V * H

    def streamed_params(self) -> int:
        """Parameters a forward pass reads in full: every decoder matrix and
        the LM head; the embedding table is only gathered by row."""
        return self.n_params() - self.vocab * self.hidden


# Tiny fp32 model of the first configuration: LM head scaled x40.
TINY = ModelDims(n_layers=1, hidden=32, n_q_heads=2, n_kv_heads=1, head_dim=16,
                 inter=64, vocab=256, lm_scale=40.0, dtype="f32")
# Qwen2.5-3B-shaped language decoder (36 layers, 2048 hidden, 16/2 heads).
QWEN3B = ModelDims(n_layers=36, hidden=2048, n_q_heads=16, n_kv_heads=2,
                   head_dim=128, inter=11008, vocab=151936, lm_scale=25.0,
                   dtype="bf16")


def stream(seed: int, name: str) -> np.random.Generator:
    """Independent generator for one named tensor."""
    ss = np.random.SeedSequence([int(seed) & 0xFFFFFFFF, zlib.crc32(name.encode())])
    return np.random.Generator(np.random.PCG64(ss))


def normal(seed: int, name: str, shape, std: float = 1.0) -> np.ndarray:
    """fp32 N(0, std^2) draws."""
    a = stream(seed, name).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def bf16_tensor(a: np.ndarray):
    """fp32 array -> torch.bfloat16 CPU tensor (round to nearest even)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def normal_bf16(seed: int, name: str, shape, std: float = 1.0):
    """(torch.bfloat16 tensor, fp32 numpy array holding the same values)."""
    t = bf16_tensor(normal(seed, name, shape, std))
    return t, t.float().numpy()


def uniform_ids(seed: int, name: str, n: int, high: int) -> np.ndarray:
    """int32 ids uniform on [0, high)."""
    return stream(seed, name).integers(0, high, size=n, dtype=np.int64).astype(np.int32)


def _cast(a: np.ndarray, dtype: str):
    """Storage form of a drawn tensor: (device-ready tensor, exact fp32 values)."""
    if dtype == "bf16":
        t = bf16_tensor(a)
        return t, t.float().numpy()
    import torch
    return torch.from_numpy(a), a


def layer_weight_names():
    return ("wq", "wk", "wv", "wo", "wg", "wu", "wd")


def layer_weight(dims: ModelDims, seed: int, layer: int, name: str):
    """One decoder-layer matrix [out, in]: (storage tensor, fp32 values)."""
    H, D, I = dims.hidden, dims.head_dim, dims.inter
    shapes = {
        "wq": (dims.n_q_heads * D, H), "wk": (dims.n_kv_heads * D, H),
        "wv": (dims.n_kv_heads * D, H), "wo": (H, dims.n_q_heads * D),
        "wg": (I, H), "wu": (I, H), "wd": (H, I),
    }
    a = normal(seed, f"layer{layer}.{name}", shapes[name], dims.w_std)
    return _cast(a, dims.dtype)


def lm_head_weight(dims: ModelDims, seed: int):
    """Untied LM head [V, H] ~ N(0, (w_std * lm_scale)^2)."""
    a = normal(seed, "lm_head", (dims.vocab, dims.hidden), dims.w_std * dims.lm_scale)
    return _cast(a, dims.dtype)


def embedding_weight(dims: ModelDims, seed: int):
    """Token embedding table [V, H] ~ N(0, w_std^2)."""
    a = normal(seed, "embed", (dims.vocab, dims.hidden), dims.w_std)
    return _cast(a, dims.dtype)


def decode_context(dims: ModelDims, seed: int, n_vision: int, n_prompt: int,
                   n_committed: int = 0):
    """Context for a decode run: vision embeddings N(0,1) [n_vision, H] and
    text ids (prompt then already-committed ids) uniform on [0, V-1)."""
    vis = normal(seed, "vision", (n_vision, dims.hidden), 1.0)
    vis_t, vis_v = _cast(vis, dims.dtype)
    ids = np.concatenate([
        uniform_ids(seed, "prompt", n_prompt, dims.vocab - 1),
        uniform_ids(seed, "committed", n_committed, dims.vocab - 1),
    ]).astype(np.int32)
    return vis_t, vis_v, ids


def attn_case(seed: int, n_rows: int, L: int, Hq: int = 16, Hkv: int = 2,
              D: int = 128, Lmax: int | None = None, n_batch: int = 1,
              dtype: str = "bf16"):
    """Block-attention inputs: q [nb, n_rows, Hq, D] and K/V caches
    [nb, Hkv, Lmax, D] holding L+n_rows valid slots, all N(0,1)."""
    Lmax = Lmax or (L + n_rows)
    q = normal(seed, "attn.q", (n_batch, n_rows, Hq, D))
    k = normal(seed, "attn.k", (n_batch, Hkv, Lmax, D))
    v = normal(seed, "attn.v", (n_batch, Hkv, Lmax, D))
    return tuple(_cast(a, dtype) for a in (q, k, v))


def lmhead_case(seed: int, R: int, H: int = 2048, V: int = 151936,
                w_std: float = 0.02, lm_scale: float = 25.0,
                dtype: str = "bf16", second_set: bool = True):
    """Fused LM-head inputs: hidden H1 [R, H] N(0,1), W [V, H], and a second
    hidden set H2 = H1 + 0.5 * N(0,1) for the certificate check."""
    h1 = normal(seed, "lm.h1", (R, H))
    w = normal(seed, "lm.w", (V, H), w_std * lm_scale)
    out = [_cast(h1, dtype), _cast(w, dtype)]
    if second_set:
        out.append(_cast(h1 + normal(seed, "lm.h2noise", (R, H), 0.5), dtype))
    return tuple(out)


def spec_case(seed: int, b: int, B: int = 16, V: int = 151936,
              logit_std: float = 22.6, planted: float = 200.0):
    """Speculative accept inputs with a planted top-1.

    Logits [b, B, V] are N(0, logit_std^2) (the spread of the scaled LM head's
    logits) with one entry per row raised to ``planted`` (well above any draw),
    so that row's top-1 id is known by construction.  Draft ids equal the
    planted id for positions < k_b and a different id from there on, with
    k_b uniform on [0, B].  Returns (logits bf16 tensor, logits fp32 values,
    planted ids [b, B], draft ids [b, B], k [b])."""
    rng = stream(seed, "spec")
    logits = normal(seed, "spec.logits", (b, B, V), logit_std)
    top = rng.integers(0, V, size=(b, B)).astype(np.int32)
    for i in range(b):
        for j in range(B):
            logits[i, j, top[i, j]] = planted
    k = rng.integers(0, B + 1, size=b).astype(np.int32)
    shift = rng.integers(1, V, size=(b, B)).astype(np.int32)
    draft = top.copy()
    for i in range(b):
        draft[i, k[i]:] = (top[i, k[i]:] + shift[i, k[i]:]) % V
    t, vals = _cast(logits, "bf16")
    return t, vals, top, draft, k
