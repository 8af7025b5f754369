"""ctypes binding of ``libdvlm.so`` (the C ABI declared in include/dvlm.h).

Argument marshalling only: every step of the decode path runs in the
library's CUDA kernels.  Tensors are passed as raw device pointers taken
from torch tensors (PyTorch provides device memory and streams); streams are
``torch.cuda.Stream`` objects or raw handles.  A non-zero status raises
``DvlmError``.  There is no fallback: if the library is missing, loading
fails loudly.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_PATH = os.path.join(PKG, "libdvlm.so")
HEADER = os.path.join(ROOT, "include", "dvlm.h")

DVLM_BF16, DVLM_FP32, DVLM_FP8_W8A8 = 0, 1, 2
MODE_THRESHOLD, MODE_SPEC_LINEAR, MODE_AR, MODE_SPEC_QUAD, MODE_ROUTE = 0, 1, 2, 3, 4
HIST = 17

_lib: Optional[ctypes.CDLL] = None


class DvlmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load libdvlm.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m block_diffusion_vlm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        _declare(L)
        _lib = L
    return _lib


def declared_symbols() -> list[str]:
    """Names of the entry points declared in include/dvlm.h."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"^DVLM_API\s+[\w\s\*]*?\b(dvlm_\w+)\s*\(", text, flags=re.M)


class Model(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("hidden", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("inter", ctypes.c_int),
                ("vocab", ctypes.c_int), ("mask_id", ctypes.c_int), ("rope_base", ctypes.c_float),
                ("eps", ctypes.c_float), ("dtype", ctypes.c_int), ("embed", ctypes.c_void_p),
                ("wqkv", ctypes.c_void_p), ("wo", ctypes.c_void_p), ("wgate", ctypes.c_void_p),
                ("wup", ctypes.c_void_p), ("wdown", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("sqkv", ctypes.c_void_p), ("so", ctypes.c_void_p), ("sgate", ctypes.c_void_p),
                ("sup", ctypes.c_void_p), ("sdown", ctypes.c_void_p)]


class DecodeCfg(ctypes.Structure):
    _fields_ = [("block_size", ctypes.c_int), ("threshold", ctypes.c_float), ("mode", ctypes.c_int),
                ("ar_seed", ctypes.c_int), ("max_new_tokens", ctypes.c_int), ("use_graphs", ctypes.c_int),
                ("route_k", ctypes.c_int), ("route_n_vis", ctypes.c_int)]


class Stats(ctypes.Structure):
    _fields_ = [("nfe", ctypes.c_int64), ("n_tokens", ctypes.c_int64), ("n_iters", ctypes.c_int64),
                ("n_rounds", ctypes.c_int64), ("commit_hist", ctypes.c_int64 * HIST),
                ("accept_hist", ctypes.c_int64 * HIST), ("n_launches", ctypes.c_int64),
                ("n_text_passes", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {"nfe": self.nfe, "n_tokens": self.n_tokens, "n_iters": self.n_iters, "n_rounds": self.n_rounds,
                "commit_hist": list(self.commit_hist), "accept_hist": list(self.accept_hist),
                "n_launches": self.n_launches, "n_text_passes": self.n_text_passes}


_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


def _declare(L: ctypes.CDLL) -> None:
    sigs = {
        "dvlm_status_string": (ctypes.c_char_p, [_i]),
        "dvlm_version": (_i, []),
        "dvlm_device_sm_count": (_i, []),
        "dvlm_block_attn": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _vp]),
        "dvlm_lmhead_workspace_size": (_sz, [_i, _i, _i, _i]),
        "dvlm_lmhead_conf_commit": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _vp, _f, _vp, _vp, _vp, _vp,
                                         _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
        "dvlm_lmhead_conf_commit_static": (_i, [_vp, _vp, _i, _i, _i, _i, _f, _vp, _vp, _f, _vp, _vp, _vp, _vp,
                                                _vp, _vp, _vp, _vp, _vp]),
        "dvlm_topk_commit": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp, _vp, _vp, _vp]),
        "dvlm_divergence_first_commit": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _vp, _vp, _vp]),
        "dvlm_spec_workspace_size": (_sz, [_i, _i, _i]),
        "dvlm_spec_verify_accept": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _vp,
                                         _sz, _vp, _vp]),
        "dvlm_engine_workspace_size": (_sz, [ctypes.POINTER(Model), _i, _i, _i]),
        "dvlm_engine_create": (_i, [ctypes.POINTER(Model), _vp, _vp, _i, _i, _i, _vp, _sz, _vp,
                                    ctypes.POINTER(_vp)]),
        "dvlm_engine_destroy": (_i, [_vp]),
        "dvlm_prefill": (_i, [_vp, _vp, _i, _vp, _i, _vp]),
        "dvlm_decode_block": (_i, [_vp, ctypes.POINTER(DecodeCfg), _vp, ctypes.POINTER(ctypes.c_int32),
                                   ctypes.POINTER(Stats), _vp]),
        "dvlm_generate": (_i, [_vp, ctypes.POINTER(DecodeCfg), _vp, ctypes.POINTER(Stats), _vp]),
        "dvlm_generate_host": (_i, [_vp, ctypes.POINTER(DecodeCfg), _vp, _i, _vp, _i, _vp, ctypes.POINTER(Stats),
                                    _vp]),
        "dvlm_engine_get_position": (_i, [_vp, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32), _vp]),
        "dvlm_engine_set_position": (_i, [_vp, ctypes.c_int32, ctypes.c_int32, _vp]),
        "dvlm_engine_check": (_i, [_vp, _vp]),
        "dvlm_forward": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp]),
        "dvlm_forward_text_only": (_i, [_vp, _vp, _vp, _i, _i, _vp, _vp]),
        "dvlm_engine_set_option": (_i, [_vp, ctypes.c_char_p, _i]),
        "dvlm_engine_get_option": (_i, [_vp, ctypes.c_char_p]),
        "dvlm_selftest_wait_timeout": (_i, [ctypes.c_longlong, _vp, _vp, _vp]),
        "dvlm_profile_forward": (_i, [_vp, _vp, _vp, _i, _i, _i, ctypes.POINTER(ctypes.c_float),
                                      ctypes.POINTER(_i), _vp]),
        "dvlm_engine_trace_record_bytes": (_sz, [ctypes.POINTER(Model)]),
        "dvlm_quantize_rows_e4m3": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
        "dvlm_forward_quad": (_i, [_vp, _vp, _i, _vp, _vp]),
        "dvlm_engine_set_paged": (_i, [_vp, _vp, _vp, _vp, _i, _i]),
        "dvlm_block_attn_split_workspace_size": (_sz, [_i, _i, _i, _i]),
        "dvlm_block_attn_split": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _sz, _vp,
                                       _vp]),
        "dvlm_block_attn_paged": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp, _vp]),
        "dvlm_engine_set_trace": (_i, [_vp, _vp, _sz, _vp]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args


def status_string(status: int) -> str:
    return lib().dvlm_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise DvlmError(status, where)


def ptr(t) -> Optional[int]:
    """Device (or host) address of a tensor, None for None."""
    if t is None:
        return None
    return t.data_ptr()


def stream_handle(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ---------------------------------------------------------------- kernels
def block_attn(q, out, k_cache, v_cache, *, n_batch, n_rows, n_clean, L, Lmax, Hq, Hkv, D, scale, dtype,
               status=None, stream=None) -> None:
    _check(lib().dvlm_block_attn(ptr(q), ptr(out), ptr(k_cache), ptr(v_cache), n_batch, n_rows, n_clean, L, Lmax,
                                 Hq, Hkv, D, float(scale), dtype, ptr(status), stream_handle(stream)),
           "dvlm_block_attn")


def block_attn_split_workspace_size(n_batch: int, n_rows: int, Hkv: int, splits: int) -> int:
    return int(lib().dvlm_block_attn_split_workspace_size(n_batch, n_rows, Hkv, splits))


def block_attn_split(q, out, k_cache, v_cache, *, n_batch, n_rows, n_clean, L, Lmax, Hq, Hkv, D, scale, splits,
                     workspace, status=None, stream=None) -> None:
    """Split-CTA block attention (dvlm_block_attn_split)."""
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().dvlm_block_attn_split(ptr(q), ptr(out), ptr(k_cache), ptr(v_cache), n_batch, n_rows, n_clean, L,
                                       Lmax, Hq, Hkv, D, float(scale), int(splits), ptr(workspace), ws_bytes,
                                       ptr(status), stream_handle(stream)),
           "dvlm_block_attn_split")


def block_attn_paged(q, out, k_pages, v_pages, block_table, lens, *, n_batch, n_rows, n_clean, n_pages, max_pages,
                     Hq, Hkv, D, scale, status=None, stream=None) -> None:
    """Attention over paged KV caches (dvlm_block_attn_paged)."""
    _check(lib().dvlm_block_attn_paged(ptr(q), ptr(out), ptr(k_pages), ptr(v_pages), ptr(block_table), ptr(lens),
                                       n_batch, n_rows, n_clean, n_pages, max_pages, Hq, Hkv, D, float(scale),
                                       ptr(status), stream_handle(stream)),
           "dvlm_block_attn_paged")


def lmhead_workspace_size(R: int, V: int, H: int, dtype: int) -> int:
    return int(lib().dvlm_lmhead_workspace_size(R, V, H, dtype))


def lmhead_conf_commit(hidden, w, *, R, H, V, dtype, apply_rmsnorm=0, eps=1e-6, masked=None, tokens=None,
                       threshold=0.9, top1_id=None, top1_prob=None, commit=None, n_commit=None, anchor_id=None,
                       anchor_conf=None, cert_len=None, workspace=None, status=None, stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().dvlm_lmhead_conf_commit(ptr(hidden), ptr(w), R, H, V, dtype, int(apply_rmsnorm), float(eps),
                                         ptr(masked), ptr(tokens), float(threshold), ptr(top1_id), ptr(top1_prob),
                                         ptr(commit), ptr(n_commit), ptr(anchor_id), ptr(anchor_conf),
                                         ptr(cert_len), ptr(workspace), ws_bytes, ptr(status),
                                         stream_handle(stream)),
           "dvlm_lmhead_conf_commit")


def lmhead_conf_commit_static(hidden, w, *, R, H, V, apply_rmsnorm=0, eps=1e-6, masked=None, tokens=None,
                              threshold=0.9, top1_id=None, top1_prob=None, commit=None, n_commit=None,
                              anchor_id=None, anchor_conf=None, cert_len=None, status=None, stream=None) -> None:
    """bf16 fused LM head with the library's fixed internal scratch (no workspace argument)."""
    _check(lib().dvlm_lmhead_conf_commit_static(ptr(hidden), ptr(w), R, H, V, int(apply_rmsnorm), float(eps),
                                                ptr(masked), ptr(tokens), float(threshold), ptr(top1_id),
                                                ptr(top1_prob), ptr(commit), ptr(n_commit), ptr(anchor_id),
                                                ptr(anchor_conf), ptr(cert_len), ptr(status), stream_handle(stream)),
           "dvlm_lmhead_conf_commit_static")


def topk_commit(top1_prob, top1_id, masked, tokens, *, R, k, commit=None, n_commit=None, status=None,
                stream=None) -> None:
    """Commit the k most confident masked rows in place (dvlm_topk_commit)."""
    _check(lib().dvlm_topk_commit(ptr(top1_prob), ptr(top1_id), ptr(masked), ptr(tokens), int(R), int(k),
                                  ptr(commit), ptr(n_commit), ptr(status), stream_handle(stream)),
           "dvlm_topk_commit")


def divergence_first_commit(full_prob, full_id, text_id, masked, tokens, *, R, k, commit=None, n_commit=None,
                            status=None, stream=None) -> None:
    """Commit k masked rows in place, TEXT-ONLY/FULL divergent rows first
    (dvlm_divergence_first_commit)."""
    _check(lib().dvlm_divergence_first_commit(ptr(full_prob), ptr(full_id), ptr(text_id), ptr(masked), ptr(tokens),
                                              int(R), int(k), ptr(commit), ptr(n_commit), ptr(status),
                                              stream_handle(stream)),
           "dvlm_divergence_first_commit")


def spec_workspace_size(b: int, B: int, V: int) -> int:
    return int(lib().dvlm_spec_workspace_size(b, B, V))


def spec_verify_accept(*, draft_ids, b, B, V, accept_len, verify_logits=None, verify_ids=None, cache_len=None,
                       poison_tail=0, k_cache=None, v_cache=None, n_layers=0, Hkv=0, D=0, Lmax=0, workspace=None,
                       status=None, stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().dvlm_spec_verify_accept(ptr(verify_logits), ptr(verify_ids), ptr(draft_ids), b, B, V,
                                         ptr(accept_len), ptr(cache_len), int(poison_tail), ptr(k_cache),
                                         ptr(v_cache), n_layers, Hkv, D, Lmax, ptr(workspace), ws_bytes,
                                         ptr(status), stream_handle(stream)),
           "dvlm_spec_verify_accept")


def quantize_rows_e4m3(a, codes, scales, *, rows, K, stream=None) -> None:
    """Per-row FP8 E4M3 codes and scales of a bf16 matrix (dvlm_quantize_rows_e4m3)."""
    _check(lib().dvlm_quantize_rows_e4m3(ptr(a), int(rows), int(K), ptr(codes), ptr(scales), stream_handle(stream)),
           "dvlm_quantize_rows_e4m3")


def selftest_wait_timeout(budget_cycles: int, status, gave_up, stream=None) -> None:
    _check(lib().dvlm_selftest_wait_timeout(int(budget_cycles), ptr(status), ptr(gave_up), stream_handle(stream)),
           "dvlm_selftest_wait_timeout")


# ---------------------------------------------------------------- engine
def make_model(dims, *, embed, wqkv, wo, wgate, wup, wdown, lm_head, dtype, scales=None) -> Model:
    """scales: (sqkv, so, sgate, sup, sdown) per-row fp32 scales of an FP8 W8A8 model."""
    sc = scales or (None,) * 5
    return Model(dims.n_layers, dims.hidden, dims.n_q_heads, dims.n_kv_heads, dims.head_dim, dims.inter,
                 dims.vocab, dims.mask_id, float(dims.rope_base), float(dims.eps), dtype, ptr(embed), ptr(wqkv),
                 ptr(wo), ptr(wgate), ptr(wup), ptr(wdown), ptr(lm_head), *(ptr(t) for t in sc))


def engine_workspace_size(model: Model, Lmax: int, max_block: int, max_ctx: int) -> int:
    return int(lib().dvlm_engine_workspace_size(ctypes.byref(model), Lmax, max_block, max_ctx))


def engine_trace_record_bytes(model: Model) -> int:
    """Bytes of one forward-trace record (dvlm_engine_trace_record_bytes)."""
    return int(lib().dvlm_engine_trace_record_bytes(ctypes.byref(model)))


class Engine:
    """Decode engine over caller-owned device buffers (see dvlm_engine_create)."""

    def __init__(self, model: Model, k_cache, v_cache, Lmax: int, max_block: int, max_ctx: int, workspace,
                 stream=None):
        self._keep = (model, k_cache, v_cache, workspace)
        h = ctypes.c_void_p()
        ws_bytes = workspace.numel() * workspace.element_size()
        _check(lib().dvlm_engine_create(ctypes.byref(model), ptr(k_cache), ptr(v_cache), Lmax, max_block, max_ctx,
                                        ptr(workspace), ws_bytes, stream_handle(stream), ctypes.byref(h)),
               "dvlm_engine_create")
        self.h = h

    def close(self) -> None:
        if getattr(self, "h", None):
            _check(lib().dvlm_engine_destroy(self.h), "dvlm_engine_destroy")
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def prefill(self, vision, n_vision: int, ids, n_ids: int, stream=None) -> None:
        _check(lib().dvlm_prefill(self.h, ptr(vision), n_vision, ptr(ids), n_ids, stream_handle(stream)),
               "dvlm_prefill")

    def decode_block(self, cfg: DecodeCfg, out_tokens, stats: Optional[Stats] = None, stream=None) -> int:
        n = ctypes.c_int32(0)
        _check(lib().dvlm_decode_block(self.h, ctypes.byref(cfg), ptr(out_tokens), ctypes.byref(n),
                                       ctypes.byref(stats) if stats is not None else None, stream_handle(stream)),
               "dvlm_decode_block")
        return n.value

    def generate(self, cfg: DecodeCfg, out_tokens, stats: Optional[Stats] = None, stream=None) -> None:
        _check(lib().dvlm_generate(self.h, ctypes.byref(cfg), ptr(out_tokens),
                                   ctypes.byref(stats) if stats is not None else None, stream_handle(stream)),
               "dvlm_generate")

    def generate_host(self, cfg: DecodeCfg, vision_host, n_vision: int, ids_host, n_ids: int, out_host,
                      stats: Optional[Stats] = None, stream=None) -> None:
        _check(lib().dvlm_generate_host(self.h, ctypes.byref(cfg), ptr(vision_host), n_vision, ptr(ids_host), n_ids,
                                        ptr(out_host), ctypes.byref(stats) if stats is not None else None,
                                        stream_handle(stream)),
               "dvlm_generate_host")

    def position(self, stream=None) -> tuple[int, int]:
        L, s = ctypes.c_int32(0), ctypes.c_int32(0)
        _check(lib().dvlm_engine_get_position(self.h, ctypes.byref(L), ctypes.byref(s), stream_handle(stream)),
               "dvlm_engine_get_position")
        return L.value, s.value

    def set_position(self, L: int, seed: int, stream=None) -> None:
        _check(lib().dvlm_engine_set_position(self.h, L, seed, stream_handle(stream)), "dvlm_engine_set_position")

    def check(self, stream=None) -> None:
        _check(lib().dvlm_engine_check(self.h, stream_handle(stream)), "dvlm_engine_check (device status)")

    def set_option(self, name: str, value: int) -> None:
        _check(lib().dvlm_engine_set_option(self.h, name.encode(), int(value)), f"dvlm_engine_set_option({name})")

    def get_option(self, name: str) -> int:
        return int(lib().dvlm_engine_get_option(self.h, name.encode()))

    def set_paged(self, k_pages, v_pages, block_table, n_pages: int, max_pages: int) -> None:
        """Switch to a paged KV cache (dvlm_engine_set_paged)."""
        self._keep = self._keep + (k_pages, v_pages, block_table)
        _check(lib().dvlm_engine_set_paged(self.h, ptr(k_pages), ptr(v_pages), ptr(block_table), int(n_pages),
                                           int(max_pages)),
               "dvlm_engine_set_paged")

    def forward_quad(self, draft, B: int, x_out, stream=None) -> None:
        """The fused draft+verify forward alone (dvlm_forward_quad)."""
        _check(lib().dvlm_forward_quad(self.h, ptr(draft), int(B), ptr(x_out), stream_handle(stream)),
               "dvlm_forward_quad")

    def set_trace(self, buf, count) -> None:
        """Record every decode-driver forward into buf (device tensor), counting
        records in count (device int32); buf=None clears (dvlm_engine_set_trace)."""
        nbytes = buf.numel() * buf.element_size() if buf is not None else 0
        _check(lib().dvlm_engine_set_trace(self.h, ptr(buf), nbytes, ptr(count) if buf is not None else None),
               "dvlm_engine_set_trace")

    KERNEL_KINDS = ("embed", "qkv_gemm", "attention", "oproj_gemm", "gateup_gemm", "down_gemm", "lm_head",
                    "persistent_forward")

    def profile_forward(self, tokens, n_rows: int, n_clean: int, *, masked=None, with_lm_head=True,
                        stream=None) -> dict:
        """Per-kernel-class device time (ms, summed over layers) and launch count of one eager forward."""
        ms = (ctypes.c_float * len(self.KERNEL_KINDS))()
        cnt = (ctypes.c_int * len(self.KERNEL_KINDS))()
        _check(lib().dvlm_profile_forward(self.h, ptr(tokens), ptr(masked), n_rows, n_clean, int(with_lm_head), ms,
                                          cnt, stream_handle(stream)),
               "dvlm_profile_forward")
        return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(self.KERNEL_KINDS)}

    def forward_text_only(self, n_rows: int, n_hidden: int, *, tokens, masked=None, x_out=None,
                          stream=None) -> None:
        """Noisy pass with cache slots 0..n_hidden-1 hidden from attention (dvlm_forward_text_only)."""
        _check(lib().dvlm_forward_text_only(self.h, ptr(tokens), ptr(masked), n_rows, n_hidden, ptr(x_out),
                                            stream_handle(stream)),
               "dvlm_forward_text_only")

    def forward(self, n_rows: int, n_clean: int, n_layers: int, *, x_in=None, tokens=None, masked=None,
                first_layer: int = 0, advance: bool = False, x_out=None, stream=None) -> None:
        _check(lib().dvlm_forward(self.h, ptr(x_in), ptr(tokens), ptr(masked), n_rows, n_clean, first_layer,
                                  n_layers, int(advance), ptr(x_out), stream_handle(stream)),
               "dvlm_forward")
