"""B200-native (sm_100a) block-diffusion decode step for Fast-dVLM-style
block-diffusion VLM decoders.

The work runs in ``libdvlm.so`` (hand-written CUDA kernels behind the C ABI of
include/dvlm.h); this package is its ctypes binding.  Build the library with
``python -m block_diffusion_vlm_b200.build``.
"""
from .binding import (DVLM_BF16, DVLM_FP32, DVLM_FP8_W8A8, MODE_AR, MODE_ROUTE, MODE_SPEC_QUAD, MODE_SPEC_LINEAR, MODE_THRESHOLD, DecodeCfg, DvlmError,
                      Engine, Model, Stats, block_attn, block_attn_paged, block_attn_split,
                      block_attn_split_workspace_size, declared_symbols, divergence_first_commit, engine_trace_record_bytes,
                      engine_workspace_size, lib,
                      lmhead_conf_commit, lmhead_conf_commit_static, lmhead_workspace_size, make_model,
                      quantize_rows_e4m3, spec_verify_accept, spec_workspace_size, status_string, topk_commit)

__all__ = ["DVLM_BF16", "DVLM_FP32", "DVLM_FP8_W8A8", "MODE_AR", "MODE_ROUTE", "MODE_SPEC_QUAD", "MODE_SPEC_LINEAR", "MODE_THRESHOLD", "DecodeCfg", "DvlmError",
           "Engine", "Model", "Stats", "block_attn", "block_attn_paged", "block_attn_split",
           "block_attn_split_workspace_size", "declared_symbols", "divergence_first_commit",
           "engine_trace_record_bytes", "engine_workspace_size", "lib",
           "lmhead_conf_commit", "lmhead_conf_commit_static", "lmhead_workspace_size", "make_model",
           "quantize_rows_e4m3", "spec_verify_accept",
           "spec_workspace_size", "status_string", "topk_commit"]
