"""CPU oracle of the block-diffusion decode step.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` leg of ``bench.py``; never by the product path.
"""
from .dvlm_oracle import *  # noqa: F401,F403
from .dvlm_oracle import (bf16_round, rms_factor, rmsnorm, rope, silu, mask_from_roles,
                          dense_masked_attention, block_attention, Conf,
                          confidence_from_logits, lm_head_conf, threshold_commit,
                          certificate_scan, prefix_accept, Dims, OracleModel, DecodeTrace,
                          prefill, decode_threshold, decode_spec_linear, decode_ar,
                          weights_from_generator, dims_from)
