"""Failure detection without a GPU fault: a device-side wait that can never be
satisfied gives up after its budget, reports DVLM_ERR_TIMEOUT through the
status word and returns; the context stays usable afterwards."""
import pytest
import torch

import block_diffusion_vlm_b200 as dv
from block_diffusion_vlm_b200 import binding

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda):
    st = torch.zeros(1, dtype=torch.int32, device=cuda)
    gave_up = torch.zeros(1, dtype=torch.int32, device=cuda)
    binding.selftest_wait_timeout(2_000_000, st, gave_up)      # ~1 ms at boost clock
    torch.cuda.synchronize()
    assert int(st.item()) == 5 and int(gave_up.item()) == 1   # DVLM_ERR_TIMEOUT
    # the context is intact: a normal kernel runs and gives the right answer
    x = torch.arange(1024, device=cuda, dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2


def test_selftest_argument_validation(cuda):
    with pytest.raises(dv.DvlmError):
        binding.selftest_wait_timeout(0, torch.zeros(1, dtype=torch.int32, device=cuda),
                                      torch.zeros(1, dtype=torch.int32, device=cuda))
