"""The kernels' failure path on a real GPU, without faulting or hanging it: a bounded wait
on an mbarrier that nothing completes runs out after a short limit, the kernel records
KDA_ERR_DEVICE_TIMEOUT and returns, and the context stays usable afterwards."""
import pytest
import torch

import chunked_linear_attention_chunk_b200 as kda
from chunked_linear_attention_chunk_b200 import synth
from helpers import G_MIN, NAMES, to_dev

pytestmark = pytest.mark.gpu

TIMEOUT = 6


def test_bounded_wait_reports_timeout_and_context_survives():
    assert kda.kda_device_status() == 0                 # clean word to start from
    kda.kda_selftest_device_timeout(20000)              # 20 ms limit
    assert kda.kda_device_status() == TIMEOUT            # the wait ran out and said so
    assert kda.kda_device_status() == 0                  # reading clears the word
    x = to_dev(synth.make_inputs(1, 70, 2, 64, 64, "bf16", seed=950, s0_std=0.1))
    o, ST = kda.kda_chunk_fwd(*(x[n] for n in NAMES), G_MIN, S0=x["S0"])
    torch.cuda.synchronize()
    assert kda.kda_device_status() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(ST).all()
