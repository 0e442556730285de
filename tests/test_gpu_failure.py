"""Failure detection without a GPU fault: a bounded wait on an mbarrier that
nothing arrives on gives up, reports HCA_ERR_TIMEOUT through the device error
word, and leaves the context usable."""
import pytest
import torch

import compressed_sliding_window_b200 as hca
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    need_gpu()
    assert hca.device_error()[0] == 0
    hca.selftest_bounded_wait(20000)          # 20 ms limit
    code, where = hca.device_error()
    assert code == 4 and where == 900
    # the context still works
    k = torch.randn(1, 256, 512, device="cuda").to(torch.bfloat16)
    s = torch.zeros(1, 256, device="cuda").to(torch.bfloat16)
    ck, _ = hca.compress(k, k, s)
    torch.cuda.synchronize()
    ref = k.float().reshape(1, 2, 128, 512).mean(2)
    assert (ck.float() - ref).abs().max().item() < 1e-2
    assert hca.device_error()[0] == 0
