"""Failure detection without a GPU fault: every pipeline wait inside the kernels is
bounded. Here a kernel waits on an mbarrier that nothing arrives on, with a short
limit; it must give up, record the timeout in the device error word, and return, so
that smgemm_check() reports SMGEMM_ERR_TIMEOUT and the context stays usable."""
import pytest
import torch

import sm_gemm_b200 as sg

pytestmark = pytest.mark.gpu


def test_abandoned_wait_is_reported_and_context_survives(cuda_device):
    assert sg.check() == sg.OK
    assert sg.selftest_wait_timeout(2000) == sg.OK          # 2 ms limit
    assert sg.check() == sg.ERR_TIMEOUT
    assert sg.check() == sg.OK                              # the record is cleared by the check
    A = torch.ones((256, 256), dtype=torch.bfloat16, device="cuda")
    out = sg.gemm_bf16(A, A, out_dtype=torch.float32)
    assert sg.check() == sg.OK
    assert (out == 256).all()


def test_selftest_rejects_bad_limits(cuda_device):
    assert sg.selftest_wait_timeout(0) == sg.ERR_INVALID_ARG
    assert sg.selftest_wait_timeout(20_000_000) == sg.ERR_INVALID_ARG
