"""Failure detection without a GPU fault: a kernel whose barrier wait is never
satisfied gives up after the library's bounded wait, records a timeout in its
unit's error word and returns; tp_device_status() reports TP_ERR_TIMEOUT once
(then the word is clear), and the context keeps working."""
import pytest
import torch

from helpers import assert_close, f64
from tensor_transformer_layer_tp_b200 import binding as B

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    B.tp_device_status()                          # start from a clear error word
    B.tp_selftest_wait_timeout()
    with pytest.raises(B.TPError) as err:
        B.tp_device_status()
    assert err.value.status == B.TP_ERR_TIMEOUT
    B.tp_device_status()                          # reported once, then cleared
    # the context still computes correctly after the timed-out kernel
    g = torch.Generator().manual_seed(3)
    a = torch.randn(256, 128, generator=g).to(torch.bfloat16)
    b = torch.randn(128, 256, generator=g).to(torch.bfloat16)
    c = torch.empty(256, 256, dtype=torch.float32, device="cuda")
    B.tp_gemm(1, 0, 256, 256, 128, [a.cuda()], 0, [b.cuda()], 0, [c], 1)
    B.tp_device_status()
    assert_close("C", c, f64(a) @ f64(b), tol=1e-5)
