"""Bounded waits end in a status, not a fault; argument errors raise."""
import pytest
import torch

from moe_gemm_absmax_b200 import w8a8

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    assert w8a8.get_device_error() == (w8a8.OK, 0)
    w8a8.debug_wait_timeout(1_000_000)          # 1 ms on a barrier nobody arrives at
    rc, site = w8a8.get_device_error()
    assert rc == w8a8.ERR_TIMEOUT and (site >> 16) == 9
    assert w8a8.get_device_error() == (w8a8.OK, 0)   # read clears it
    x = torch.randn(4, 64, device="cuda").to(torch.bfloat16)
    q, s = w8a8.quant_act(x)
    torch.cuda.synchronize()
    assert q.shape == (4, 64)


def test_no_device_error_after_normal_work():
    x = torch.randn(300, 1024, device="cuda").to(torch.bfloat16)
    w = torch.randn(512, 1024, device="cuda") * 0.02
    qw, sw = w8a8.quant_rows_f32(w)
    w8a8.linear(x, qw, sw)
    w8a8.linear(x[:3], qw, sw)
    assert w8a8.get_device_error() == (w8a8.OK, 0)


def test_argument_errors_raise():
    x = torch.zeros(4, 60, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(w8a8.W8A8Error) as e:
        w8a8.quant_act(x)
    assert e.value.status == w8a8.ERR_INVALID_ARG
    with pytest.raises(TypeError):
        w8a8.quant_act(torch.zeros(4, 64, device="cuda"))
