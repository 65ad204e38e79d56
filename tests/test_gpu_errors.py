"""Failure detection on the GPU without faulting it.

A kernel that waits on a barrier nobody completes must give up after the
wait limit and report SVDQ_ERR_TIMEOUT through the device status word, and
the CUDA context must stay usable afterwards.  A device with another compute
capability must be rejected before anything is launched.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def test_bounded_wait_reports_timeout_and_context_survives():
    from bit_w4a4_quantized_token_b200 import _lib, layer
    from bit_w4a4_quantized_token_b200 import workloads as W

    assert _lib.svdq_device_status(clear=True)[0] == 0
    _lib.svdq_debug_set_wait_limit_ns(50_000_000)          # 50 ms
    try:
        _lib.svdq_debug_timeout_probe()
        st, site = _lib.svdq_device_status(clear=True)
        assert st == _lib.SVDQ_ERR_TIMEOUT
        assert site == 0xEE
        assert _lib.svdq_device_status(clear=True)[0] == 0   # cleared
    finally:
        _lib.svdq_debug_set_wait_limit_ns(0)
    # the context still works: a real layer call succeeds and is correct
    from .parity import check_case

    check_case(W.TINY)
    assert _lib.svdq_device_status(clear=True)[0] == 0


def test_other_capability_rejected_before_launch():
    from bit_w4a4_quantized_token_b200 import _lib, layer
    from bit_w4a4_quantized_token_b200 import workloads as W

    inp = {k: v.cuda() for k, v in W.make_inputs(W.TINY).items()}
    _lib.svdq_debug_override_capability(12, 0)               # an sm_120 part
    try:
        with pytest.raises(_lib.SvdqError) as e:
            layer.pack_weight(inp["R"], inp["lam"], inp["L_down"], inp["L_up"], inp["b"])
        assert e.value.status == _lib.SVDQ_ERR_UNSUPPORTED_DEVICE
    finally:
        _lib.svdq_debug_override_capability(-1)
    layer.pack_weight(inp["R"], inp["lam"], inp["L_down"], inp["L_up"], inp["b"])
    torch.cuda.synchronize()
