"""The quantizer entry point that allocates nothing (svdq_quantize_act_noalloc).

It serves callers that cannot allocate device memory themselves -- code that
only receives input and output buffers from a host framework, or that must
keep cudaMalloc's device-wide synchronisation off its hot path -- by using a
built-in device array as the K-split workspace.  Its results must equal those
of svdq_quantize_act, on consecutive calls (the built-in array keeps the
previous call's contents).  The no-alloc calls are made with the split's
partials forced through the workspace, so that the built-in array is the
memory they go through.

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test.
"""
import pytest
import torch

from bit_w4a4_quantized_token_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _lowrank_close(a: torch.Tensor, b: torch.Tensor) -> None:
    """Rank-r activations (hi + lo bf16 planes) within 1e-2 relative rms."""
    va = a.double()[0] + a.double()[1]
    vb = b.double()[0] + b.double()[1]
    err = float(torch.sqrt(torch.mean((va - vb) ** 2)) / torch.sqrt(torch.mean(vb ** 2)).clamp_min(1e-30))
    assert err <= 1e-2, err


@pytest.mark.parametrize("precision,case", [
    ("nvfp4", W.QKV),                                                          # 2.4 MB of workspace
    ("nvfp4", W.scaled(W.QKV, M=300, K=1024, N=512, rank=64, name="ragged_r64")),
    ("int4", W.scaled(W.INT4_QKV, M=256, K=1024, N=512, rank=32, name="int4_small")),
], ids=lambda v: v if isinstance(v, str) else v.name)
def test_noalloc_matches_workspace_entry_point(precision, case):
    from bit_w4a4_quantized_token_b200 import _lib, layer

    assert _lib.svdq_quantize_act_workspace_bytes(precision, case.M, case.K, case.rank) > 0
    inp = W.make_inputs(case)
    d = {k: v.cuda() for k, v in inp.items()}
    packed = layer.pack_weight(d["R"], d["lam"], d["L_down"], d["L_up"], d["b"], precision=precision)
    ref = layer.quantize_act(d["x"], packed)          # existing entry point, caller-owned workspace
    gs = packed.group_size
    for call in range(2):                              # two calls in a row share the built-in array
        out = layer.alloc_act(packed, case.M, d["x"].device)
        compute = 1
        if precision == "nvfp4":
            out.x_tensor_scale.fill_(-1.0)             # overwritten by the amax pre-pass
        _lib.svdq_debug_force_quant_plan(1)            # partials through the (built-in) workspace
        try:
            _lib.svdq_quantize_act_noalloc(precision, gs, d["x"], case.M, case.K, packed.inv_lambda,
                                           out.x_tensor_scale, compute, packed.w_tensor_scale, packed.L_down_t,
                                           case.rank, out.x_codes, out.x_scales, out.lowrank_act)
        finally:
            _lib.svdq_debug_force_quant_plan(0)
        torch.cuda.synchronize()
        st, site = _lib.svdq_device_status(clear=True)
        assert st == 0, (st, site)
        assert torch.equal(out.x_codes, ref.x_codes), call
        assert torch.equal(out.x_scales, ref.x_scales), call
        if precision == "nvfp4":
            assert torch.equal(out.x_tensor_scale[:1], ref.x_tensor_scale[:1]), call
        _lowrank_close(out.lowrank_act, ref.lowrank_act)
        # the GEMM on the no-alloc quantizer's output matches too.  Both outputs
        # are bf16 roundings of nearly the same fp32 value (the split's partials
        # are added in a different grouping), so they may differ by one bf16
        # ulp: the bar is the output bar of the parity tests, with that ulp
        # allowed for beyond the error.
        y_ref = layer.gemm(ref, packed)
        y = layer.gemm(out, packed)
        torch.cuda.synchronize()
        yr, yo = y_ref.double(), y.double()
        rms = float(torch.sqrt(torch.mean(yr ** 2)))
        ulp = torch.exp2(torch.floor(torch.log2(yr.abs().clamp_min(2.0 ** -126))) - 7)
        assert float(torch.max(torch.abs(yo - yr) - ulp)) <= 1e-2 * rms
        assert float(torch.mean((torch.abs(yo - yr) <= ulp).double())) >= 0.999


def test_noalloc_rejects_shapes_beyond_the_builtin_array():
    from bit_w4a4_quantized_token_b200 import _lib

    # rank 128 on the QKV shape needs 36 x 4 x 128 x 128 x 4 B = 9.4 MB > 8 MiB
    assert _lib.svdq_quantize_act_workspace_bytes("nvfp4", 4608, 3072, 128) > 8 << 20
    fake = 1 << 20
    with pytest.raises(_lib.SvdqError) as e:
        _lib.svdq_quantize_act_noalloc("nvfp4", 16, fake, 4608, 3072, fake, fake, 0, fake, fake, 128, fake, fake,
                                       fake)
    assert e.value.status == _lib.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert "8388608" in _lib.lib.svdq_last_error().decode()
