"""Parity of the weight-only int4 GEMM (W4A16) with the CPU oracle.

The `awq_w4a16` scheme of the Diffusers docs page "Nunchaku Lite" (section
"Supported quantization types": int4 with group 64, the INT4 weight-only
AWQ-style kernel): the weight is packed by svdq_pack_weight(int4, 64) with
all smoothing divisors 1 and no rank-r branch, x is used as it comes, and the
output is held to the linear layer's bf16 bar against the oracle's exact
fp64 sum.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_quantized_token_b200 import workloads as W

from .parity import check_y, sample_rows, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_w4a4_quantized_token_b200 import _lib

    yield
    st, site = _lib.svdq_device_status(clear=True)
    assert st == 0, f"device status {st} (site {site})"


def _run(case, rows=None, with_bias=True):
    from bit_w4a4_quantized_token_b200 import _lib, layer
    from oracle import oracle as O

    inp = W.make_inputs(case)
    x, Wt, b = inp["x"].cuda(), inp["R"].cuda(), inp["b"].cuda()
    ones = torch.ones(case.K, dtype=torch.float32, device="cuda")
    packed = layer.pack_weight(Wt, ones, None, None, b if with_bias else None, precision="int4")
    y = torch.empty(case.M, case.N, dtype=torch.bfloat16, device="cuda")
    _lib.svdq_gemm_w4a16(x, case.M, packed.w_codes, packed.w_scales, case.N, case.K, packed.bias, y)
    torch.cuda.synchronize()
    wc, ws = O.int4_quantize(W.bits(inp["R"]), np.ones(case.K, np.float32))
    x_bits = W.bits(inp["x"])
    ref, refb = O.w4a16_linear(x_bits, wc, ws, W.bits(inp["b"]) if with_bias else None, rows=rows)
    got = u16(y) if rows is None else u16(y)[np.asarray(rows)]
    return got, ref, refb


SMALL = [
    W.scaled(W.QKV, M=300, K=320, N=272, rank=0, name="w4a16_ragged"),
    W.scaled(W.QKV, M=1, K=64, N=16, rank=0, name="w4a16_min"),
    W.scaled(W.QKV, M=256, K=1024, N=512, rank=0, name="w4a16_tiles"),
    W.scaled(W.FC2, M=130, K=2048, N=784, rank=0, name="w4a16_fc2like"),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_w4a16_small(case):
    got, ref, refb = _run(case)
    check_y(got, ref, refb, case.name)


def test_w4a16_without_bias():
    case = W.scaled(W.QKV, M=200, K=192, N=256, rank=0, name="w4a16_nobias")
    got, ref, refb = _run(case, with_bias=False)
    check_y(got, ref, refb, case.name)


def test_w4a16_full_size_sampled_rows():
    """The QKV projection shape (4608 x 3072 -> 9216), rows from every 128-row tile."""
    case = W.scaled(W.QKV, rank=0, name="w4a16_qkv")
    rows = sample_rows(case.M, n=512, seed=31)
    got, ref, refb = _run(case, rows=rows)
    check_y(got, ref, refb, case.name)


def test_w4a16_argument_checks():
    from bit_w4a4_quantized_token_b200 import _lib

    fake = 1 << 20
    args = dict(x=fake, M=64, w_codes=fake, w_scales=fake, N=256, K=256, bias=None, y=fake)
    for bad, status in ((dict(N=264), _lib.SVDQ_ERR_UNSUPPORTED_SHAPE),
                        (dict(K=96), _lib.SVDQ_ERR_UNSUPPORTED_SHAPE),
                        (dict(M=0), _lib.SVDQ_ERR_UNSUPPORTED_SHAPE),
                        (dict(x=None), _lib.SVDQ_ERR_INVALID_ARG),
                        (dict(bias=fake + 8), _lib.SVDQ_ERR_INVALID_ARG)):
        with pytest.raises(_lib.SvdqError) as e:
            _lib.svdq_gemm_w4a16(**dict(args, **bad))
        assert e.value.status == status, bad
