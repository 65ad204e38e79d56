"""Parity of the fused GELU MLP with the CPU oracle and with the unfused path.

The DiT feed-forward block fc1 -> GELU -> fc2 (the GELU-MLP fusion of the
Diffusers docs page "Nunchaku Lite", section "Fused kernels"): fc1's GEMM
epilogue applies GELU and performs fc2's activation step itself.  Checks:

* the GELU pass alone against the oracle on the same bf16 inputs;
* the fused path against the unfused one on the GPU (fc1 -> bf16 y ->
  svdq_gelu -> svdq_quantize_act with the same static scale): identical
  nvfp4 codes and scales, bit for bit, and the rank-r activations to the
  precision of two fp32 summation orders;
* fc2's output after the fused path against the oracle's fc2 applied to the
  GPU's own h (the same input bits: its codes and scales bit for bit, the
  output at the linear layer's bf16 bar), plus its rank-r activations at the
  usual 1e-2;
* the same output against the oracle's whole fp64 chain from x: fc1's bf16
  outputs, and so h and fc2's codes, may differ from the oracle's where two
  correct fp32 summation orders round differently (the codes agree on >= 99 %
  of the elements), so there only the 1 %-of-rms bound holds on every element
  and the 1-ulp agreement is asked of >= 99 % of them;
* the workspace of partial sums is left zeroed;
* fc1 with only the GELU in its epilogue (svdq_gemm_w4a4_gelu) stores the
  GELU pass's h on fc1's y, bit for bit.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_quantized_token_b200 import workloads as W

from .parity import bf16_ulp_distance, check_lowrank, check_y, sample_rows, u16, unswizzle_nvfp4_scales

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_w4a4_quantized_token_b200 import _lib

    yield
    st, site = _lib.svdq_device_status(clear=True)
    assert st == 0, f"device status {st} (site {site})"


def _layer_bits(inp, rank):
    return {"lam": inp["lam"].numpy(), "R": W.bits(inp["R"]), "L_down": W.bits(inp["L_down"]) if rank else None,
            "L_up": W.bits(inp["L_up"]) if rank else None, "b": W.bits(inp["b"])}


def _run(M, D, Hd, r1, r2, approx, rows=None, cal_rows=None):
    """fc1: D -> Hd (rank r1), fc2: Hd -> D (rank r2), M tokens."""
    from bit_w4a4_quantized_token_b200 import _lib, layer
    from oracle import oracle as O

    c1 = W.scaled(W.FC1, M=M, K=D, N=Hd, rank=r1, name="mlp_fc1")
    c2 = W.scaled(W.FC2, M=M, K=Hd, N=D, rank=r2, name="mlp_fc2")
    i1, i2 = W.make_inputs(c1), W.make_inputs(c2)
    fc1, fc2 = _layer_bits(i1, r1), _layer_bits(i2, r2)
    x_bits = W.bits(i1["x"])
    S1 = O.nvfp4_tensor_scale(x_bits, fc1["lam"])
    # fc2's static activation scale, calibrated by the oracle on some rows
    cal = np.arange(min(M, 64)) if cal_rows is None else cal_rows
    _, h_cal, _ = O.gelu_mlp(x_bits, fc1, fc2, S1, 1.0, approx, rows=cal)
    S2 = O.nvfp4_tensor_scale(h_cal, fc2["lam"])

    dev = "cuda"
    p1 = layer.pack_weight(i1["R"].to(dev), i1["lam"].to(dev), i1["L_down"].to(dev) if r1 else None,
                           i1["L_up"].to(dev) if r1 else None, i1["b"].to(dev))
    p2 = layer.pack_weight(i2["R"].to(dev), i2["lam"].to(dev), i2["L_down"].to(dev) if r2 else None,
                           i2["L_up"].to(dev) if r2 else None, i2["b"].to(dev))
    q1 = layer.quantize_act(i1["x"].to(dev), p1, x_tensor_scale=S1)
    # fused: fc1 GEMM + GELU + fc2's activation step, then fc2's GEMM
    qf = layer.alloc_act(p2, M, dev)
    qf.x_tensor_scale.fill_(S2)
    ws = torch.zeros(max(1, _lib.svdq_gelu_mlp_workspace_bytes(M, r2) // 4), dtype=torch.float32, device=dev)
    _lib.svdq_gemm_w4a4_gelu_quant("nvfp4", 16, q1.x_codes, q1.x_scales, q1.x_tensor_scale, M, p1.w_codes,
                                   p1.w_scales, p1.w_tensor_scale, Hd, D, q1.lowrank_act, p1.L_up_t, r1, p1.bias,
                                   approx, p2.inv_lambda, p2.L_down_t, r2, qf.x_tensor_scale, p2.w_tensor_scale,
                                   qf.x_codes, qf.x_scales, qf.lowrank_act, ws if r2 else None)
    y2f = layer.gemm(qf, p2)
    # unfused: fc1 -> bf16 y1 -> GELU pass -> fc2's quantizer -> fc2's GEMM
    y1 = layer.gemm(q1, p1)
    h = torch.empty_like(y1)
    _lib.svdq_gelu(y1, h, M * Hd, approx)
    qu = layer.quantize_act(h, p2, x_tensor_scale=S2)
    y2u = layer.gemm(qu, p2)
    # the partial fusion: fc1's epilogue applies only the GELU and stores h
    hs = torch.empty_like(y1)
    _lib.svdq_gemm_w4a4_gelu("nvfp4", 16, q1.x_codes, q1.x_scales, q1.x_tensor_scale, M, p1.w_codes, p1.w_scales,
                             p1.w_tensor_scale, Hd, D, q1.lowrank_act, p1.L_up_t, r1, p1.bias, approx, hs)
    torch.cuda.synchronize()
    assert float(ws.abs().max()) == 0.0, "workspace not left zeroed"
    assert torch.equal(hs, h), "the GELU epilogue's h differs from the GELU pass on fc1's y"
    r1o, ho, r2o = O.gelu_mlp(x_bits, fc1, fc2, S1, S2, approx, rows=rows)
    # fc2 alone on the GPU's h (the unfused pass's bits; the fused path hands fc2 the same codes)
    h_rows = u16(h) if rows is None else u16(h)[np.asarray(rows)]
    r2c = O.svdq_linear("nvfp4", np.ascontiguousarray(h_rows), fc2["lam"], fc2["R"], fc2["L_down"], fc2["L_up"],
                        fc2["b"], S_x=S2)
    return dict(qf=qf, qu=qu, y2f=y2f, y2u=y2u, y1=y1, h=h, r1o=r1o, ho=ho, r2o=r2o, r2c=r2c, S1=S1, S2=S2, p2=p2)


def _check_fc2(o, M, Hd, r2, rows=None):
    """fc2 after the fused path: against the oracle on the GPU's own h (same
    inputs, the layer's bar) and against the oracle's chain from x."""
    qf, r2c, r2o = o["qf"], o["r2c"], o["r2o"]
    sel = np.arange(M) if rows is None else np.asarray(rows)
    codes = qf.x_codes[: M * Hd // 2].cpu().numpy().reshape(M, Hd // 2)[sel]
    scales = unswizzle_nvfp4_scales(qf.x_scales.cpu().numpy(), M, Hd)[sel]
    assert np.array_equal(codes, r2c.x_codes), "fc2 codes differ from the oracle's on the same h"
    assert np.array_equal(scales, r2c.x_scales), "fc2 scales differ from the oracle's on the same h"
    y = u16(o["y2f"])[sel]
    check_y(y, r2c.y, r2c.y_bf16, "fc2 output, oracle on the same h")
    assert np.mean(codes == r2o.x_codes) >= 0.99
    assert np.mean(scales == r2o.x_scales) >= 0.99
    check_y(y, r2o.y, r2o.y_bf16, "fc2 output, oracle chain from x", min_frac1=0.99)


SMALL = [
    # (M, D, Hd, r1, r2, approx): ragged M; Hd % 256 == 128 (a last tile whose
    # second half has no columns); rank 16 and 0 for fc2; both GELU forms
    (300, 256, 640, 32, 32, 0),
    (300, 256, 640, 32, 32, 1),
    (1, 128, 512, 16, 16, 0),
    (520, 384, 1024, 0, 0, 0),
    (129, 256, 384, 32, 16, 1),
]


@pytest.mark.parametrize("M,D,Hd,r1,r2,approx", SMALL, ids=lambda v: str(v))
def test_fused_mlp_small(M, D, Hd, r1, r2, approx):
    o = _run(M, D, Hd, r1, r2, approx)
    qf, qu = o["qf"], o["qu"]
    # fused == unfused: the same codes (rows < M; padding rows hold no codes)
    # and scales (padding rows included: both write 0 there)
    nb = M * Hd // 2
    assert torch.equal(qf.x_codes[:nb], qu.x_codes[:nb]), "nvfp4 codes of h differ from the unfused path"
    assert torch.equal(qf.x_scales, qu.x_scales), "nvfp4 scales of h differ from the unfused path"
    if r2:
        a = (qf.lowrank_act[0].double() + qf.lowrank_act[1].double())
        b = (qu.lowrank_act[0].double() + qu.lowrank_act[1].double())
        rel = float((a - b).norm() / b.norm().clamp_min(1e-30))
        assert rel <= 1e-5, rel
    if r2:
        check_lowrank(qf.lowrank_act, o["r2c"].L,
                      float(np.float32(o["S2"]) * np.float32(float(o["p2"].w_tensor_scale[0]))))
    _check_fc2(o, M, Hd, r2)


def test_gelu_pass_matches_oracle_on_every_bf16():
    """The unfused GELU pass (the same bf16 -> bf16 function the fused
    epilogue uses) on every finite bf16 value: the oracle rounds the fp64
    value once; the kernel rounds erfc / exp computed in fp32, so a value
    within fp32 error of a bf16 rounding boundary may land one ulp away.
    An odd count (65279) also runs the kernel's scalar tail."""
    from bit_w4a4_quantized_token_b200 import _lib
    from oracle import oracle as O

    bits = np.arange(65536, dtype=np.uint32)
    finite = ((bits >> 7) & 0xFF) != 0xFF
    xb = bits[finite].astype(np.uint16)[:-1]
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
    n = xb.size
    for approx in (0, 1):
        y = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        _lib.svdq_gelu(x.cuda(), y, n, approx)
        torch.cuda.synchronize()
        ref = O.gelu_bf16(xb, approx)
        got = u16(y)
        d = bf16_ulp_distance(got, ref)
        assert d.max() <= 1 and np.mean(d == 0) >= 0.999, (approx, int(d.max()), float(np.mean(d == 0)))
        for v in (0x0000, 0x8000, 0x4220, 0xC220):    # +-0, +-40
            i = int(np.nonzero(xb == v)[0][0])
            assert got[i] == ref[i], hex(v)


def test_fused_mlp_full_size_sampled_rows():
    """The DiT MLP (3072 -> 12288 -> 3072, rank 32, 4608 tokens), 64 rows
    spread over every 128-row tile."""
    rows = sample_rows(4608, n=64, seed=43)
    o = _run(4608, 3072, 12288, 32, 32, 0, rows=rows, cal_rows=rows[:16])
    qf, qu = o["qf"], o["qu"]
    assert torch.equal(qf.x_codes[:4608 * 6144], qu.x_codes[:4608 * 6144])
    assert torch.equal(qf.x_scales, qu.x_scales)
    _check_fc2(o, 4608, 12288, 32, rows=rows)


def test_fused_mlp_argument_checks():
    from bit_w4a4_quantized_token_b200 import _lib

    fake = 1 << 20
    args = dict(precision="nvfp4", group_size=16, x_codes=fake, x_scales=fake, x_tensor_scale=fake, M=64,
                w_codes=fake, w_scales=fake, w_tensor_scale=fake, N=512, K=256, lowrank_act=fake, L_up_t=fake,
                rank=32, bias=None, gelu_approx=0, next_inv_lambda=fake, next_L_down_t=fake, next_rank=32,
                next_x_tensor_scale=fake, next_w_tensor_scale=fake, next_x_codes=fake, next_x_scales=fake,
                next_lowrank_act=fake, workspace=fake, workspace_bytes=64 * 32 * 4)
    for bad, status in ((dict(N=576), _lib.SVDQ_ERR_UNSUPPORTED_SHAPE),
                        (dict(next_rank=64), _lib.SVDQ_ERR_UNSUPPORTED_SHAPE),
                        (dict(next_rank=8), _lib.SVDQ_ERR_INVALID_ARG),
                        (dict(gelu_approx=2), _lib.SVDQ_ERR_INVALID_ARG),
                        (dict(precision="int4", group_size=64), _lib.SVDQ_ERR_INVALID_ARG),
                        (dict(workspace_bytes=64 * 32 * 4 - 4), _lib.SVDQ_ERR_INVALID_ARG),
                        (dict(next_x_tensor_scale=None), _lib.SVDQ_ERR_INVALID_ARG)):
        with pytest.raises(_lib.SvdqError) as e:
            _lib.svdq_gemm_w4a4_gelu_quant(**dict(args, **bad))
        assert e.value.status == status, bad


def test_gelu_epilogue_argument_checks():
    from bit_w4a4_quantized_token_b200 import _lib

    fake = 1 << 20
    args = dict(precision="nvfp4", group_size=16, x_codes=fake, x_scales=fake, x_tensor_scale=fake, M=64,
                w_codes=fake, w_scales=fake, w_tensor_scale=fake, N=512, K=256, lowrank_act=fake, L_up_t=fake,
                rank=32, bias=None, gelu_approx=0, y=fake)
    for bad, status in ((dict(N=576), _lib.SVDQ_ERR_UNSUPPORTED_SHAPE),
                        (dict(gelu_approx=2), _lib.SVDQ_ERR_INVALID_ARG),
                        (dict(precision="int4", group_size=64), _lib.SVDQ_ERR_INVALID_ARG),
                        (dict(y=None), _lib.SVDQ_ERR_INVALID_ARG),
                        (dict(y=fake + 2), _lib.SVDQ_ERR_INVALID_ARG)):
        with pytest.raises(_lib.SvdqError) as e:
            _lib.svdq_gemm_w4a4_gelu(**dict(args, **bad))
        assert e.value.status == status, bad
