"""Parity of the fused QKV + RMSNorm + RoPE path with the CPU oracle.

The fused to_qkv projection (the tutorial page's "structural rewrite"
passage; the Diffusers docs page "Nunchaku Lite", section "Fused kernels"):
the SVDQ W4A4 linear layer, then per head of Q and K an RMSNorm and the
rotary embedding.  The fused kernel applies both to the fp32 result before the
single bf16 rounding, so it is held to the linear layer's output bar against
the oracle's exact fp64 chain.  The unfused kernel works on the bf16 output
already in memory; it is held to the same bar against the oracle applied to
that bf16 output.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_quantized_token_b200 import workloads as W

from .parity import check_y, oracle_for, sample_rows, to_dev, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_w4a4_quantized_token_b200 import _lib

    yield
    st, site = _lib.svdq_device_status(clear=True)
    assert st == 0, f"device status {st} (site {site})"


def _run(case, heads, rows=None, with_bias=True):
    from bit_w4a4_quantized_token_b200 import _lib, layer
    from oracle import oracle as O

    inp = W.make_inputs(case)
    ex = W.qkv_inputs(case.M, heads)
    d = to_dev(inp)
    r = case.rank
    packed = layer.pack_weight(d["R"], d["lam"], d["L_down"] if r else None, d["L_up"] if r else None,
                               d["b"] if with_bias else None)
    q = layer.quantize_act(d["x"], packed)
    dx = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in ex.items()}
    y = torch.empty(case.M, case.N, dtype=torch.bfloat16, device="cuda")
    _lib.svdq_gemm_w4a4_qkv_norm_rope("nvfp4", 16, q.x_codes, q.x_scales, q.x_tensor_scale, case.M, packed.w_codes,
                                      packed.w_scales, packed.w_tensor_scale, case.N, case.K, q.lowrank_act,
                                      packed.L_up_t, r, packed.bias, heads, ex["head_dim"], dx["norm_q"],
                                      dx["norm_k"], ex["eps"], dx["cos"], dx["sin"], y)
    y_plain = layer.gemm(q, packed)
    torch.cuda.synchronize()
    ref = oracle_for(case, inp, rows=rows, with_bias=with_bias)
    sel = slice(None) if rows is None else np.asarray(rows)
    cos = ex["cos"].double().numpy()[sel]
    sin = ex["sin"].double().numpy()[sel]
    out, outb = O.qkv_norm_rope(ref.y, heads, ex["head_dim"], W.bits(ex["norm_q"]), W.bits(ex["norm_k"]),
                                ex["eps"], cos, sin)
    return y, y_plain, ref, out, outb, ex, dx


SMALL = [
    (W.scaled(W.QKV, M=300, K=512, N=768, rank=32, name="qkv_h2_ragged"), 2),
    (W.scaled(W.QKV, M=1, K=256, N=384, rank=16, name="qkv_h1_m1"), 1),
    (W.scaled(W.QKV, M=520, K=1024, N=1536, rank=0, name="qkv_h4_rank0"), 4),
]


@pytest.mark.parametrize("case,heads", SMALL, ids=lambda v: v.name if hasattr(v, "name") else str(v))
def test_fused_qkv_norm_rope_small(case, heads):
    y, y_plain, ref, out, outb, _, _ = _run(case, heads)
    check_y(u16(y), out, outb, "fused qkv")
    # V columns are the plain layer output, bit for bit
    v0 = 2 * heads * 128
    assert torch.equal(y[:, v0:], y_plain[:, v0:])


def test_fused_qkv_without_bias():
    case = W.scaled(W.QKV, M=129, K=256, N=384, rank=32, name="qkv_nobias")
    y, _, _, out, outb, _, _ = _run(case, 1, with_bias=False)
    check_y(u16(y), out, outb, "fused qkv, no bias")


def test_unfused_norm_rope_matches_oracle_on_bf16_y():
    """The separate pass on the projection's bf16 output, in place and out of place."""
    from bit_w4a4_quantized_token_b200 import _lib
    from oracle import oracle as O

    case, heads = W.scaled(W.QKV, M=300, K=512, N=768, rank=32, name="qkv_unfused"), 2
    _, y_plain, _, _, _, ex, dx = _run(case, heads)
    y_bits = u16(y_plain)
    yv = (y_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    out, outb = O.qkv_norm_rope(yv, heads, 128, W.bits(ex["norm_q"]), W.bits(ex["norm_k"]), ex["eps"],
                                ex["cos"].double().numpy(), ex["sin"].double().numpy())
    y2 = torch.empty_like(y_plain)
    _lib.svdq_qkv_norm_rope(y_plain, y2, case.M, heads, 128, dx["norm_q"], dx["norm_k"], ex["eps"], dx["cos"],
                            dx["sin"])
    _lib.svdq_qkv_norm_rope(y_plain, y_plain, case.M, heads, 128, dx["norm_q"], dx["norm_k"], ex["eps"], dx["cos"],
                            dx["sin"])
    torch.cuda.synchronize()
    assert torch.equal(y2, y_plain)
    check_y(u16(y2), out, outb, "unfused qkv")


def test_fused_qkv_full_size_sampled_rows():
    """The DiT QKV projection (24 heads of 128), every 128-row tile position."""
    rows = sample_rows(W.QKV.M, n=64, seed=21)
    y, _, _, out, outb, _, _ = _run(W.QKV, 24, rows=rows)
    check_y(u16(y)[rows], out, outb, "fused qkv full size")


def test_qkv_argument_checks():
    from bit_w4a4_quantized_token_b200 import _lib

    fake = 1 << 20
    args = dict(precision="nvfp4", group_size=16, x_codes=fake, x_scales=fake, x_tensor_scale=fake, M=64,
                w_codes=fake, w_scales=fake, w_tensor_scale=fake, N=768, K=256, lowrank_act=fake, L_up_t=fake,
                rank=32, bias=None, heads=2, head_dim=128, norm_q=fake, norm_k=fake, eps=1e-6, rope_cos=fake,
                rope_sin=fake, y=fake)
    for bad, status in ((dict(head_dim=64), _lib.SVDQ_ERR_UNSUPPORTED_SHAPE),
                        (dict(N=512), _lib.SVDQ_ERR_UNSUPPORTED_SHAPE),
                        (dict(eps=0.0), _lib.SVDQ_ERR_INVALID_ARG),
                        (dict(precision="int4", group_size=64), _lib.SVDQ_ERR_INVALID_ARG),
                        (dict(rope_cos=None), _lib.SVDQ_ERR_INVALID_ARG)):
        with pytest.raises(_lib.SvdqError) as e:
            _lib.svdq_gemm_w4a4_qkv_norm_rope(**dict(args, **bad))
        assert e.value.status == status, bad
