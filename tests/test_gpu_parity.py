"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Codes, group scales and tensor scales must match bit for bit; the bf16 output
must satisfy max|d| <= 1e-2 rms(y_ref) and be within 1 bf16 ulp of the
oracle's rounding on >= 99.9 % of elements; the rank-r activations must match
within 1e-2 relative rms.  Small cases compare every element; the full-size
cases (the launch configuration the benchmark times) compare codes and scales
in full and the output on sampled rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_quantized_token_b200 import workloads as W

from .parity import check_case, check_y, oracle_for, run_gpu, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_w4a4_quantized_token_b200 import _lib

    yield
    st, site = _lib.svdq_device_status(clear=True)
    assert st == 0, f"device status {st} (site {site})"


SMALL = [
    W.TINY,                                                              # the tiny case, full
    W.scaled(W.TINY, M=200, K=320, N=272, rank=16, name="ragged"),      # ragged M, K tail, N tail
    W.scaled(W.QKV, M=300, K=1024, N=512, rank=64, name="multi_tile_r64"),
    W.scaled(W.QKV, M=129, K=512, N=384, rank=0, name="rank0"),
    W.scaled(W.QKV, M=256, K=768, N=256, rank=128, name="r128"),
    W.scaled(W.FC2, M=130, K=2048, N=512, rank=32, name="fc2_small"),
    W.scaled(W.FC2, M=260, K=3136, N=272, rank=32, name="streamed_scales_ragged"),   # K > 3072, 49 k-steps
    W.scaled(W.QKV, M=1, K=64, N=16, rank=16, name="minimal"),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_small_cases_full(case):
    check_case(case)


@pytest.mark.parametrize("mode", [1, 2], ids=["single_cta_tiles", "cta_pair_tiles"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: c.name)
def test_small_cases_each_gemm_kernel(case, mode):
    """Both nvfp4 GEMM kernels (128 x 256 tiles on one CTA, 256 x 256 tiles on
    a CTA pair) on every small case, whatever M would pick."""
    from bit_w4a4_quantized_token_b200 import _lib

    _lib.svdq_debug_force_gemm_tiles(mode)
    try:
        check_case(case)
    finally:
        _lib.svdq_debug_force_gemm_tiles(0)


# the ways the quantizer adds the rank-r partials of a K split: through the
# workspace (global memory; every split adds a slice of rows, or the last CTA
# adds all of them) and inside one thread-block cluster (distributed shared
# memory); a ragged tail, the largest cluster, rank 128
QUANT_PLAN_CASES = [
    W.scaled(W.QKV, M=300, K=1024, N=512, rank=64, name="qp_ragged_r64"),
    W.scaled(W.QKV, M=128, K=3072, N=256, rank=32, name="qp_one_block_k3072"),
    W.scaled(W.QKV, M=520, K=1536, N=384, rank=128, name="qp_r128"),
    W.scaled(W.INT4_QKV, M=200, K=1024, N=272, rank=16, name="qp_int4"),
]


@pytest.mark.parametrize("mode", [1, 2, 3], ids=["workspace", "cluster", "workspace_last_cta"])
@pytest.mark.parametrize("case", QUANT_PLAN_CASES, ids=lambda c: c.name)
def test_quantizer_split_modes(case, mode):
    from bit_w4a4_quantized_token_b200 import _lib

    _lib.svdq_debug_force_quant_plan(mode)
    try:
        check_case(case)
    finally:
        _lib.svdq_debug_force_quant_plan(0)


def test_static_tensor_scale():
    case = W.scaled(W.QKV, M=160, K=512, N=256, rank=32, name="static_S")
    check_case(case, x_tensor_scale=0.0625)


def test_no_bias():
    check_case(W.scaled(W.QKV, M=64, K=256, N=128, rank=32, name="nobias"), with_bias=False)


def test_R_zero_reduces_to_lowrank_branch():
    case = W.scaled(W.QKV, M=96, K=256, N=192, rank=32, name="R0")
    inp = W.make_inputs(case)
    inp["R"] = torch.zeros_like(inp["R"])
    check_case(case, inp=inp)


def test_x_zero_gives_bias():
    case = W.scaled(W.QKV, M=64, K=256, N=128, rank=32, name="x0")
    inp = W.make_inputs(case)
    inp["x"] = torch.zeros_like(inp["x"])
    packed, q, y = run_gpu(case, inp)
    assert float(q.x_tensor_scale[0]) == 1.0
    assert not q.x_codes.any() and not q.x_scales.any()
    assert torch.equal(y.cpu(), inp["b"].expand(case.M, case.N))


def test_grid_exact_unit_scales():
    """x and R on the E2M1 grid with a +-6 in every group and S = 1: the GEMM
    is exact, so y equals the oracle's bf16 rounding bit for bit."""
    rng = np.random.default_rng(3)
    M, K, N = 128, 256, 256
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])

    def on_grid(rows):
        v = rng.choice(grid, size=(rows, K)) * rng.choice([-1.0, 1.0], size=(rows, K))
        v[:, ::16] = 6.0
        return torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)

    case = W.Case("grid", M, K, N, 0, "nvfp4", 0, 0)
    inp = {"x": on_grid(M), "R": on_grid(N), "lam": torch.ones(K), "L_down": None, "L_up": None,
           "b": torch.from_numpy(rng.standard_normal(N).astype(np.float32)).to(torch.bfloat16)}
    inp["R"] = inp["R"]
    from bit_w4a4_quantized_token_b200 import _lib, layer

    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    packed = layer.pack_weight(d["R"], d["lam"], None, None, d["b"])
    packed.w_tensor_scale.fill_(1.0)      # static unit scales on both sides
    # re-quantize the weight with S_w = 1: quantize it as an activation with lambda = 1
    wq = layer.quantize_act(d["R"], packed, x_tensor_scale=1.0)
    packed.w_codes = wq.x_codes
    packed.w_scales.zero_()
    packed.w_scales[: wq.x_scales.numel()].copy_(wq.x_scales.view(-1))
    _lib.svdq_replicate_weight_scales(packed.w_scales, N, K)
    q = layer.quantize_act(d["x"], packed, x_tensor_scale=1.0)
    y = layer.gemm(q, packed)
    xv = inp["x"].double().numpy()
    wv = inp["R"].double().numpy()
    exact = xv @ wv.T + inp["b"].double().numpy()
    from oracle import oracle as O

    ref_bits = np.array([[O.bf16_from_double(float(t)) for t in row] for row in exact], np.uint16)
    assert np.array_equal(u16(y), ref_bits)


def test_deterministic():
    case = W.scaled(W.QKV, M=300, K=1024, N=512, rank=32, name="det")
    inp = W.make_inputs(case)
    _, q1, y1 = run_gpu(case, inp)
    _, q2, y2 = run_gpu(case, inp)
    assert torch.equal(y1, y2) and torch.equal(q1.lowrank_act, q2.lowrank_act)


# ------------------------------------------------------------ full sizes
def rows_in_every_half_tile(M: int, per_half: int, seed: int) -> np.ndarray:
    """per_half rows from each 128-row half of every 256-row CTA-pair tile,
    plus the first and last rows of every half."""
    rng = np.random.default_rng(seed)
    rows = []
    for h0 in range(0, M, 128):
        h1 = min(M, h0 + 128)
        pick = rng.choice(np.arange(h0, h1), size=min(per_half, h1 - h0), replace=False)
        rows.extend(pick.tolist() + [h0, h1 - 1])
    return np.array(sorted(set(rows)))


@pytest.mark.parametrize("case", [W.QKV, W.FC1, W.FC2], ids=lambda c: c.name)
def test_full_size_every_row(case):
    """Every output row of the DiT projections, at the launch configuration
    the benchmark times."""
    check_case(case)


@pytest.mark.parametrize("case", [W.OUTPROJ[r] for r in (0, 16, 32, 64, 128)], ids=lambda c: c.name)
def test_full_size_outproj_rows(case):
    """The batch-4 out-projection (18432 rows): 16 random rows from each of
    the 144 halves of the 72 CTA-pair tiles plus each half's first and last
    row (about 2600 rows)."""
    rows = rows_in_every_half_tile(case.M, 16, seed=case.seed)
    assert len(rows) >= 2048
    check_case(case, rows=rows)


# ------------------------------------------------------------ int4 quantizers
@pytest.mark.parametrize("case", [W.scaled(W.INT4_QKV, M=200, K=320, N=272, rank=16, name="int4_ragged"),
                                  W.scaled(W.INT4_QKV, M=256, K=1024, N=512, rank=32, name="int4_small"),
                                  W.INT4_QKV], ids=lambda c: c.name)
def test_int4_quantizers(case):
    """Codes and bf16 group scales bit-exact; rank-r activations within 1e-2 rms."""
    from bit_w4a4_quantized_token_b200 import layer

    from .parity import check_lowrank, unswizzle_int4_scales

    inp = W.make_inputs(case)
    d = {k: v.cuda() for k, v in inp.items()}
    packed = layer.pack_weight(d["R"], d["lam"], d["L_down"], d["L_up"], d["b"], precision="int4")
    q = layer.quantize_act(d["x"], packed)
    torch.cuda.synchronize()
    ref = oracle_for(case, inp, with_y=False)
    M, K, N = case.M, case.K, case.N
    assert np.array_equal(packed.w_codes.cpu().numpy().reshape(N, K // 2), ref.w_codes)
    assert np.array_equal(q.x_codes.cpu().numpy().reshape(M, K // 2), ref.x_codes)
    assert np.array_equal(unswizzle_int4_scales(packed.w_scales.cpu().numpy(), N, K), ref.w_scales)
    assert np.array_equal(unswizzle_int4_scales(q.x_scales.cpu().numpy(), M, K), ref.x_scales)
    check_lowrank(q.lowrank_act, ref.L, 1.0)


# ------------------------------------------------------------ int4 W4A4 GEMM
INT4_SMALL = [
    W.scaled(W.INT4_QKV, M=64, K=256, N=256, rank=32, name="int4_tiny"),
    W.scaled(W.INT4_QKV, M=200, K=320, N=272, rank=16, name="int4_ragged"),   # K tail (5 groups), N tail
    W.scaled(W.INT4_QKV, M=300, K=1024, N=512, rank=64, name="int4_multi_tile"),
    W.scaled(W.INT4_QKV, M=129, K=512, N=384, rank=0, name="int4_rank0"),
]


@pytest.mark.parametrize("case", INT4_SMALL, ids=lambda c: c.name)
def test_int4_small_cases_full(case):
    check_case(case)


def test_int4_full_size_every_row():
    check_case(W.INT4_QKV)
