"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these re-types the oracle's formulas: each checks one oracle step
against an independent ground truth -- a brute-force nearest-value search, a
library routine (torch's float8_e4m3fn cast), exact rational arithmetic
(fractions.Fraction), a closed form (inputs on the E2M1 grid with unit scales),
or an invariant (sign symmetry, power-of-two equivariance), or a special case
that reduces the layer to a plain fp64 matmul (rank 0, R = 0).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from bit_w4a4_quantized_token_b200 import workloads as W

E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # OCP MX FP4 E2M1 values


# ------------------------------------------------------------ helpers
def brute_e2m1(v: float) -> int:
    """Nearest E2M1 value by exhaustive search; ties to the even code."""
    a = abs(Fraction(float(v)))
    best = None
    for idx, g in enumerate(E2M1_GRID):
        d = abs(a - Fraction(g))
        key = (d, idx & 1)            # smaller distance, then even code
        if best is None or key < best[0]:
            best = (key, idx)
    sign = 8 if np.signbit(np.float32(v)) else 0
    return sign | best[1]


def torch_e4m3_value(byte: int) -> float:
    return float(torch.tensor([byte], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64))


E4M3_POS = [(b, torch_e4m3_value(b)) for b in range(0x7F)]   # 0x00..0x7E, all finite


def brute_e4m3(v: float) -> int:
    """Nearest non-negative E4M3FN value (<= 448) by exhaustive search, ties to even."""
    a = Fraction(float(v))
    best = None
    for b, val in E4M3_POS:
        key = (abs(a - Fraction(val)), b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return best[1]


def brute_bf16(d: float) -> int:
    """bf16 bits nearest to the double d (ties to even), by exact comparison."""
    f32 = np.array([d], dtype=np.float32)
    t = int(f32.view(np.uint32)[0] >> 16)
    sign = t & 0x8000
    mag = t & 0x7FFF
    best = None
    for cand in (mag - 1, mag, mag + 1):
        if cand < 0 or cand >= 0x7F80:
            continue
        val = Fraction(float(np.array([(sign | cand) << 16], dtype=np.uint32).view(np.float32)[0]))
        key = (abs(Fraction(d) - val), cand & 1)
        if best is None or key < best[0]:
            best = (key, sign | cand)
    return best[1]


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def py_nvfp4_dequant(codes, scales, S):
    """Independent dequantization: nibble -> grid value, byte -> torch E4M3 value."""
    codes = np.asarray(codes, np.uint8)
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(codes.shape[0], -1)
    grid = np.array(E2M1_GRID + [-g for g in E2M1_GRID])
    vals = grid[nib]
    sc = torch.from_numpy(np.ascontiguousarray(scales)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return vals * np.repeat(sc, 16, axis=1) * float(S)


# ------------------------------------------------------------- E2M1
def test_e2m1_grid_roundtrip(oracle_mod):
    O = oracle_mod
    for code in range(16):
        v = O.e2m1_decode(code)
        expect = E2M1_GRID[code & 7] * (-1 if code & 8 else 1)
        assert v == expect
        # -0.0 keeps its sign bit: code 8 encodes back to 8
        assert O.e2m1_encode(np.float32(-0.0) if code == 8 else v) == code


def test_e2m1_midpoints_tie_to_even(oracle_mod):
    O = oracle_mod
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    expect = [0, 2, 2, 4, 4, 6, 6]          # the even neighbour each time
    for m, e in zip(mids, expect):
        assert O.e2m1_encode(m) == e, m
        assert O.e2m1_encode(-m) == (8 | e), m
        assert brute_e2m1(m) == e


def test_e2m1_saturates(oracle_mod):
    for v in (6.0, 6.5, 7.0, 100.0, 3.0e38):
        assert oracle_mod.e2m1_encode(v) == 7
        assert oracle_mod.e2m1_encode(-v) == 15


def test_e2m1_bruteforce_random(oracle_mod):
    rng = np.random.default_rng(123)
    vals = np.concatenate([
        rng.uniform(-7, 7, 20000).astype(np.float32),
        rng.standard_normal(5000).astype(np.float32) * 0.3,
        # one fp32 ulp either side of every midpoint
        np.array([np.nextafter(np.float32(m), np.float32(s * 10)) * sgn
                  for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0) for s in (-1, 1) for sgn in (-1, 1)],
                 dtype=np.float32),
    ])
    for v in vals:
        assert oracle_mod.e2m1_encode(float(v)) == brute_e2m1(float(v)), v


# ------------------------------------------------------------- E4M3
def test_e4m3_exhaustive_roundtrip(oracle_mod):
    O = oracle_mod
    for b in range(256):
        if b & 0x7F == 0x7F:       # NaN encodings
            continue
        v = O.e4m3_decode(b)
        assert v == torch_e4m3_value(b), b
        assert O.e4m3_encode(np.float32(v) if b != 0x80 else np.float32(-0.0)) == b, b


def test_e4m3_matches_torch_cast(oracle_mod):
    rng = np.random.default_rng(7)
    v = np.concatenate([
        np.exp2(rng.uniform(-12, np.log2(448.0), 20000)),
        np.array([E4M3_POS[i][1] + E4M3_POS[i + 1][1] for i in range(0x7E)]) / 2.0,   # exact midpoints
    ]).astype(np.float32)
    v = np.minimum(v, 448.0).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle_mod.e4m3_encode(float(t)) for t in v], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_saturates_and_bruteforce(oracle_mod):
    for t in (448.0, 449.0, 464.0, 500.0, 1e30):
        assert oracle_mod.e4m3_encode(t) == 0x7E
    rng = np.random.default_rng(9)
    for t in np.exp2(rng.uniform(-11, 8.8, 300)).astype(np.float32):
        assert oracle_mod.e4m3_encode(float(t)) == brute_e4m3(float(t))


# ------------------------------------------------------------- bf16
def test_bf16_rounding_exact(oracle_mod):
    rng = np.random.default_rng(11)
    ds = list(rng.standard_normal(3000) * np.exp2(rng.uniform(-20, 20, 3000)))
    # exact ties between neighbouring bf16 values
    for base in (1.0, 1.5, 3.0, -2.25, 1e-3):
        b = np.float32(base).view(np.uint32) & 0xFFFF0000
        lo = float(np.array([b], np.uint32).view(np.float32)[0])
        hi = float(np.array([b + 0x10000], np.uint32).view(np.float32)[0])
        ds.append((lo + hi) / 2)
    for d in ds:
        assert oracle_mod.bf16_from_double(float(d)) == brute_bf16(float(d)), d


# -------------------------------------------------- nvfp4 group quantizer
def test_tensor_scale_rule(oracle_mod):
    O = oracle_mod
    x = f32_to_bf16_bits(np.array([[1.0, -3.5, 2.0, 0.25] * 4], np.float32))
    lam = np.full(16, 0.5, np.float32)            # x / 0.5 = 2x exactly
    assert O.nvfp4_tensor_scale(x, lam) == np.float32(7.0) / np.float32(2688.0)
    z = np.zeros((2, 16), np.uint16)
    assert O.nvfp4_tensor_scale(z, None) == 1.0


def test_nvfp4_group_bruteforce(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(5)
    x = f32_to_bf16_bits(rng.standard_normal((2, 32)).astype(np.float32) * 3)
    lam = rng.uniform(0.5, 4, 32).astype(np.float32)
    S = O.nvfp4_tensor_scale(x, lam)
    codes, scales = O.nvfp4_quantize(x, lam, S)
    xs = (bf16_bits_to_f64(x).astype(np.float32) * (np.float32(1) / lam)).astype(np.float32)
    for m in range(2):
        for g in range(2):
            v = xs[m, g * 16:(g + 1) * 16]
            a = np.max(np.abs(v))
            t = np.float32(a) / (np.float32(6) * np.float32(S))
            e = scales[m, g]
            assert e == brute_e4m3(float(t))                  # nearest E4M3 of the target
            dec = np.float32(torch_e4m3_value(int(e))) * np.float32(S)
            inv = np.float32(1) / dec
            for i in range(16):
                k = g * 16 + i
                c = (codes[m, k // 2] >> (4 * (k & 1))) & 15
                assert c == brute_e2m1(float(np.float32(v[i]) * inv))
    # reconstruction error per element is at most one grid gap (2) times dec
    deq = py_nvfp4_dequant(codes, scales, S)
    dec_b = np.repeat(np.array([[torch_e4m3_value(int(s)) for s in row] for row in scales]) * S, 16, axis=1)
    assert np.all(np.abs(deq - xs) <= 1.0 * dec_b + 1e-30)


def test_nvfp4_sign_symmetry(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(6)
    xf = rng.standard_normal((3, 64)).astype(np.float32)
    x = f32_to_bf16_bits(xf)
    xn = f32_to_bf16_bits(-xf)
    lam = rng.uniform(0.5, 4, 64).astype(np.float32)
    S = O.nvfp4_tensor_scale(x, lam)
    assert O.nvfp4_tensor_scale(xn, lam) == S
    c1, s1 = O.nvfp4_quantize(x, lam, S)
    c2, s2 = O.nvfp4_quantize(xn, lam, S)
    assert np.array_equal(s1, s2)
    assert np.array_equal(c1 ^ 0x88, c2)


def test_nvfp4_pow2_equivariance(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(8)
    xf = rng.standard_normal((4, 64)).astype(np.float32)
    x = f32_to_bf16_bits(xf)
    S = float(np.max(np.abs(bf16_bits_to_f64(x)))) / (6 * 16)   # group scales near 16
    S = float(np.float32(S))
    c0, s0 = O.nvfp4_quantize(x, None, S)
    v0 = np.array([[torch_e4m3_value(int(b)) for b in row] for row in s0])
    for j in range(-3, 4):
        xj = f32_to_bf16_bits(bf16_bits_to_f64(x).astype(np.float32) * np.float32(2.0 ** j))
        cj, sj = O.nvfp4_quantize(xj, None, S)
        vj = np.array([[torch_e4m3_value(int(b)) for b in row] for row in sj])
        assert np.array_equal(cj, c0), j
        assert np.array_equal(vj, v0 * 2.0 ** j), j


# ------------------------------------------------- closed-form layer cases
def _grid_matrix(rng, rows, K):
    """Values on the E2M1 grid with a +-6 in every group of 16."""
    g = np.array(E2M1_GRID)
    v = rng.choice(g, size=(rows, K)) * rng.choice([-1.0, 1.0], size=(rows, K))
    v[:, ::16] = 6.0 * rng.choice([-1.0, 1.0], size=(rows, K // 16))
    return v


def test_exact_on_grid_unit_scales(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(10)
    M, K, N = 4, 64, 8
    xv, wv = _grid_matrix(rng, M, K), _grid_matrix(rng, N, K)
    x, R = f32_to_bf16_bits(xv), f32_to_bf16_bits(wv)
    b = f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32))
    xc, xs = O.nvfp4_quantize(x, None, 1.0)
    wc, ws = O.nvfp4_quantize(R, None, 1.0)
    assert np.all(xs == 0x38) and np.all(ws == 0x38)           # E4M3(1.0)
    xd, wd = O.nvfp4_dequant(xc, xs, 1.0), O.nvfp4_dequant(wc, ws, 1.0)
    assert np.array_equal(xd, xv) and np.array_equal(wd, wv)   # codes are exact
    y, ybf = O.nvfp4_linear(xd, wd, None, None, b)
    exact = xv @ wv.T + bf16_bits_to_f64(b)                     # small dyadics: exact
    assert np.array_equal(y, exact)
    assert np.array_equal(ybf, np.array([[brute_bf16(float(t)) for t in row] for row in exact], np.uint16))


def test_rank0_is_plain_w4a4_gemm(oracle_mod):
    O = oracle_mod
    case = W.scaled(W.TINY, M=16, K=128, N=32, rank=0)
    inp = W.make_inputs(case)
    x, R, b = W.bits(inp["x"]), W.bits(inp["R"]), W.bits(inp["b"])
    lam = inp["lam"].numpy()
    res = O.svdq_linear("nvfp4", x, lam, R, None, None, b)
    xd = py_nvfp4_dequant(res.x_codes, res.x_scales, res.S_x)
    wd = py_nvfp4_dequant(res.w_codes, res.w_scales, res.S_w)
    ref = torch.from_numpy(xd) @ torch.from_numpy(wd).T + torch.from_numpy(bf16_bits_to_f64(b))
    np.testing.assert_allclose(res.y, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_R_zero_gives_lowrank_branch(oracle_mod):
    O = oracle_mod
    case = W.scaled(W.TINY, M=8, K=64, N=48, rank=32)
    inp = W.make_inputs(case)
    x, b = W.bits(inp["x"]), W.bits(inp["b"])
    lam = inp["lam"].numpy()
    R = np.zeros((case.N, case.K), np.uint16)
    Ld, Lu = W.bits(inp["L_down"]), W.bits(inp["L_up"])
    res = O.svdq_linear("nvfp4", x, lam, R, Ld, Lu, b)
    assert res.S_w == 1.0
    assert not res.w_codes.any() and not res.w_scales.any()
    xs = bf16_bits_to_f64(x) / lam.astype(np.float64)
    ref = (xs @ bf16_bits_to_f64(Ld)) @ bf16_bits_to_f64(Lu) + bf16_bits_to_f64(b)
    np.testing.assert_allclose(res.y, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res.L, xs @ bf16_bits_to_f64(Ld), rtol=1e-10, atol=1e-12)


def test_lowrank_matches_fp64_chain(oracle_mod):
    O = oracle_mod
    case = W.scaled(W.TINY, M=5, K=96, N=16, rank=16)
    inp = W.make_inputs(case)
    x, Ld = W.bits(inp["x"]), W.bits(inp["L_down"])
    lam = inp["lam"].numpy()
    L = O.lowrank_down(x, lam, Ld)
    ref = (bf16_bits_to_f64(x) / lam.astype(np.float64)) @ bf16_bits_to_f64(Ld)
    np.testing.assert_allclose(L, ref, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ int4
def test_int4_bruteforce(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(12)
    x = f32_to_bf16_bits(rng.standard_normal((2, 128)).astype(np.float32) * 2)
    lam = rng.uniform(0.5, 4, 128).astype(np.float32)
    codes, scales = O.int4_quantize(x, lam)
    q = O.int4_codes_to_int(codes)
    xs = (bf16_bits_to_f64(x).astype(np.float32) * (np.float32(1) / lam)).astype(np.float32)
    for m in range(2):
        for g in range(2):
            v = xs[m, g * 64:(g + 1) * 64]
            a = float(np.max(np.abs(v)))
            assert scales[m, g] == brute_bf16(float(np.float32(a) / np.float32(7)))
            s = np.float32(bf16_bits_to_f64(scales[m, g]))
            inv = np.float32(1) / s
            for i in range(64):
                t = Fraction(float(np.float32(v[i]) * inv))
                best = min(range(-8, 8), key=lambda c: (abs(t - c), c & 1))
                assert q[m, g * 64 + i] == best


def test_int4_exact_grid(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(13)
    M, K, N = 3, 128, 8
    xv = rng.integers(-7, 8, size=(M, K)).astype(np.float64)
    wv = rng.integers(-7, 8, size=(N, K)).astype(np.float64)
    xv[:, ::64] = 7
    wv[:, ::64] = -7
    x, R = f32_to_bf16_bits(xv), f32_to_bf16_bits(wv)
    xc, xs = O.int4_quantize(x, None)
    wc, ws = O.int4_quantize(R, None)
    assert np.all(xs == 0x3F80) and np.all(ws == 0x3F80)     # bf16(1.0)
    assert np.array_equal(O.int4_codes_to_int(xc), xv.astype(np.int8))
    y, _ = O.int4_linear(xc, xs, wc, ws, None, None, None)
    assert np.array_equal(y, xv @ wv.T)


def test_int4_linear_matches_dequant_matmul(oracle_mod):
    O = oracle_mod
    case = W.scaled(W.INT4_QKV, M=8, K=256, N=24, rank=16)
    inp = W.make_inputs(case)
    x, R, b = W.bits(inp["x"]), W.bits(inp["R"]), W.bits(inp["b"])
    Ld, Lu = W.bits(inp["L_down"]), W.bits(inp["L_up"])
    lam = inp["lam"].numpy()
    res = O.svdq_linear("int4", x, lam, R, Ld, Lu, b)
    xd = O.int4_codes_to_int(res.x_codes) * np.repeat(bf16_bits_to_f64(res.x_scales), 64, axis=1)
    wd = O.int4_codes_to_int(res.w_codes) * np.repeat(bf16_bits_to_f64(res.w_scales), 64, axis=1)
    xs = bf16_bits_to_f64(x) / lam.astype(np.float64)
    ref = xd @ wd.T + (xs @ bf16_bits_to_f64(Ld)) @ bf16_bits_to_f64(Lu) + bf16_bits_to_f64(b)
    np.testing.assert_allclose(res.y, ref, rtol=1e-10, atol=1e-12)


def test_nvfp4_linear_row_subset(oracle_mod):
    """Sampled rows equal the same rows of the full computation."""
    O = oracle_mod
    case = W.scaled(W.TINY, M=12, K=64, N=32, rank=16)
    inp = W.make_inputs(case)
    args = [W.bits(inp["x"]), inp["lam"].numpy(), W.bits(inp["R"]), W.bits(inp["L_down"]),
            W.bits(inp["L_up"]), W.bits(inp["b"])]
    full = O.svdq_linear("nvfp4", *args)
    rows = np.array([11, 0, 5])
    sub = O.svdq_linear("nvfp4", *args, rows=rows)
    assert np.array_equal(sub.y, full.y[rows])


def test_int4_ties_to_even(oracle_mod):
    """With amax 7 the group scale is exactly 1, so half-integers are exact ties."""
    O = oracle_mod
    v = np.array([[7.0, 0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 3.5, -3.5, 4.5, -4.5, 5.5, -5.5, 6.5, -6.5, 0.0] * 4],
                 np.float32)
    codes, scales = O.int4_quantize(f32_to_bf16_bits(v), None)
    assert np.all(scales == 0x3F80)
    q = O.int4_codes_to_int(codes)[0, :16]
    assert list(q) == [7, 0, 0, 2, -2, 2, -2, 4, -4, 4, -4, 6, -6, 6, -6, 0]


# ------------------------------------------------- weight-only int4 (W4A16)
def test_w4a16_exact_on_integer_grid(oracle_mod):
    """Integer weights with amax 7 per group get scale 1, so y is the exact
    integer product x . W^T (small integers are exact in bf16)."""
    O = oracle_mod
    rng = np.random.default_rng(21)
    M, K, N = 4, 192, 6
    xv = rng.integers(-20, 21, size=(M, K)).astype(np.float64)
    wv = rng.integers(-7, 8, size=(N, K)).astype(np.float64)
    wv[:, ::64] = 7
    wc, ws = O.int4_quantize(f32_to_bf16_bits(wv), None)
    assert np.all(ws == 0x3F80)
    bias = rng.integers(-5, 6, size=N).astype(np.float64)
    y, ybf = O.w4a16_linear(f32_to_bf16_bits(xv), wc, ws, f32_to_bf16_bits(bias))
    assert np.array_equal(y, xv @ wv.T + bias)
    assert np.array_equal(ybf, f32_to_bf16_bits(xv @ wv.T + bias))


def test_w4a16_bruteforce_tiny(oracle_mod):
    """Exact rational evaluation of sum_k x q s + b, then the nearest bf16."""
    O = oracle_mod
    rng = np.random.default_rng(22)
    M, K, N = 2, 128, 3
    x = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    w = f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.1)
    b = f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32))
    wc, ws = O.int4_quantize(w, None)
    y, ybf = O.w4a16_linear(x, wc, ws, b)
    nib = [[(int(wc[n, k // 2]) >> (4 * (k & 1))) & 15 for k in range(K)] for n in range(N)]
    for m in range(M):
        for n in range(N):
            acc = Fraction(float(bf16_bits_to_f64(b[n])))
            for k in range(K):
                q = nib[n][k] - 16 if nib[n][k] >= 8 else nib[n][k]
                acc += Fraction(float(bf16_bits_to_f64(x[m, k]))) * q * Fraction(float(bf16_bits_to_f64(ws[n, k // 64])))
            assert abs(Fraction(y[m, n]) - acc) <= abs(acc) * Fraction(1, 2 ** 45) + Fraction(1, 2 ** 80)
            assert ybf[m, n] == brute_bf16(float(acc))


def test_w4a16_is_linear_in_x_and_bias_free_at_zero(oracle_mod):
    """y(2x) = 2 y(x) exactly (power-of-two scaling), y(0) = b, and the rows
    are independent (a row subset equals the same rows of the full call)."""
    O = oracle_mod
    rng = np.random.default_rng(23)
    M, K, N = 5, 256, 7
    xf = rng.standard_normal((M, K)).astype(np.float32)
    w = f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32))
    b = f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32))
    wc, ws = O.int4_quantize(w, None)
    y1, _ = O.w4a16_linear(f32_to_bf16_bits(xf), wc, ws, None)
    y2, _ = O.w4a16_linear(f32_to_bf16_bits(2 * xf), wc, ws, None)
    assert np.array_equal(y2, 2 * y1)
    y0, y0bf = O.w4a16_linear(np.zeros((M, K), np.uint16), wc, ws, b)
    assert np.array_equal(y0bf, np.broadcast_to(b, (M, N)))
    rows = np.array([4, 1])
    ys, _ = O.w4a16_linear(f32_to_bf16_bits(xf), wc, ws, b, rows=rows)
    yf, _ = O.w4a16_linear(f32_to_bf16_bits(xf), wc, ws, b)
    assert np.array_equal(ys, yf[rows])


# ------------------------------------------------------------ GELU MLP pins
# Standard normal CDF values (textbook tables): Phi(1), Phi(-3), Phi(2).
PHI_1, PHI_M3, PHI_2 = 0.8413447460685429, 0.0013498980316300946, 0.9772498680518208


def test_gelu_exact_form_table_values(oracle_mod):
    """GELU(x) = x Phi(x): checked against tabulated Phi and its limits."""
    O = oracle_mod
    assert O.gelu(0.0, 0) == 0.0
    assert abs(O.gelu(1.0, 0) - PHI_1) <= 1e-15
    assert abs(O.gelu(-3.0, 0) - (-3.0 * PHI_M3)) <= 1e-17
    assert abs(O.gelu(2.0, 0) - 2.0 * PHI_2) <= 4e-16
    assert O.gelu(10.0, 0) == 10.0                       # Phi(10) rounds to 1
    v = O.gelu(-10.0, 0)                                 # -10 Phi(-10) = -7.6e-23: the tail keeps its digits
    assert v < 0 and abs(v / -7.619853024160527e-23 - 1) < 1e-9


def test_gelu_odd_part_identity(oracle_mod):
    """Phi(x) + Phi(-x) = 1 gives GELU(x) - GELU(-x) = x, for both forms
    (the tanh form's sigmoid obeys the same symmetry)."""
    O = oracle_mod
    rng = np.random.default_rng(31)
    for x in rng.uniform(-6, 6, 200):
        for approx in (0, 1):
            d = O.gelu(float(x), approx) - O.gelu(float(-x), approx)
            assert abs(d - x) <= 4e-15 * max(1.0, abs(x)), (x, approx)


def test_gelu_tanh_form_is_close_to_exact_form(oracle_mod):
    """The tanh form approximates x Phi(x) to a few 1e-4 over the real line;
    a wrong constant (sqrt(2/pi), 0.044715) moves it well beyond."""
    O = oracle_mod
    xs = np.linspace(-8, 8, 3201)
    err = max(abs(O.gelu(float(x), 1) - O.gelu(float(x), 0)) for x in xs)
    assert 1e-5 < err < 5e-4
    # at x = 1 the tanh form is 0.5 (1 + tanh(sqrt(2/pi) 1.044715))
    assert abs(O.gelu(1.0, 1) - 0.5 * (1 + np.tanh(np.sqrt(2 / np.pi) * 1.044715))) <= 1e-15


def test_gelu_bf16_rounds_once(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(32)
    x = f32_to_bf16_bits(np.concatenate([rng.standard_normal(300) * 3, [0.0, -0.0, 40.0, -40.0]]).astype(np.float32))
    for approx in (0, 1):
        out = O.gelu_bf16(x, approx)
        for i in range(0, x.size, 7):
            assert out[i] == brute_bf16(O.gelu(float(bf16_bits_to_f64(x[i])), approx)), (i, approx)


def test_gelu_mlp_saturated_negative_gives_fc2_bias(oracle_mod):
    """fc1 outputs near -100 make h = GELU(y1) = -0 exactly, so fc2 quantizes an
    all-zero activation (codes 0x88, zero scales, no rank-r term) and its
    output is its bias, bit for bit."""
    O = oracle_mod
    rng = np.random.default_rng(33)
    M, D, Hd, r = 4, 64, 128, 16

    def layer(N, K, bias):
        return {"lam": rng.uniform(0.5, 2, K).astype(np.float32),
                "R": f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 1e-3),
                "L_down": f32_to_bf16_bits(rng.standard_normal((K, r)).astype(np.float32) * 1e-3),
                "L_up": f32_to_bf16_bits(rng.standard_normal((r, N)).astype(np.float32) * 1e-3),
                "b": f32_to_bf16_bits(bias.astype(np.float32))}

    fc1 = layer(Hd, D, np.full(Hd, -100.0))
    fc2 = layer(D, Hd, rng.standard_normal(D))
    x = f32_to_bf16_bits(rng.standard_normal((M, D)).astype(np.float32))
    r1, h, r2 = O.gelu_mlp(x, fc1, fc2, S_x1=0.01, S_x2=0.01)
    assert np.all(h == 0x8000)
    assert np.all(r2.x_codes == 0x88) and np.all(r2.x_scales == 0)
    assert np.array_equal(r2.y_bf16, np.broadcast_to(fc2["b"], (M, D)))
    # rows are independent
    _, h1, r2b = O.gelu_mlp(x, fc1, fc2, S_x1=0.01, S_x2=0.01, rows=[3, 1])
    assert np.array_equal(r2b.y_bf16, r2.y_bf16[[3, 1]])


# ------------------------------------------- fused QKV + RMSNorm + RoPE pins
def _bf16_weights(rng, D):
    return f32_to_bf16_bits(rng.uniform(0.5, 1.5, size=D).astype(np.float32))


def test_rms_norm_closed_forms(oracle_mod):
    """A constant head vector c normalises to c / sqrt(c^2 + eps) * w; an
    alternating +-a vector to +-a / sqrt(a^2 + eps) * w."""
    O = oracle_mod
    rng = np.random.default_rng(11)
    D, eps = 128, 1e-6
    w = _bf16_weights(rng, D)
    wv = bf16_bits_to_f64(w)
    for c in (3.0, -0.25, 1e-2):
        out = O.rms_norm_head(np.full(D, c), w, eps)
        np.testing.assert_allclose(out, c / np.sqrt(c * c + eps) * wv, rtol=1e-14)
    a = 2.5
    v = np.where(np.arange(D) % 2 == 0, a, -a)
    np.testing.assert_allclose(O.rms_norm_head(v, w, eps), v / np.sqrt(a * a + eps) * wv, rtol=1e-14)
    # eps matters for a zero vector: no division by zero, result zero
    assert not np.any(O.rms_norm_head(np.zeros(D), w, eps))


def test_rope_identity_at_angle_zero(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(12)
    v = rng.standard_normal(128)
    assert np.array_equal(O.rope_head(v, np.ones(64), np.zeros(64)), v)


def test_rope_is_complex_rotation(oracle_mod):
    """Pair (2i, 2i+1) read as the complex number v[2i] + j v[2i+1], multiplied
    by exp(j theta_i): a sign or index mistake in either component fails."""
    O = oracle_mod
    rng = np.random.default_rng(13)
    v = rng.standard_normal(128)
    th = rng.uniform(-np.pi, np.pi, size=64)
    out = O.rope_head(v, np.cos(th), np.sin(th))
    z = (v[0::2] + 1j * v[1::2]) * np.exp(1j * th)
    np.testing.assert_allclose(out[0::2], z.real, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out[1::2], z.imag, rtol=0, atol=1e-14)
    # a quarter turn maps (a, b) to (-b, a)
    q = O.rope_head(v, np.zeros(64), np.ones(64))
    assert np.array_equal(q[0::2], -v[1::2]) and np.array_equal(q[1::2], v[0::2])


def test_rope_preserves_pair_norms_and_composes(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(14)
    v = rng.standard_normal(128)
    t1, t2 = rng.uniform(-3, 3, size=64), rng.uniform(-3, 3, size=64)
    r1 = O.rope_head(v, np.cos(t1), np.sin(t1))
    np.testing.assert_allclose(np.hypot(r1[0::2], r1[1::2]), np.hypot(v[0::2], v[1::2]), rtol=1e-14)
    r12 = O.rope_head(r1, np.cos(t2), np.sin(t2))
    r_sum = O.rope_head(v, np.cos(t1 + t2), np.sin(t1 + t2))
    np.testing.assert_allclose(r12, r_sum, rtol=0, atol=1e-13)


def test_qkv_norm_rope_layout(oracle_mod):
    """Q is columns [0, HD), K [HD, 2HD), V [2HD, 3HD) and passes through; Q
    heads take the Q weight, K heads the K weight, each row its own angles;
    the bf16 output is the rounding of the fp64 one."""
    O = oracle_mod
    rng = np.random.default_rng(15)
    H, D, rows, eps = 3, 128, 5, 1e-6
    y = rng.standard_normal((rows, 3 * H * D)) * 4.0
    wq, wk = _bf16_weights(rng, D), _bf16_weights(rng, D)
    th = rng.uniform(-np.pi, np.pi, size=(rows, D // 2))
    out, outb = O.qkv_norm_rope(y, H, D, wq, wk, eps, np.cos(th), np.sin(th))
    assert np.array_equal(out[:, 2 * H * D:], y[:, 2 * H * D:])
    for m in (0, rows - 1):
        for part, w in ((0, wq), (1, wk)):
            for h in (0, H - 1):
                cols = slice(part * H * D + h * D, part * H * D + (h + 1) * D)
                want = O.rope_head(O.rms_norm_head(y[m, cols], w, eps), np.cos(th[m]), np.sin(th[m]))
                assert np.array_equal(out[m, cols], want)
    assert all(outb[m, n] == O.bf16_from_double(float(out[m, n])) for m in range(rows) for n in range(0, 3 * H * D, 97))


# ------------------------------------------------------- SVD split pins
def test_svd_split_eckart_young(oracle_mod):
    """The residual of the best rank-r approximation: ||R||_F^2 is the sum of
    the squared singular values past r, ||R||_2 the (r+1)-th; W_hat is
    reassembled exactly; L_down has orthonormal columns, L_up orthogonal rows
    of norms s_i."""
    O = oracle_mod
    rng = np.random.default_rng(31)
    N, K, r = 48, 40, 6
    W = f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32))
    lam = rng.uniform(0.5, 4.0, size=K).astype(np.float32)
    R, Ld, Lu, s = O.svd_split(W, lam, r)
    W_hat = bf16_bits_to_f64(W) * lam.astype(np.float64)[None, :]
    np.testing.assert_allclose(R + Lu.T @ Ld.T, W_hat, rtol=0, atol=1e-12)
    assert np.linalg.norm(R) ** 2 == pytest.approx(float(np.sum(s[r:] ** 2)), rel=1e-10)
    assert np.linalg.norm(R, 2) == pytest.approx(float(s[r]), rel=1e-10)
    np.testing.assert_allclose(Ld.T @ Ld, np.eye(r), atol=1e-12)
    np.testing.assert_allclose(Lu @ Lu.T, np.diag(s[:r] ** 2), atol=1e-9 * s[0] ** 2)
    assert np.all(np.diff(s) <= 0)


def test_svd_split_low_rank_weight(oracle_mod):
    """A weight that is rank r up to its bf16 rounding: the residual is no
    larger than that rounding (the truncation is the best rank-r fit)."""
    O = oracle_mod
    rng = np.random.default_rng(32)
    N, K, r = 64, 48, 5
    exact = rng.standard_normal((N, r)) @ rng.standard_normal((r, K))
    W = f32_to_bf16_bits(exact.astype(np.float32))
    R, _, _, s = O.svd_split(W, np.ones(K, np.float32), r)
    assert np.linalg.norm(R) <= np.linalg.norm(bf16_bits_to_f64(W) - exact) * (1 + 1e-9)
    # rank 0 leaves the whole smoothed weight in R
    lam = rng.uniform(0.5, 4.0, size=K).astype(np.float32)
    R0, Ld0, Lu0, _ = O.svd_split(W, lam, 0)
    assert np.array_equal(R0, bf16_bits_to_f64(W) * lam.astype(np.float64)[None, :])
    assert Ld0.shape == (K, 0) and Lu0.shape == (0, N)
