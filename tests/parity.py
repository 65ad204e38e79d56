"""Helpers shared by the parity tests: run the CUDA path through the C ABI and
run the oracle on the same seeded inputs, then compare.

The library's packed layouts are translated back to the oracle's logical
layouts here, with index maps written out independently of the CUDA code.
"""
from __future__ import annotations

import numpy as np
import torch

from bit_w4a4_quantized_token_b200 import workloads as W
from oracle import oracle as O


# ------------------------------------------------------------ layouts
def nvfp4_scale_index(rows: int, K: int) -> np.ndarray:
    """Byte offsets of the (row, group) scales in the tensor-core scale layout:
    512-byte blocks of 128 rows x 4 groups; inside a block the byte of
    (row r, group g) is at (r % 32) * 16 + ((r % 128) // 32) * 4 + g % 4."""
    kg = K // 16
    r = np.arange(rows)[:, None]
    g = np.arange(kg)[None, :]
    block = (r // 128) * (kg // 4) + g // 4
    return block * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + g % 4


def unswizzle_nvfp4_scales(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    return np.asarray(buf, np.uint8).reshape(-1)[nvfp4_scale_index(rows, K)]


def nvfp4_scale_padding_is_zero(buf: np.ndarray, rows: int, K: int) -> bool:
    rows_pad = (rows + 127) // 128 * 128
    idx = nvfp4_scale_index(rows_pad, K)[rows:]
    return not np.asarray(buf, np.uint8).reshape(-1)[idx].any()


def replicate_nvfp4_weight_scales(buf: np.ndarray, N: int, K: int) -> np.ndarray:
    """The GEMM-ready copy of nvfp4 weight scales (the C header's "nvfp4 weight
    scales" layout) built from the block layout at the start of `buf`: per
    256-row tile t and 256 columns kb, per k-step k, each 16-byte row l of the
    blocks (2t+h, 4kb+k) four times, at (4q + l/8)*256 + h*128 + (l%8)*16."""
    kg4, n_rb = K // 64, (N + 127) // 128
    n_t, n_kb = (N + 255) // 256, (K + 255) // 256
    blocks = np.zeros((2 * n_t, 4 * n_kb, 32, 16), np.uint8)
    blocks[:n_rb, :kg4] = np.asarray(buf, np.uint8).reshape(-1)[: n_rb * kg4 * 512].reshape(n_rb, kg4, 32, 16)
    b = blocks.reshape(n_t, 2, n_kb, 4, 4, 8, 16)                 # t, h, kb, k, l/8, l%8, byte
    b = b.transpose(0, 2, 3, 4, 1, 5, 6)                          # t, kb, k, l/8, h, l%8, byte
    rep = np.broadcast_to(b[:, :, :, None], (n_t, n_kb, 4, 4, 4, 2, 8, 16))   # q before l/8
    return np.ascontiguousarray(rep).reshape(-1)


def unswizzle_int4_scales(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """int4 scales are bf16, group-major: element (r, g) at g * rows_pad + r."""
    rows_pad = (rows + 127) // 128 * 128
    flat = np.asarray(buf, np.uint8).reshape(-1).view(np.uint16)
    return flat[: (K // 64) * rows_pad].reshape(K // 64, rows_pad)[:, :rows].T.copy()


# ------------------------------------------------------------ comparisons
def bf16_ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in units in the last place between two bf16 arrays (bit patterns)."""
    # map sign-magnitude to a monotone integer line
    def mono(x):
        x = np.asarray(x, np.uint16).astype(np.int32)
        mag = x & 0x7FFF
        return np.where(x & 0x8000, -mag, mag)
    return np.abs(mono(a_bits) - mono(b_bits))


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |v| (the error of rounding v to bf16)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 8)


def check_y(y_gpu_bits: np.ndarray, y_ref: np.ndarray, y_ref_bits: np.ndarray, what: str = "y",
            min_frac1: float = 0.999) -> dict:
    """The output bar.

    1. max_i (|y_gpu - y_ref| - half_ulp_bf16(y_ref)) <= 1e-2 rms(y_ref): the
       error beyond the unavoidable rounding of the exact fp64 value y_ref to
       the bf16 output is at most 1 % of the output rms.  (Half a bf16 ulp of
       the largest outputs is itself more than 1 % of the rms, so the bound
       cannot apply to the rounding of the bf16 store.)
    2. the bf16 output is within 1 ulp of the oracle's own bf16 rounding of
       y_ref on >= min_frac1 of the elements (99.9 % for a layer given the
       same inputs as the oracle).
    """
    y_gpu = (np.asarray(y_gpu_bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite outputs"
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = np.abs(y_gpu - y_ref)
    excess = float(np.max(err - bf16_half_ulp(y_ref)))
    ulps = bf16_ulp_distance(y_gpu_bits, y_ref_bits)
    frac1 = float(np.mean(ulps <= 1))
    stats = {"rms": rms, "max_abs_err": float(err.max()), "max_excess_over_half_ulp_rel_rms": excess / rms,
             "frac_within_1ulp": frac1, "max_ulps": int(ulps.max())}
    assert excess <= 1e-2 * rms, f"{what}: {stats}"
    assert frac1 >= min_frac1, f"{what}: {stats}"
    return stats


def check_lowrank(L_gpu: torch.Tensor, L_ref: np.ndarray, prescale: float) -> float:
    """Rank-r activations (hi + lo bf16 planes) within 1e-2 relative rms."""
    planes = L_gpu.double().cpu().numpy()
    got = (planes[0] + planes[1]) * prescale
    err = float(np.sqrt(np.mean((got - L_ref) ** 2)) / max(np.sqrt(np.mean(L_ref ** 2)), 1e-30))
    assert err <= 1e-2, err
    return err


# ------------------------------------------------------------ running
def to_dev(inp: dict, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def run_gpu(case: W.Case, inp: dict, x_tensor_scale=None, with_bias=True):
    from bit_w4a4_quantized_token_b200 import layer

    d = to_dev(inp)
    r = case.rank
    packed = layer.pack_weight(d["R"], d["lam"], d["L_down"] if r else None, d["L_up"] if r else None,
                               d["b"] if with_bias else None, precision=case.precision)
    q = layer.quantize_act(d["x"], packed, x_tensor_scale=x_tensor_scale)
    y = layer.gemm(q, packed)
    torch.cuda.synchronize()
    return packed, q, y


def oracle_for(case: W.Case, inp: dict, rows=None, S_x=None, with_bias=True, with_y=True):
    r = case.rank
    return O.svdq_linear(case.precision, W.bits(inp["x"]), inp["lam"].numpy(), W.bits(inp["R"]),
                         W.bits(inp["L_down"]) if r else None, W.bits(inp["L_up"]) if r else None,
                         W.bits(inp["b"]) if with_bias else None, S_x=S_x, rows=rows, with_y=with_y)


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_case(case: W.Case, rows=None, x_tensor_scale=None, with_bias=True, inp=None) -> dict:
    """Full comparison of one case; rows=None compares every output row."""
    inp = W.make_inputs(case) if inp is None else inp
    packed, q, y = run_gpu(case, inp, x_tensor_scale=x_tensor_scale, with_bias=with_bias)
    M, K, N = case.M, case.K, case.N
    S_x = None if x_tensor_scale is None else float(np.float32(x_tensor_scale))
    ref = oracle_for(case, inp, rows=rows, S_x=S_x, with_bias=with_bias)
    out = {}
    # codes and scales: bit-exact
    assert np.array_equal(packed.w_codes.cpu().numpy().reshape(N, K // 2), ref.w_codes), "weight codes"
    assert np.array_equal(q.x_codes.cpu().numpy().reshape(M, K // 2), ref.x_codes), "activation codes"
    if case.precision == "nvfp4":
        assert float(packed.w_tensor_scale[0]) == np.float32(ref.S_w), "S_w"
        assert float(q.x_tensor_scale[0]) == np.float32(ref.S_x), "S_x"
        ws = packed.w_scales.cpu().numpy()
        xs = q.x_scales.cpu().numpy()
        assert np.array_equal(unswizzle_nvfp4_scales(ws, N, K), ref.w_scales), "weight scales"
        assert np.array_equal(unswizzle_nvfp4_scales(xs, M, K), ref.x_scales), "activation scales"
        assert nvfp4_scale_padding_is_zero(ws, N, K) and nvfp4_scale_padding_is_zero(xs, M, K)
        sb = (N + 127) // 128 * 128 * K // 16
        assert np.array_equal(ws[sb:], replicate_nvfp4_weight_scales(ws, N, K)), "GEMM-ready weight scales"
        prescale = float(np.float32(ref.S_x) * np.float32(ref.S_w))
    else:
        assert np.array_equal(unswizzle_int4_scales(packed.w_scales.cpu().numpy(), N, K), ref.w_scales)
        assert np.array_equal(unswizzle_int4_scales(q.x_scales.cpu().numpy(), M, K), ref.x_scales)
        prescale = 1.0
    if case.rank:
        out["lowrank_rel_rms"] = check_lowrank(q.lowrank_act, ref.L, prescale)
    ybits = u16(y)
    if rows is not None:
        ybits = ybits[np.asarray(rows)]
    out.update(check_y(ybits, ref.y, ref.y_bf16))
    return out


def sample_rows(M: int, n: int = 48, seed: int = 0) -> np.ndarray:
    """Rows spread over every 128-row tile position plus the ragged tail."""
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, size=min(n, M), replace=False).tolist())
    rows.update([0, 31, 32, 63, 64, 95, 96, 127, M - 1, M - 2])
    return np.array(sorted(r for r in rows if 0 <= r < M))
