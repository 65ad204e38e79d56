"""CPU oracle of the SVDQuant W4A4 linear layer (Python face of svdq_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this module.  It shares no
code with the CUDA library and never imports it.

Every function works on the plain logical layouts (row-major arrays; two 4-bit
codes per byte with the even k in the low nibble; one scale per (row, group)).
The arithmetic lives in ``svdq_oracle.c``; this file only marshals numpy
arrays and composes the steps in the order the layer defines them:

    y = dequant(Q4(x/lambda)) . dequant(Q4(R))^T + ((x/lambda) . L_down) . L_up + b

(the ``svdq_w4a4`` layer of the Diffusers docs page "Nunchaku Lite", section
"Supported quantization types": nvfp4 with group 16, int4 with group 64, both
with the SVDQ low-rank correction; rank 32 in the config schema section).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svdq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

NVFP4_GROUP = 16
INT4_GROUP = 64


def build(force: bool = False) -> str:
    """Compile svdq_oracle.c into liboracle.so (IEEE fp32, no contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        L = ctypes.c_long
        D = ctypes.c_double
        lib.oracle_rms_norm_head.argtypes = [P, L, P, D]
        lib.oracle_rms_norm_head.restype = None
        lib.oracle_rope_head.argtypes = [P, L, P, P]
        lib.oracle_rope_head.restype = None
        lib.oracle_qkv_norm_rope.argtypes = [P, L, L, L, P, P, D, P, P, P, P]
        lib.oracle_qkv_norm_rope.restype = None
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_from_double.argtypes = [ctypes.c_double]
        lib.oracle_bf16_from_double.restype = ctypes.c_uint16
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.oracle_e2m1_encode.restype = ctypes.c_int
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_int]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_int
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_int]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_nvfp4_tensor_scale.argtypes = [P, P, L, L]
        lib.oracle_nvfp4_tensor_scale.restype = ctypes.c_float
        lib.oracle_nvfp4_quantize.argtypes = [P, P, L, L, ctypes.c_float, P, P]
        lib.oracle_nvfp4_quantize.restype = None
        lib.oracle_nvfp4_dequant.argtypes = [P, P, ctypes.c_float, L, L, P]
        lib.oracle_nvfp4_dequant.restype = None
        lib.oracle_int4_quantize.argtypes = [P, P, L, L, P, P]
        lib.oracle_int4_quantize.restype = None
        lib.oracle_lowrank_down.argtypes = [P, P, L, L, P, L, P]
        lib.oracle_lowrank_down.restype = None
        lib.oracle_nvfp4_linear.argtypes = [P, P, L, L, P, L, P, P, L, P, P, P]
        lib.oracle_nvfp4_linear.restype = None
        lib.oracle_int4_linear.argtypes = [P, P, P, L, L, P, P, L, P, P, L, P, P, P]
        lib.oracle_int4_linear.restype = None
        lib.oracle_w4a16_linear.argtypes = [P, P, L, L, P, P, L, P, P, P]
        lib.oracle_w4a16_linear.restype = None
        lib.oracle_gelu.argtypes = [D, ctypes.c_int]
        lib.oracle_gelu.restype = D
        lib.oracle_gelu_bf16.argtypes = [P, L, ctypes.c_int, P]
        lib.oracle_gelu_bf16.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    """bf16 data is carried as its uint16 bit pattern."""
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


# ---------------------------------------------------------------- scalars
def bf16_to_float(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to fp64."""
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_from_double(d: float) -> int:
    return int(_load().oracle_bf16_from_double(float(d)))


def e2m1_encode(v: float) -> int:
    return int(_load().oracle_e2m1_encode(float(v)))


def e2m1_decode(code: int) -> float:
    return float(_load().oracle_e2m1_decode(int(code)))


def e4m3_encode(v: float) -> int:
    return int(_load().oracle_e4m3_encode(float(v)))


def e4m3_decode(byte: int) -> float:
    return float(_load().oracle_e4m3_decode(int(byte)))


# ------------------------------------------------------------------ nvfp4
def nvfp4_tensor_scale(x_bits: np.ndarray, lam: np.ndarray | None) -> float:
    """S = fl32(amax|x/lambda| / 2688) (1 for an all-zero tensor)."""
    x_bits = _u16(x_bits)
    rows, K = x_bits.shape
    lam = _f32(lam)
    return float(_load().oracle_nvfp4_tensor_scale(_ptr(x_bits), _ptr(lam), rows, K))


def nvfp4_quantize(x_bits: np.ndarray, lam: np.ndarray | None, S: float):
    """Return (codes [rows, K/2] u8, scales [rows, K/16] u8 E4M3)."""
    x_bits = _u16(x_bits)
    rows, K = x_bits.shape
    assert K % NVFP4_GROUP == 0
    lam = _f32(lam)
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // NVFP4_GROUP), np.uint8)
    _load().oracle_nvfp4_quantize(_ptr(x_bits), _ptr(lam), rows, K, float(S), _ptr(codes), _ptr(scales))
    return codes, scales


def nvfp4_dequant(codes: np.ndarray, scales: np.ndarray, S: float) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((rows, K), np.float64)
    _load().oracle_nvfp4_dequant(_ptr(codes), _ptr(scales), float(S), rows, K, _ptr(out))
    return out


# ------------------------------------------------------------------- int4
def int4_quantize(x_bits: np.ndarray, lam: np.ndarray | None):
    """Return (codes [rows, K/2] u8 two's-complement nibbles, scales [rows, K/64] bf16 bits)."""
    x_bits = _u16(x_bits)
    rows, K = x_bits.shape
    assert K % INT4_GROUP == 0
    lam = _f32(lam)
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // INT4_GROUP), np.uint16)
    _load().oracle_int4_quantize(_ptr(x_bits), _ptr(lam), rows, K, _ptr(codes), _ptr(scales))
    return codes, scales


def int4_codes_to_int(codes: np.ndarray) -> np.ndarray:
    """Unpack two's-complement nibbles to int8 values [rows, K]."""
    codes = np.asarray(codes, np.uint8)
    lo = (codes & 15).astype(np.int16)
    hi = (codes >> 4).astype(np.int16)
    q = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    return np.where(q >= 8, q - 16, q).astype(np.int8)


# ----------------------------------------------------------- rank-r branch
def lowrank_down(x_bits: np.ndarray, lam: np.ndarray, L_down_bits: np.ndarray) -> np.ndarray:
    """L = (x / lambda) . L_down in fp64, shape [M, r]."""
    x_bits = _u16(x_bits)
    L_down_bits = _u16(L_down_bits)
    M, K = x_bits.shape
    r = L_down_bits.shape[1] if L_down_bits.ndim == 2 else 0
    out = np.zeros((M, max(r, 0)), np.float64)
    if r == 0:
        return out
    _load().oracle_lowrank_down(_ptr(x_bits), _ptr(_f32(lam)), M, K, _ptr(L_down_bits), r, _ptr(out))
    return out


# ------------------------------------------------------------------- GEMM
def nvfp4_linear(xd: np.ndarray, wd: np.ndarray, L: np.ndarray | None, L_up_bits: np.ndarray | None,
                 bias_bits: np.ndarray | None, rows: np.ndarray | None = None):
    """fp64 y and its bf16 bits for the chosen rows of the dequantized x."""
    xd = np.ascontiguousarray(xd, np.float64)
    wd = np.ascontiguousarray(wd, np.float64)
    K = xd.shape[1]
    N = wd.shape[0]
    r = 0 if L is None else L.shape[1]
    rows_arr = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nrows = xd.shape[0] if rows is None else len(rows_arr)
    y = np.zeros((nrows, N), np.float64)
    ybf = np.zeros((nrows, N), np.uint16)
    Lc = None if r == 0 else np.ascontiguousarray(L, np.float64)
    Lu = None if r == 0 else _u16(L_up_bits)
    b = None if bias_bits is None else _u16(bias_bits)
    _load().oracle_nvfp4_linear(_ptr(xd), _ptr(rows_arr), nrows, K, _ptr(wd), N, _ptr(Lc), _ptr(Lu), r,
                                _ptr(b), _ptr(y), _ptr(ybf))
    return y, ybf


def int4_linear(xc, xs, wc, ws, L, L_up_bits, bias_bits, rows=None):
    xc = np.ascontiguousarray(xc, np.uint8)
    wc = np.ascontiguousarray(wc, np.uint8)
    xs = _u16(xs)
    ws = _u16(ws)
    K = xc.shape[1] * 2
    N = wc.shape[0]
    r = 0 if L is None else L.shape[1]
    rows_arr = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nrows = xc.shape[0] if rows is None else len(rows_arr)
    y = np.zeros((nrows, N), np.float64)
    ybf = np.zeros((nrows, N), np.uint16)
    Lc = None if r == 0 else np.ascontiguousarray(L, np.float64)
    Lu = None if r == 0 else _u16(L_up_bits)
    b = None if bias_bits is None else _u16(bias_bits)
    _load().oracle_int4_linear(_ptr(xc), _ptr(xs), _ptr(rows_arr), nrows, K, _ptr(wc), _ptr(ws), N,
                               _ptr(Lc), _ptr(Lu), r, _ptr(b), _ptr(y), _ptr(ybf))
    return y, ybf


def w4a16_linear(x_bits, wc, ws, bias_bits, rows=None):
    """Weight-only int4: y = x . (q s)^T + b in fp64 and its bf16 bits.

    x_bits [M, K] bf16 bits used as they are; wc [N, K/2] two's-complement
    nibbles and ws [N, K/64] bf16 bits as ``int4_quantize`` returns them.
    """
    x_bits = _u16(x_bits)
    wc = np.ascontiguousarray(wc, np.uint8)
    ws = _u16(ws)
    K = x_bits.shape[1]
    N = wc.shape[0]
    rows_arr = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nrows = x_bits.shape[0] if rows is None else len(rows_arr)
    y = np.zeros((nrows, N), np.float64)
    ybf = np.zeros((nrows, N), np.uint16)
    b = None if bias_bits is None else _u16(bias_bits)
    _load().oracle_w4a16_linear(_ptr(x_bits), _ptr(rows_arr), nrows, K, _ptr(wc), _ptr(ws), N, _ptr(b),
                                _ptr(y), _ptr(ybf))
    return y, ybf


# ------------------------------------------------------------- GELU MLP
def gelu(x: float, approx: int = 0) -> float:
    """GELU of one value in fp64 (approx 0: x Phi(x); 1: the tanh form)."""
    return float(_load().oracle_gelu(float(x), int(approx)))


def gelu_bf16(x_bits: np.ndarray, approx: int = 0) -> np.ndarray:
    """bf16 bits -> GELU in fp64 -> bf16 bits (one rounding)."""
    x_bits = _u16(x_bits)
    out = np.zeros_like(x_bits)
    _load().oracle_gelu_bf16(_ptr(x_bits), x_bits.size, int(approx), _ptr(out))
    return out


def gelu_mlp(x_bits, fc1: dict, fc2: dict, S_x1: float, S_x2: float, approx: int = 0, rows=None):
    """The DiT MLP block fc1 -> GELU -> fc2 with both linears SVDQ W4A4 nvfp4
    layers: y1 = fc1(x) rounded to bf16, h = bf16(GELU(y1)), and fc2 applied
    to h with its static activation tensor scale S_x2 (the fused kernel of the
    Diffusers docs page "Nunchaku Lite", section "Fused kernels", hands the
    same h to fc2's quantizer without writing it out).

    fc1, fc2: dicts of bf16 bits / arrays with keys lam, R, L_down, L_up, b.
    rows: optional subset of token rows (the MLP is row-wise).
    Returns (fc1 result, h bits, fc2 result) for the chosen rows."""
    x_bits = _u16(x_bits)
    if rows is not None:
        x_bits = np.ascontiguousarray(x_bits[np.asarray(rows)])
    r1 = svdq_linear("nvfp4", x_bits, fc1["lam"], fc1["R"], fc1["L_down"], fc1["L_up"], fc1["b"], S_x=S_x1)
    h = gelu_bf16(r1.y_bf16, approx)
    r2 = svdq_linear("nvfp4", h, fc2["lam"], fc2["R"], fc2["L_down"], fc2["L_up"], fc2["b"], S_x=S_x2)
    return r1, h, r2


# --------------------------------------------- fused QKV + RMSNorm + RoPE
def rms_norm_head(v: np.ndarray, w_bits: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm of one head vector (fp64) with bf16 weights."""
    out = np.ascontiguousarray(v, np.float64).copy()
    _load().oracle_rms_norm_head(_ptr(out), out.shape[0], _ptr(_u16(w_bits)), float(eps))
    return out


def rope_head(v: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotary embedding of one head vector (fp64): pair i rotates by (cos[i], sin[i])."""
    out = np.ascontiguousarray(v, np.float64).copy()
    _load().oracle_rope_head(_ptr(out), out.shape[0], _ptr(np.ascontiguousarray(cos, np.float64)),
                             _ptr(np.ascontiguousarray(sin, np.float64)))
    return out


def qkv_norm_rope(y: np.ndarray, heads: int, head_dim: int, wq_bits, wk_bits, eps: float,
                  cos: np.ndarray, sin: np.ndarray):
    """Per-head RMSNorm and RoPE of the Q and K columns of a to_qkv output.

    y [rows, 3 * heads * head_dim] fp64 (the linear layer's exact output);
    cos, sin [rows, head_dim / 2] the tokens' rotary tables.  Returns the fp64
    result and its bf16 bits (V columns pass through)."""
    y = np.ascontiguousarray(y, np.float64)
    rows, N = y.shape
    assert N == 3 * heads * head_dim
    out = np.zeros_like(y)
    outb = np.zeros(y.shape, np.uint16)
    _load().oracle_qkv_norm_rope(_ptr(y), rows, heads, head_dim, _ptr(_u16(wq_bits)), _ptr(_u16(wk_bits)),
                                 float(eps), _ptr(np.ascontiguousarray(cos, np.float64)),
                                 _ptr(np.ascontiguousarray(sin, np.float64)), _ptr(out), _ptr(outb))
    return out, outb


# ------------------------------------------------ offline SVDQuant split
def svd_split(W_bits: np.ndarray, lam: np.ndarray, rank: int):
    """The offline split of the SVDQuant paper that the Diffusers docs page
    "Nunchaku Lite" builds on (introduction; the tutorial's quantize_hf.py
    --rank 32 step): the smoothed weight W_hat = W diag(lambda) [N, K] is
    split into its best rank-r approximation (the truncated SVD) and the
    residual R = W_hat - L_up^T L_down^T, so that
        x W^T = (x / lambda) W_hat^T = (x / lambda) R^T + ((x / lambda) L_down) L_up.
    Returns (R [N, K], L_down [K, r], L_up [r, N], singular values), fp64;
    the factors are unique up to the signs of singular-vector pairs, their
    product and R are unique when s_r > s_{r+1}.  A library SVD (LAPACK
    through numpy) is the step that computes the decomposition."""
    W = bf16_to_float(_u16(W_bits)).astype(np.float64)
    W_hat = W * np.asarray(lam, np.float64)[None, :]
    U, s, Vt = np.linalg.svd(W_hat, full_matrices=False)
    L_up = (U[:, :rank] * s[:rank]).T
    L_down = Vt[:rank].T
    R = W_hat - L_up.T @ L_down.T
    return R, L_down, L_up, s


# ------------------------------------------------------- whole layer
class OracleResult:
    """Everything the oracle derives for one layer call (logical layouts)."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def svdq_linear(precision: str, x_bits, lam, R_bits, L_down_bits, L_up_bits, bias_bits,
                S_x: float | None = None, rows=None, with_y: bool = True) -> OracleResult:
    """The layer, step by step in the order it is defined.

    precision  "nvfp4" (group 16, E4M3 group scales, fp32 tensor scale) or
               "int4" (group 64, bf16 group scales).
    S_x        nvfp4 activation tensor scale; None computes it from amax.
    rows       optional subset of output rows (all rows when None).
    """
    r = 0 if L_down_bits is None else L_down_bits.shape[1]
    L = lowrank_down(x_bits, lam, L_down_bits) if r else None
    if precision == "nvfp4":
        S_w = nvfp4_tensor_scale(R_bits, None)
        wc, wsc = nvfp4_quantize(R_bits, None, S_w)
        if S_x is None:
            S_x = nvfp4_tensor_scale(x_bits, lam)
        xc, xsc = nvfp4_quantize(x_bits, lam, S_x)
        res = OracleResult(precision=precision, S_x=S_x, S_w=S_w, x_codes=xc, x_scales=xsc,
                           w_codes=wc, w_scales=wsc, L=L)
        if with_y:
            xd = nvfp4_dequant(xc, xsc, S_x)
            wd = nvfp4_dequant(wc, wsc, S_w)
            res.y, res.y_bf16 = nvfp4_linear(xd, wd, L, L_up_bits, bias_bits, rows)
        return res
    if precision == "int4":
        wc, wsc = int4_quantize(R_bits, None)
        xc, xsc = int4_quantize(x_bits, lam)
        res = OracleResult(precision=precision, x_codes=xc, x_scales=xsc, w_codes=wc, w_scales=wsc, L=L)
        if with_y:
            res.y, res.y_bf16 = int4_linear(xc, xsc, wc, wsc, L, L_up_bits, bias_bits, rows)
        return res
    raise ValueError(precision)
