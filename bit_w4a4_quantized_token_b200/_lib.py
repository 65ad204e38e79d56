"""ctypes binding of the C ABI in include/svdq.h (argument marshalling only).

Every function has the name of its C entry point and takes torch tensors
(or None for NULL) plus an optional CUDA stream; it passes their device
pointers to the shared library and raises ``SvdqError`` on any status other
than SVDQ_OK.  No arithmetic of the layer happens here.  If the compiled
library is missing, importing this module fails loudly: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq_b200.so")

SVDQ_OK = 0
SVDQ_ERR_INVALID_ARG = 1
SVDQ_ERR_UNSUPPORTED_SHAPE = 2
SVDQ_ERR_UNSUPPORTED_DEVICE = 3
SVDQ_ERR_CUDA = 4
SVDQ_ERR_TIMEOUT = 5

SVDQ_NVFP4 = 0
SVDQ_INT4 = 1
PRECISIONS = {"nvfp4": SVDQ_NVFP4, "int4": SVDQ_INT4}
GROUP_SIZES = {"nvfp4": 16, "int4": 64}

# Every entry point declared in include/svdq.h.
EXPORTS = (
    "svdq_status_string", "svdq_abi_version", "svdq_last_error", "svdq_buffer_sizes", "svdq_pack_weight",
    "svdq_replicate_weight_scales",
    "svdq_quantize_act_workspace_bytes", "svdq_quantize_act", "svdq_quantize_act_noalloc", "svdq_gemm_w4a4",
    "svdq_gemm_w4a4_qkv_norm_rope", "svdq_qkv_norm_rope", "svdq_gelu_mlp_workspace_bytes",
    "svdq_gemm_w4a4_gelu_quant", "svdq_gemm_w4a4_gelu", "svdq_gelu", "svdq_gemm_w4a16", "svdq_svd_split_workspace_bytes",
    "svdq_svd_split",
    "svdq_device_status",
    "svdq_debug_set_wait_limit_ns", "svdq_debug_timeout_probe", "svdq_debug_override_capability",
    "svdq_debug_force_gemm_tiles", "svdq_debug_force_quant_plan",
)


class SvdqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == SVDQ_ERR_CUDA:
            detail = f" [{lib.svdq_last_error().decode()}]"
        super().__init__(f"{where}: {status_string(status)} (status {status}){detail}")


class svdq_sizes(ctypes.Structure):
    _fields_ = [("codes_bytes", ctypes.c_size_t), ("scales_bytes", ctypes.c_size_t),
                ("lowrank_bytes", ctypes.c_size_t), ("w_scales_bytes", ctypes.c_size_t)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"the CUDA library {LIB_PATH} is not built; run __graft_entry__.build() "
                          "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
    lib.svdq_status_string.argtypes = [I]
    lib.svdq_status_string.restype = ctypes.c_char_p
    lib.svdq_abi_version.argtypes = []
    lib.svdq_abi_version.restype = I
    lib.svdq_last_error.argtypes = []
    lib.svdq_last_error.restype = ctypes.c_char_p
    lib.svdq_buffer_sizes.argtypes = [I, I64, I64, I, ctypes.POINTER(svdq_sizes)]
    lib.svdq_buffer_sizes.restype = I
    lib.svdq_pack_weight.argtypes = [I, I, P, I64, I64, P, P, P, I, P, P, P, P, P, P, P]
    lib.svdq_pack_weight.restype = I
    lib.svdq_replicate_weight_scales.argtypes = [P, I64, I64, P]
    lib.svdq_replicate_weight_scales.restype = I
    lib.svdq_quantize_act_workspace_bytes.argtypes = [I, I64, I64, I, ctypes.POINTER(ctypes.c_size_t)]
    lib.svdq_quantize_act_workspace_bytes.restype = I
    lib.svdq_quantize_act.argtypes = [I, I, P, I64, I64, P, P, I, P, P, I, P, P, P, P, ctypes.c_size_t, P]
    lib.svdq_quantize_act.restype = I
    lib.svdq_quantize_act_noalloc.argtypes = [I, I, P, I64, I64, P, P, I, P, P, I, P, P, P, P]
    lib.svdq_quantize_act_noalloc.restype = I
    lib.svdq_gemm_w4a4.argtypes = [I, I, P, P, P, I64, P, P, P, I64, I64, P, P, I, P, P, P]
    lib.svdq_gemm_w4a4.restype = I
    F = ctypes.c_float
    lib.svdq_gemm_w4a4_qkv_norm_rope.argtypes = [I, I, P, P, P, I64, P, P, P, I64, I64, P, P, I, P, I, I, P, P, F,
                                                 P, P, P, P]
    lib.svdq_gemm_w4a4_qkv_norm_rope.restype = I
    lib.svdq_qkv_norm_rope.argtypes = [P, P, I64, I, I, P, P, F, P, P, P]
    lib.svdq_qkv_norm_rope.restype = I
    lib.svdq_gelu_mlp_workspace_bytes.argtypes = [I64, I, ctypes.POINTER(ctypes.c_size_t)]
    lib.svdq_gelu_mlp_workspace_bytes.restype = I
    lib.svdq_gemm_w4a4_gelu_quant.argtypes = [I, I, P, P, P, I64, P, P, P, I64, I64, P, P, I, P, I, P, P, I, P, P, P,
                                              P, P, P, ctypes.c_size_t, P]
    lib.svdq_gemm_w4a4_gelu_quant.restype = I
    lib.svdq_gemm_w4a4_gelu.argtypes = [I, I, P, P, P, I64, P, P, P, I64, I64, P, P, I, P, I, P, P]
    lib.svdq_gemm_w4a4_gelu.restype = I
    lib.svdq_gelu.argtypes = [P, P, I64, I, P]
    lib.svdq_gelu.restype = I
    lib.svdq_gemm_w4a16.argtypes = [P, I64, P, P, I64, I64, P, P, P]
    lib.svdq_gemm_w4a16.restype = I
    lib.svdq_svd_split_workspace_bytes.argtypes = [I64, I64, I, I, ctypes.POINTER(ctypes.c_size_t)]
    lib.svdq_svd_split_workspace_bytes.restype = I
    lib.svdq_svd_split.argtypes = [P, P, I64, I64, I, P, I, I, P, P, P, P, P, ctypes.c_size_t, P]
    lib.svdq_svd_split.restype = I
    lib.svdq_device_status.argtypes = [I, ctypes.POINTER(ctypes.c_int)]
    lib.svdq_device_status.restype = I
    lib.svdq_debug_set_wait_limit_ns.argtypes = [U64]
    lib.svdq_debug_set_wait_limit_ns.restype = I
    lib.svdq_debug_timeout_probe.argtypes = [P]
    lib.svdq_debug_timeout_probe.restype = I
    lib.svdq_debug_override_capability.argtypes = [I, I]
    lib.svdq_debug_override_capability.restype = None
    lib.svdq_debug_force_gemm_tiles.argtypes = [I]
    lib.svdq_debug_force_gemm_tiles.restype = I
    lib.svdq_debug_force_quant_plan.argtypes = [I]
    lib.svdq_debug_force_quant_plan.restype = I
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.svdq_status_string(int(status)).decode()


def _ptr(t) -> int | None:
    """Device pointer of a tensor (None -> NULL); raw ints pass through."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != SVDQ_OK:
        raise SvdqError(status, where)


def _prec(p) -> int:
    return PRECISIONS[p] if isinstance(p, str) else int(p)


def svdq_abi_version() -> int:
    return int(lib.svdq_abi_version())


def svdq_buffer_sizes(precision, rows: int, K: int, rank: int) -> dict:
    out = svdq_sizes()
    _check(lib.svdq_buffer_sizes(_prec(precision), int(rows), int(K), int(rank), ctypes.byref(out)),
           "svdq_buffer_sizes")
    return {"codes_bytes": out.codes_bytes, "scales_bytes": out.scales_bytes, "lowrank_bytes": out.lowrank_bytes,
            "w_scales_bytes": out.w_scales_bytes}


def svdq_pack_weight(precision, group_size, R, N, K, lam, L_down, L_up, rank, w_codes, w_scales,
                     w_tensor_scale, inv_lambda, L_down_t, L_up_t, stream=None) -> None:
    _check(lib.svdq_pack_weight(_prec(precision), int(group_size), _ptr(R), int(N), int(K), _ptr(lam),
                                _ptr(L_down), _ptr(L_up), int(rank), _ptr(w_codes), _ptr(w_scales),
                                _ptr(w_tensor_scale), _ptr(inv_lambda), _ptr(L_down_t), _ptr(L_up_t),
                                _stream(stream)), "svdq_pack_weight")


def svdq_replicate_weight_scales(w_scales, N, K, stream=None) -> None:
    _check(lib.svdq_replicate_weight_scales(_ptr(w_scales), int(N), int(K), _stream(stream)),
           "svdq_replicate_weight_scales")


def svdq_quantize_act_workspace_bytes(precision, M: int, K: int, rank: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib.svdq_quantize_act_workspace_bytes(_prec(precision), int(M), int(K), int(rank), ctypes.byref(out)),
           "svdq_quantize_act_workspace_bytes")
    return int(out.value)


def svdq_quantize_act(precision, group_size, x, M, K, inv_lambda, x_tensor_scale, compute_scale,
                      w_tensor_scale, L_down_t, rank, x_codes, x_scales, lowrank_act, workspace=None,
                      workspace_bytes=0, stream=None) -> None:
    if workspace is not None and not isinstance(workspace, int) and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib.svdq_quantize_act(_prec(precision), int(group_size), _ptr(x), int(M), int(K), _ptr(inv_lambda),
                                 _ptr(x_tensor_scale), int(bool(compute_scale)), _ptr(w_tensor_scale),
                                 _ptr(L_down_t), int(rank), _ptr(x_codes), _ptr(x_scales), _ptr(lowrank_act),
                                 _ptr(workspace), int(workspace_bytes), _stream(stream)), "svdq_quantize_act")


def svdq_quantize_act_noalloc(precision, group_size, x, M, K, inv_lambda, x_tensor_scale, compute_scale,
                              w_tensor_scale, L_down_t, rank, x_codes, x_scales, lowrank_act, stream=None) -> None:
    """svdq_quantize_act with the library's built-in workspace (for callers that cannot allocate)."""
    _check(lib.svdq_quantize_act_noalloc(_prec(precision), int(group_size), _ptr(x), int(M), int(K),
                                         _ptr(inv_lambda), _ptr(x_tensor_scale), int(bool(compute_scale)),
                                         _ptr(w_tensor_scale), _ptr(L_down_t), int(rank), _ptr(x_codes),
                                         _ptr(x_scales), _ptr(lowrank_act), _stream(stream)),
           "svdq_quantize_act_noalloc")


def svdq_gemm_w4a4(precision, group_size, x_codes, x_scales, x_tensor_scale, M, w_codes, w_scales,
                   w_tensor_scale, N, K, lowrank_act, L_up_t, rank, bias, y, stream=None) -> None:
    _check(lib.svdq_gemm_w4a4(_prec(precision), int(group_size), _ptr(x_codes), _ptr(x_scales),
                              _ptr(x_tensor_scale), int(M), _ptr(w_codes), _ptr(w_scales), _ptr(w_tensor_scale),
                              int(N), int(K), _ptr(lowrank_act), _ptr(L_up_t), int(rank), _ptr(bias), _ptr(y),
                              _stream(stream)), "svdq_gemm_w4a4")


def svdq_gemm_w4a4_qkv_norm_rope(precision, group_size, x_codes, x_scales, x_tensor_scale, M, w_codes, w_scales,
                                 w_tensor_scale, N, K, lowrank_act, L_up_t, rank, bias, heads, head_dim, norm_q,
                                 norm_k, eps, rope_cos, rope_sin, y, stream=None) -> None:
    _check(lib.svdq_gemm_w4a4_qkv_norm_rope(_prec(precision), int(group_size), _ptr(x_codes), _ptr(x_scales),
                                            _ptr(x_tensor_scale), int(M), _ptr(w_codes), _ptr(w_scales),
                                            _ptr(w_tensor_scale), int(N), int(K), _ptr(lowrank_act), _ptr(L_up_t),
                                            int(rank), _ptr(bias), int(heads), int(head_dim), _ptr(norm_q),
                                            _ptr(norm_k), float(eps), _ptr(rope_cos), _ptr(rope_sin), _ptr(y),
                                            _stream(stream)), "svdq_gemm_w4a4_qkv_norm_rope")


def svdq_qkv_norm_rope(y_in, y_out, M, heads, head_dim, norm_q, norm_k, eps, rope_cos, rope_sin,
                       stream=None) -> None:
    _check(lib.svdq_qkv_norm_rope(_ptr(y_in), _ptr(y_out), int(M), int(heads), int(head_dim), _ptr(norm_q),
                                  _ptr(norm_k), float(eps), _ptr(rope_cos), _ptr(rope_sin), _stream(stream)),
           "svdq_qkv_norm_rope")


def svdq_gelu_mlp_workspace_bytes(M, next_rank) -> int:
    out = ctypes.c_size_t(0)
    _check(lib.svdq_gelu_mlp_workspace_bytes(int(M), int(next_rank), ctypes.byref(out)),
           "svdq_gelu_mlp_workspace_bytes")
    return int(out.value)


def svdq_gemm_w4a4_gelu_quant(precision, group_size, x_codes, x_scales, x_tensor_scale, M, w_codes, w_scales,
                              w_tensor_scale, N, K, lowrank_act, L_up_t, rank, bias, gelu_approx, next_inv_lambda,
                              next_L_down_t, next_rank, next_x_tensor_scale, next_w_tensor_scale, next_x_codes,
                              next_x_scales, next_lowrank_act, workspace, workspace_bytes=0, stream=None) -> None:
    if workspace is not None and not isinstance(workspace, int) and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib.svdq_gemm_w4a4_gelu_quant(
        _prec(precision), int(group_size), _ptr(x_codes), _ptr(x_scales), _ptr(x_tensor_scale), int(M),
        _ptr(w_codes), _ptr(w_scales), _ptr(w_tensor_scale), int(N), int(K), _ptr(lowrank_act), _ptr(L_up_t),
        int(rank), _ptr(bias), int(gelu_approx), _ptr(next_inv_lambda), _ptr(next_L_down_t), int(next_rank),
        _ptr(next_x_tensor_scale), _ptr(next_w_tensor_scale), _ptr(next_x_codes), _ptr(next_x_scales),
        _ptr(next_lowrank_act), _ptr(workspace), int(workspace_bytes), _stream(stream)), "svdq_gemm_w4a4_gelu_quant")


def svdq_gemm_w4a4_gelu(precision, group_size, x_codes, x_scales, x_tensor_scale, M, w_codes, w_scales,
                        w_tensor_scale, N, K, lowrank_act, L_up_t, rank, bias, gelu_approx, y, stream=None) -> None:
    _check(lib.svdq_gemm_w4a4_gelu(
        _prec(precision), int(group_size), _ptr(x_codes), _ptr(x_scales), _ptr(x_tensor_scale), int(M),
        _ptr(w_codes), _ptr(w_scales), _ptr(w_tensor_scale), int(N), int(K), _ptr(lowrank_act), _ptr(L_up_t),
        int(rank), _ptr(bias), int(gelu_approx), _ptr(y), _stream(stream)), "svdq_gemm_w4a4_gelu")


def svdq_gelu(x, y, n, approx=0, stream=None) -> None:
    _check(lib.svdq_gelu(_ptr(x), _ptr(y), int(n), int(approx), _stream(stream)), "svdq_gelu")


def svdq_gemm_w4a16(x, M, w_codes, w_scales, N, K, bias, y, stream=None) -> None:
    _check(lib.svdq_gemm_w4a16(_ptr(x), int(M), _ptr(w_codes), _ptr(w_scales), int(N), int(K), _ptr(bias), _ptr(y),
                               _stream(stream)), "svdq_gemm_w4a16")


def svdq_svd_split_workspace_bytes(N: int, K: int, rank: int, oversample: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib.svdq_svd_split_workspace_bytes(int(N), int(K), int(rank), int(oversample), ctypes.byref(out)),
           "svdq_svd_split_workspace_bytes")
    return int(out.value)


def svdq_svd_split(W, lam, N, K, rank, omega, oversample, power_iters, R, L_down, L_up, singular_values,
                   workspace, workspace_bytes=0, stream=None) -> None:
    if workspace is not None and not isinstance(workspace, int) and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib.svdq_svd_split(_ptr(W), _ptr(lam), int(N), int(K), int(rank), _ptr(omega), int(oversample),
                              int(power_iters), _ptr(R), _ptr(L_down), _ptr(L_up), _ptr(singular_values),
                              _ptr(workspace), int(workspace_bytes), _stream(stream)), "svdq_svd_split")


def svdq_device_status(clear: bool = True) -> tuple[int, int]:
    """(status, site) after synchronising the device; does not raise."""
    site = ctypes.c_int(0)
    st = lib.svdq_device_status(int(bool(clear)), ctypes.byref(site))
    return int(st), int(site.value)


def svdq_debug_set_wait_limit_ns(ns: int) -> None:
    _check(lib.svdq_debug_set_wait_limit_ns(int(ns)), "svdq_debug_set_wait_limit_ns")


def svdq_debug_timeout_probe(stream=None) -> None:
    _check(lib.svdq_debug_timeout_probe(_stream(stream)), "svdq_debug_timeout_probe")


def svdq_debug_override_capability(major: int, minor: int = 0) -> None:
    lib.svdq_debug_override_capability(int(major), int(minor))


def svdq_debug_force_gemm_tiles(mode: int) -> None:
    """nvfp4 GEMM kernel: 0 = automatic, 1 = single-CTA 128x256 tiles, 2 = CTA-pair tiles."""
    _check(lib.svdq_debug_force_gemm_tiles(int(mode)), "svdq_debug_force_gemm_tiles")


def svdq_debug_force_quant_plan(mode: int) -> None:
    """K-split reduction of the quantizer: 0 = automatic, 1 = workspace (global
    memory), 2 = one thread-block cluster (distributed shared memory)."""
    _check(lib.svdq_debug_force_quant_plan(int(mode)), "svdq_debug_force_quant_plan")
