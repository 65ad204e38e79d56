"""PyTorch-facing helpers around the C ABI: they allocate the packed buffers as
torch tensors and call the entry points in order.  Device memory and streams
come from PyTorch; every step of the layer runs in the CUDA library.

    packed = pack_weight(R, lam, L_down, L_up, precision="nvfp4")   # once per layer
    y = svdq_linear(x, packed)                                      # quantize_act + gemm_w4a4
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _lib

_U8 = torch.uint8


def _empty(nbytes: int, device) -> torch.Tensor:
    # 256-byte aligned by the caching allocator; at least one byte so data_ptr is valid
    return torch.empty(max(int(nbytes), 1), dtype=_U8, device=device)


@dataclass
class PackedWeight:
    precision: str
    N: int
    K: int
    rank: int
    w_codes: torch.Tensor
    w_scales: torch.Tensor
    w_tensor_scale: torch.Tensor | None
    inv_lambda: torch.Tensor
    L_down_t: torch.Tensor | None
    L_up_t: torch.Tensor | None
    bias: torch.Tensor | None

    @property
    def group_size(self) -> int:
        return _lib.GROUP_SIZES[self.precision]


@dataclass
class QuantizedAct:
    M: int
    x_codes: torch.Tensor
    x_scales: torch.Tensor
    x_tensor_scale: torch.Tensor | None
    lowrank_act: torch.Tensor | None
    workspace: torch.Tensor | None = None   # zero-filled once; the library keeps it zeroed


def pack_weight(R: torch.Tensor, lam: torch.Tensor, L_down: torch.Tensor | None, L_up: torch.Tensor | None,
                bias: torch.Tensor | None = None, precision: str = "nvfp4", stream=None) -> PackedWeight:
    N, K = R.shape
    rank = 0 if L_down is None else int(L_down.shape[1])
    dev = R.device
    sz = _lib.svdq_buffer_sizes(precision, N, K, rank)
    w_codes = _empty(sz["codes_bytes"], dev)
    w_scales = _empty(sz["w_scales_bytes"], dev)   # nvfp4: block layout, then the GEMM-ready copy
    w_ts = torch.empty(4, dtype=torch.float32, device=dev) if precision == "nvfp4" else None
    inv_lambda = torch.empty(K, dtype=torch.float32, device=dev)
    L_down_t = torch.empty(2, rank, K, dtype=torch.bfloat16, device=dev) if rank else None
    L_up_t = torch.empty(N, rank, dtype=torch.bfloat16, device=dev) if rank else None
    _lib.svdq_pack_weight(precision, _lib.GROUP_SIZES[precision], R.contiguous(), N, K, lam.contiguous(),
                          None if rank == 0 else L_down.contiguous(), None if rank == 0 else L_up.contiguous(),
                          rank, w_codes, w_scales, w_ts, inv_lambda, L_down_t, L_up_t, stream)
    return PackedWeight(precision, N, K, rank, w_codes, w_scales, w_ts, inv_lambda, L_down_t, L_up_t,
                        None if bias is None else bias.contiguous())


def alloc_act(packed: PackedWeight, M: int, device) -> QuantizedAct:
    sz = _lib.svdq_buffer_sizes(packed.precision, M, packed.K, packed.rank)
    ws = _lib.svdq_quantize_act_workspace_bytes(packed.precision, M, packed.K, packed.rank)
    return QuantizedAct(
        M,
        _empty(sz["codes_bytes"], device),
        _empty(sz["scales_bytes"], device),
        torch.empty(4, dtype=torch.float32, device=device) if packed.precision == "nvfp4" else None,
        torch.empty(2, M, packed.rank, dtype=torch.bfloat16, device=device) if packed.rank else None,
        torch.zeros(ws, dtype=torch.uint8, device=device) if ws else None,
    )


def quantize_act(x: torch.Tensor, packed: PackedWeight, out: QuantizedAct | None = None,
                 x_tensor_scale: float | torch.Tensor | None = None, stream=None) -> QuantizedAct:
    """x [M, K] bf16 -> codes, scales, rank-r activations.  x_tensor_scale None
    derives S_x from amax on the device; a float or a device tensor is used as
    a static scale."""
    M, K = x.shape
    assert K == packed.K
    q = out if out is not None else alloc_act(packed, M, x.device)
    compute = 1
    if packed.precision == "nvfp4" and x_tensor_scale is not None:
        compute = 0
        if isinstance(x_tensor_scale, torch.Tensor):
            q.x_tensor_scale[:1].copy_(x_tensor_scale.reshape(-1)[:1])
        else:
            q.x_tensor_scale.fill_(float(x_tensor_scale))
    _lib.svdq_quantize_act(packed.precision, packed.group_size, x, M, K, packed.inv_lambda, q.x_tensor_scale,
                           compute, packed.w_tensor_scale, packed.L_down_t, packed.rank, q.x_codes, q.x_scales,
                           q.lowrank_act, q.workspace, stream=stream)
    return q


def gemm(q: QuantizedAct, packed: PackedWeight, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if y is None:
        y = torch.empty(q.M, packed.N, dtype=torch.bfloat16, device=q.x_codes.device)
    _lib.svdq_gemm_w4a4(packed.precision, packed.group_size, q.x_codes, q.x_scales, q.x_tensor_scale, q.M,
                        packed.w_codes, packed.w_scales, packed.w_tensor_scale, packed.N, packed.K, q.lowrank_act,
                        packed.L_up_t, packed.rank, packed.bias, y, stream)
    return y


def svdq_linear(x: torch.Tensor, packed: PackedWeight, x_tensor_scale=None, stream=None) -> torch.Tensor:
    """One forward of the SVDQ W4A4 linear layer: two launches, no host sync."""
    return gemm(quantize_act(x, packed, x_tensor_scale=x_tensor_scale, stream=stream), packed, stream=stream)
