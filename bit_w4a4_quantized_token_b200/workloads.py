"""Seeded synthetic inputs for the SVDQ W4A4 linear layer.

This module only draws random numbers; it holds none of the layer's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

The shapes stand in for the pages' workload (ERNIE-Image-Turbo / FLUX-class
diffusion transformers at 1024x1024, Diffusers docs "Nunchaku Lite" and the
tutorial's "Benchmark" table): 4096 image + 512 text tokens = 4608 rows, hidden
size 3072, rank 32.  No trained weights or prompts are involved.

Recipe (fixed; every draw is fp32 on a torch CPU generator, then rounded to
bf16 nearest-even where the tensor is bf16):
  1. x       ~ N(0, 1)            [M, K]   (fc2: GELU_erf(N(0, 1)))
  2. outlier channels idx = randperm(K)[:n_out], x[:, idx] *= 20,
     n_out = round(0.01 K) (4 for the tiny case)
  3. lambda  ~ U[0.5, 4]          [K]      (fp32, stays fp32)
  4. R       ~ N(0, 1) / sqrt(K)  [N, K]
  5. L_down  ~ N(0, 1) / sqrt(K)  [K, r]
  6. L_up    ~ N(0, 1) * 0.1 / sqrt(r)  [r, N]
  7. b       ~ N(0, 1) * 0.01     [N]
"N(0, s)" is read as standard deviation s.  Case i uses seed i.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Case:
    name: str
    M: int
    K: int
    N: int
    rank: int
    precision: str          # "nvfp4" (group 16) or "int4" (group 64)
    seed: int
    n_outliers: int
    gelu_input: bool = False

    @property
    def group_size(self) -> int:
        return 16 if self.precision == "nvfp4" else 64

    @property
    def flops(self) -> int:
        """Algorithmic GEMM flops 2MNK (the low-rank branch is not counted)."""
        return 2 * self.M * self.N * self.K


def _outliers(K: int) -> int:
    return int(round(0.01 * K))


TINY = Case("tiny", 64, 256, 256, 32, "nvfp4", 0, 4)
QKV = Case("qkv", 4608, 3072, 9216, 32, "nvfp4", 1, _outliers(3072))
FC1 = Case("fc1", 4608, 3072, 12288, 32, "nvfp4", 2, _outliers(3072))
FC2 = Case("fc2", 4608, 12288, 3072, 32, "nvfp4", 2, _outliers(12288), gelu_input=True)
OUTPROJ = {r: Case(f"outproj_r{r}", 18432, 3072, 3072, r, "nvfp4", 3, _outliers(3072))
           for r in (0, 16, 32, 64, 128)}
INT4_QKV = Case("int4_qkv", 4608, 3072, 9216, 32, "int4", 4, _outliers(3072))

ALL_CASES = [TINY, QKV, FC1, FC2, *OUTPROJ.values(), INT4_QKV]
BY_NAME = {c.name: c for c in ALL_CASES}


def scaled(case: Case, M: int | None = None, K: int | None = None, N: int | None = None,
           rank: int | None = None, name: str | None = None) -> Case:
    """Same recipe and seed at other sizes (for oracle-sized parity cases)."""
    K = case.K if K is None else K
    return Case(name or f"{case.name}_small", case.M if M is None else M, K, case.N if N is None else N,
                case.rank if rank is None else rank, case.precision, case.seed,
                max(1, _outliers(K)) if K != case.K else case.n_outliers, case.gelu_input)


def make_inputs(case: Case) -> dict:
    """Draw the layer's inputs on the CPU in the fixed order."""
    g = torch.Generator(device="cpu")
    g.manual_seed(case.seed)
    M, K, N, r = case.M, case.K, case.N, case.rank
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    if case.gelu_input:
        x = torch.nn.functional.gelu(x, approximate="none")
    idx = torch.randperm(K, generator=g)[: case.n_outliers]
    x[:, idx] *= 20.0
    lam = torch.rand(K, generator=g, dtype=torch.float32) * 3.5 + 0.5
    R = torch.randn(N, K, generator=g, dtype=torch.float32) / math.sqrt(K)
    L_down = torch.randn(K, r, generator=g, dtype=torch.float32) / math.sqrt(K)
    L_up = torch.randn(r, N, generator=g, dtype=torch.float32) * (0.1 / math.sqrt(max(r, 1)))
    b = torch.randn(N, generator=g, dtype=torch.float32) * 0.01
    return {
        "x": x.to(torch.bfloat16),
        "outliers": idx,
        "lam": lam,
        "R": R.to(torch.bfloat16),
        "L_down": L_down.to(torch.bfloat16),
        "L_up": L_up.to(torch.bfloat16),
        "b": b.to(torch.bfloat16),
    }


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (for the oracle)."""
    import numpy as np

    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


QKV_HEAD_DIM = 128          # FLUX-class DiT attention heads: 24 x 128 = 3072 = hidden size
QKV_EPS = 1e-6


def qkv_inputs(M: int, heads: int, seed: int = 7) -> dict:
    """Extra inputs of the fused QKV + RMSNorm + RoPE path, drawn after the
    layer's own: the Q and K RMSNorm weights ~ U[0.5, 2] (bf16) and one rotary
    angle per (token, pair) ~ U[-pi, pi), given as fp32 cos and sin tables
    [M, 64] (the per-token rotary embedding the attention block receives)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    D = QKV_HEAD_DIM
    wq = (torch.rand(D, generator=g, dtype=torch.float32) * 1.5 + 0.5).to(torch.bfloat16)
    wk = (torch.rand(D, generator=g, dtype=torch.float32) * 1.5 + 0.5).to(torch.bfloat16)
    theta = (torch.rand(M, D // 2, generator=g, dtype=torch.float64) * 2.0 - 1.0) * math.pi
    return {"heads": heads, "head_dim": D, "eps": QKV_EPS, "norm_q": wq, "norm_k": wk,
            "cos": torch.cos(theta).to(torch.float32), "sin": torch.sin(theta).to(torch.float32)}


def svd_split_inputs(N: int, K: int, rank: int, oversample: int = 8, seed: int = 5) -> dict:
    """Inputs of the offline SVD split: a weight W [N, K] (bf16) with a planted
    rank-`rank` component -- orthonormal factors U [N, r] and V [K, r] from the
    QR decomposition of Gaussian draws, singular values 30 * 0.93^i -- plus
    Gaussian noise of standard deviation 0.1 / sqrt(K) (a few dominant
    directions over a noise floor, like trained projection weights); the
    smoothing divisors lambda ~ U[0.5, 4]; the Gaussian test matrix Omega
    [K, rank + oversample] ~ N(0, 1) (fp32) that the randomized range finder
    consumes."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    U, _ = torch.linalg.qr(torch.randn(N, rank, generator=g, dtype=torch.float64))
    V, _ = torch.linalg.qr(torch.randn(K, rank, generator=g, dtype=torch.float64))
    s = 30.0 * 0.93 ** torch.arange(rank, dtype=torch.float64)
    noise = torch.randn(N, K, generator=g, dtype=torch.float64) * (0.1 / math.sqrt(K))
    W = (U * s) @ V.T + noise
    lam = torch.rand(K, generator=g, dtype=torch.float32) * 3.5 + 0.5
    omega = torch.randn(K, rank + oversample, generator=g, dtype=torch.float32)
    return {"W": W.to(torch.bfloat16), "lam": lam, "omega": omega, "rank": rank, "oversample": oversample}
