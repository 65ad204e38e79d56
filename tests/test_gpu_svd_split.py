"""The offline SVDQuant split on the GPU against the CPU oracle's exact
truncated SVD (the decomposition the Diffusers docs page "Nunchaku Lite"
builds on; the tutorial's offline quantization step).

The GPU computes the rank-r part with a randomized range finder (subspace
iteration), so it approximates the exact truncation: its rank-r product must
match the oracle's within 1e-2 relative Frobenius norm (the bf16 rounding of
the factors alone is ~2^-9) on weights whose spectrum decays past r; the
leading singular values within 1e-3; and its residual must be the bf16
rounding of W_hat minus the product of its own bf16 factors.  The split then
feeds the W4A4 layer, whose output is checked against x W^T.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_quantized_token_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_w4a4_quantized_token_b200 import _lib

    yield
    st, site = _lib.svdq_device_status(clear=True)
    assert st == 0, f"device status {st} (site {site})"


def _bf16(t):
    return t.float().double().cpu().numpy()


def run_split(N, K, rank, power_iters=3, oversample=8):
    from bit_w4a4_quantized_token_b200 import _lib

    inp = W.svd_split_inputs(N, K, rank, oversample)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    R = torch.empty(N, K, dtype=torch.bfloat16, device="cuda")
    Ld = torch.empty(K, rank, dtype=torch.bfloat16, device="cuda")
    Lu = torch.empty(rank, N, dtype=torch.bfloat16, device="cuda")
    sv = torch.empty(rank + oversample, dtype=torch.float32, device="cuda")
    ws = torch.empty(_lib.svdq_svd_split_workspace_bytes(N, K, rank, oversample), dtype=torch.uint8, device="cuda")
    _lib.svdq_svd_split(d["W"], d["lam"], N, K, rank, d["omega"], oversample, power_iters, R, Ld, Lu, sv, ws)
    torch.cuda.synchronize()
    return inp, R, Ld, Lu, sv


@pytest.mark.parametrize("N,K,rank", [(512, 384, 16), (640, 320, 32), (9216, 3072, 32)],
                         ids=["small_r16", "ragged_r32", "qkv_r32"])
def test_svd_split_matches_truncated_svd(N, K, rank):
    from oracle import oracle as O

    inp, R, Ld, Lu, sv = run_split(N, K, rank)
    Rr, Ldr, Lur, s = O.svd_split(W.bits(inp["W"]), inp["lam"].numpy(), rank)
    P_ref = Lur.T @ Ldr.T
    P_gpu = _bf16(Lu).T @ _bf16(Ld).T
    rel = np.linalg.norm(P_gpu - P_ref) / np.linalg.norm(P_ref)
    assert rel <= 1e-2, rel
    np.testing.assert_allclose(sv.cpu().numpy()[:rank].astype(np.float64), s[:rank], rtol=1e-3)
    # the residual is W_hat minus the product of the GPU's own bf16 factors, rounded to bf16
    W_hat = _bf16(inp["W"]) * inp["lam"].double().numpy()[None, :]
    want = W_hat - P_gpu
    got = _bf16(R)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -126))) - 7)
    excess = np.abs(got - want) - ulp
    assert float(excess.max()) <= 1e-5 * float(np.abs(W_hat).max()), float(excess.max())
    # the residual is small: the rank-r part took the planted directions
    assert np.linalg.norm(got) <= 1.05 * np.linalg.norm(Rr)


def test_split_feeds_the_w4a4_layer():
    """W -> split -> pack -> quantize -> GEMM: y close to x W^T + b, and much
    closer than quantizing W_hat directly with no low-rank branch."""
    from bit_w4a4_quantized_token_b200 import layer

    N, K, M, rank = 768, 512, 256, 32
    inp, R, Ld, Lu, _ = run_split(N, K, rank)
    g = torch.Generator().manual_seed(9)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.01).to(torch.bfloat16)
    lam = inp["lam"].cuda()
    exact = x.double().numpy() @ inp["W"].double().numpy().T + b.double().numpy()
    packed = layer.pack_weight(R, lam, Ld, Lu, b.cuda())
    y = layer.svdq_linear(x.cuda(), packed).double().cpu().numpy()
    W_hat = (inp["W"].float() * inp["lam"][None, :]).to(torch.bfloat16).cuda()
    direct = layer.pack_weight(W_hat, lam, None, None, b.cuda())
    y0 = layer.svdq_linear(x.cuda(), direct).double().cpu().numpy()
    err = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    err0 = np.linalg.norm(y0 - exact) / np.linalg.norm(exact)
    assert err < 0.05, err
    assert err < 0.5 * err0, (err, err0)
