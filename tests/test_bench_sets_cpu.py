"""Host logic of bench.py's rotating input sets (no GPU): every workload the
bench times gets enough sets that, in each of its step, quantizer-only and
GEMM-only graphs, a set comes back only after at least 256 MiB of other sets'
data, i.e. twice the B200's 126 MB L2, so every timed step reads its inputs
from HBM; and the byte counts it sizes them with match the packed layouts."""
import pytest

import bench
from bit_w4a4_quantized_token_b200 import workloads as W

NAMES = ["qkv", "fc1", "fc2"] + [f"outproj_r{r}" for r in (0, 16, 32, 64, 128)] + ["int4_qkv"]


@pytest.mark.parametrize("name", NAMES)
def test_reuse_distance_covers_twice_the_l2(name):
    c = W.BY_NAME[name]
    n = bench.input_sets(c)
    assert n >= 3
    for per_step in (bench.quant_bytes(c), bench.gemm_bytes(c), bench.set_bytes_estimate(c)):
        assert (n - 1) * per_step >= 256 << 20


def test_set_bytes_of_the_qkv_workload():
    c = W.QKV   # M 4608, K 3072, N 9216, rank 32, nvfp4
    M, K, N, r = c.M, c.K, c.N, c.rank
    x, y = 2 * M * K, 2 * M * N
    act = M * K // 2 + M * K // 16 + 4 * M * r          # codes, group scales, hi/lo rank-r planes
    w = N * K // 2 + N * K // 16 + 36 * 12 * 16384      # codes, scale blocks, GEMM-ready scale copy
    assert bench.set_bytes_estimate(c) == x + y + act + w + 6 * N * r
    assert bench.input_sets(c) == 9


def test_config_names_the_protocol():
    cfg = bench.workload_config(W.QKV, False, 1)
    assert cfg["l2"].startswith("inputs larger than L2: 9 rotating input sets")
