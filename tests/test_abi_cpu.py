"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point the header declares, validates arguments before touching
the device, and reports a missing or wrong device as SVDQ_ERR_UNSUPPORTED_DEVICE."""
import json
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from bit_w4a4_quantized_token_b200 import build

    build.build()
    from bit_w4a4_quantized_token_b200 import _lib

    return _lib


def declared_functions():
    src = open(os.path.join(ROOT, "include", "svdq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L.lib, n), n
    assert sorted(L.EXPORTS) == names


def test_abi_version_and_strings(L):
    assert L.svdq_abi_version() == 2
    for st in range(6):
        assert L.status_string(st)
    assert "unsupported device" in L.status_string(L.SVDQ_ERR_UNSUPPORTED_DEVICE)


def test_buffer_sizes(L):
    s = L.svdq_buffer_sizes("nvfp4", 4608, 3072, 32)
    # a packed weight's scales: the block layout, then 16 KB per 256 x 256 tile of the GEMM-ready copy
    assert s == {"codes_bytes": 4608 * 1536, "scales_bytes": 4608 * 192, "lowrank_bytes": 4608 * 128,
                 "w_scales_bytes": 4608 * 192 + 18 * 12 * 16384}
    s = L.svdq_buffer_sizes("nvfp4", 200, 320, 16)          # rows padded to 256 for the scales
    assert s["scales_bytes"] == 256 * 20 and s["w_scales_bytes"] == 256 * 20 + 1 * 2 * 16384
    s = L.svdq_buffer_sizes("int4", 200, 320, 0)
    assert s["scales_bytes"] == 2 * 256 * 5 and s["lowrank_bytes"] == 0
    assert s["w_scales_bytes"] == s["scales_bytes"]
    for bad in [("nvfp4", 0, 64, 0), ("nvfp4", 8, 96, 0), ("nvfp4", 8, 0, 0)]:
        with pytest.raises(L.SvdqError) as e:
            L.svdq_buffer_sizes(*bad)
        assert e.value.status == L.SVDQ_ERR_UNSUPPORTED_SHAPE
    for bad_rank in (-16, 8, 272):
        with pytest.raises(L.SvdqError) as e:
            L.svdq_buffer_sizes("nvfp4", 8, 64, bad_rank)
        assert e.value.status == L.SVDQ_ERR_INVALID_ARG


def test_schemes_match_the_pages(L):
    """Only the (precision, group size) pairs of the scheme table are accepted."""
    golden = json.load(open(os.path.join(ROOT, "tests", "golden", "schemes.json")))
    accepted = {(s["precision"], s["group_size"]) for s in golden["schemes"] if s["method"] == "svdq_w4a4"}
    assert accepted == {("nvfp4", 16), ("int4", 64)}
    assert golden["config_example"]["svdq_w4a4"]["rank"] == 32
    fake = 1 << 20          # aligned non-null fake pointers: validation must stop before any use
    for prec in ("nvfp4", "int4"):
        for g in (8, 16, 32, 64, 128):
            try:
                L.svdq_gemm_w4a4(prec, g, fake, fake, fake, 64, fake, fake, fake, 256, 256, fake, fake, 32,
                                 None, fake, stream=0)
                status = 0
            except L.SvdqError as e:
                status = e.status
            if (prec, g) in accepted:
                # arguments are valid: the next check is the device (none here, or not sm_100)
                assert status in (0, L.SVDQ_ERR_UNSUPPORTED_DEVICE)
            else:
                assert status == L.SVDQ_ERR_INVALID_ARG, (prec, g)


def _gemm_status(L, **kw):
    fake = 1 << 20
    args = dict(precision="nvfp4", group_size=16, x_codes=fake, x_scales=fake, x_tensor_scale=fake, M=64,
                w_codes=fake, w_scales=fake, w_tensor_scale=fake, N=256, K=256, lowrank_act=fake, L_up_t=fake,
                rank=32, bias=None, y=fake, stream=0)
    args.update(kw)
    try:
        L.svdq_gemm_w4a4(**args)
        return 0
    except L.SvdqError as e:
        return e.status


def test_argument_validation_before_device(L):
    assert _gemm_status(L, x_codes=None) == L.SVDQ_ERR_INVALID_ARG
    assert _gemm_status(L, y=(1 << 20) + 8) == L.SVDQ_ERR_INVALID_ARG          # misaligned
    assert _gemm_status(L, K=96) == L.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert _gemm_status(L, N=264) == L.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert _gemm_status(L, M=0) == L.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert _gemm_status(L, rank=24) == L.SVDQ_ERR_INVALID_ARG
    assert _gemm_status(L, rank=32, lowrank_act=None) == L.SVDQ_ERR_INVALID_ARG
    assert _gemm_status(L, rank=0, lowrank_act=None, L_up_t=None) in (0, L.SVDQ_ERR_UNSUPPORTED_DEVICE)
    assert _gemm_status(L, bias=(1 << 20) + 2) == L.SVDQ_ERR_INVALID_ARG
    assert _gemm_status(L, precision="int4", group_size=64, x_tensor_scale=None,
                        w_tensor_scale=None) in (0, L.SVDQ_ERR_UNSUPPORTED_DEVICE)


def test_replicate_weight_scales_argument_checks(L):
    """The GEMM-ready weight-scale copy: argument errors come before any device check."""
    fake = 1 << 20

    def status(**kw):
        args = dict(w_scales=fake, N=256, K=256, stream=0)
        args.update(kw)
        try:
            L.svdq_replicate_weight_scales(**args)
            return 0
        except L.SvdqError as e:
            return e.status

    assert status(w_scales=None) == L.SVDQ_ERR_INVALID_ARG
    assert status(w_scales=fake + 8) == L.SVDQ_ERR_INVALID_ARG      # misaligned
    assert status(N=8) == L.SVDQ_ERR_UNSUPPORTED_SHAPE              # N % 16 != 0
    assert status(K=96) == L.SVDQ_ERR_UNSUPPORTED_SHAPE             # K % 64 != 0
    assert status(N=0) == L.SVDQ_ERR_UNSUPPORTED_SHAPE
    assert status() in (0, L.SVDQ_ERR_UNSUPPORTED_DEVICE)


def test_capability_check_rejects_other_devices(L):
    """With any capability other than 10.0 (or no GPU) nothing is launched."""
    L.svdq_debug_override_capability(12, 0)        # an sm_120 consumer Blackwell part
    try:
        assert _gemm_status(L) == L.SVDQ_ERR_UNSUPPORTED_DEVICE
        L.svdq_debug_override_capability(9, 0)     # Hopper
        assert _gemm_status(L) == L.SVDQ_ERR_UNSUPPORTED_DEVICE
    finally:
        L.svdq_debug_override_capability(-1)


def test_force_gemm_tiles_hook(L):
    """Modes 0-2 are accepted (no device needed); anything else is rejected with a message."""
    for mode in (1, 2, 0):
        L.svdq_debug_force_gemm_tiles(mode)
    for bad in (-1, 3):
        with pytest.raises(L.SvdqError) as e:
            L.svdq_debug_force_gemm_tiles(bad)
        assert e.value.status == L.SVDQ_ERR_INVALID_ARG
        assert "not 0, 1 or 2" in L.lib.svdq_last_error().decode()


def test_force_quant_plan_hook(L):
    """Modes 0-3 are accepted (no device needed); anything else is rejected with a message."""
    for mode in (1, 2, 3, 0):
        L.svdq_debug_force_quant_plan(mode)
    for bad in (-1, 4):
        with pytest.raises(L.SvdqError) as e:
            L.svdq_debug_force_quant_plan(bad)
        assert e.value.status == L.SVDQ_ERR_INVALID_ARG
        assert "not 0, 1, 2 or 3" in L.lib.svdq_last_error().decode()


def test_quantize_act_workspace_bytes(L):
    # QKV shape: 36 row blocks x 4 K-splits x 128 rows x rank 32 fp32, plus two counters per row block
    # (36 x 8 bytes, rounded up to 512)
    assert L.svdq_quantize_act_workspace_bytes("nvfp4", 4608, 3072, 32) == 512 + 36 * 4 * 128 * 32 * 4
    # 144 row blocks fill the GPU without a K split: no workspace
    assert L.svdq_quantize_act_workspace_bytes("nvfp4", 18432, 3072, 32) == 0
    assert L.svdq_quantize_act_workspace_bytes("int4", 4608, 3072, 0) == 0
    # the split never exceeds the number of 64-column chunks
    assert L.svdq_quantize_act_workspace_bytes("nvfp4", 64, 256, 32) == 256 + 1 * 4 * 128 * 32 * 4
