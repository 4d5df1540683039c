"""The C-ABI library on the host: it loads, exports every declared symbol,
sizes workspaces and rejects bad arguments before any launch (no GPU needed:
every call here returns before touching the device)."""
import ctypes
import os
import re

import pytest

from routed_expert_ffn_fp32_b200 import build, moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.load_library()


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert set(declared) == set(moe.EXPORTS)
    for name in declared:
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr), name


def test_version_and_status_strings(lib):
    assert moe.moe_version() == "0.1.0"
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert moe.status_string(s)
    assert moe.status_string(17) == "unknown status"


def test_workspace_bytes():
    s = moe.shape_of(5, 4096, 1408, 64, 2)
    n_gemv = moe.moe_workspace_bytes(s, moe.MOE_PATH_GEMV)
    rows = 5 * 2
    assert n_gemv >= rows * (4096 + 1408) * 4
    assert moe.moe_workspace_bytes(s, moe.MOE_PATH_GEMV, has_shared=True) > n_gemv
    assert moe.moe_workspace_bytes(s, moe.MOE_PATH_AUTO) >= n_gemv
    for bad in [(0, 4096, 1408, 64, 2), (1, 4016, 1408, 64, 2), (1, 4096, 1400, 64, 2),
                (1, 4096, 1408, 2000, 2), (1, 4096, 1408, 64, 17)]:
        assert moe.moe_workspace_bytes(moe.shape_of(*bad)) == 0, bad
    assert moe.moe_workspace_bytes(s, path=7) == 0
    assert moe.moe_workspace_bytes(s, precision=3) == 0


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_rejects_bad_arguments_before_launch(lib):
    s = moe.shape_of(4, 256, 128, 8, 2)
    A = 0x100000  # aligned, never dereferenced: every call below returns first
    ex = moe.moe_mxfp4_experts_t(A, A, A, A, A, A, 8)
    # null / misaligned pointers
    assert lib.moe_layer_forward(None, _fake(A), None, ctypes.byref(ex), None, s, 0, 0, _fake(A),
                                 None, None, _fake(A), 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_forward(_fake(A + 2), _fake(A), None, ctypes.byref(ex), None, s, 0, 0,
                                 _fake(A), None, None, _fake(A), 1 << 30,
                                 None) == moe.MOE_ERR_INVALID_ARG
    # expert count mismatch
    ex_bad = moe.moe_mxfp4_experts_t(A, A, A, A, A, A, 7)
    assert lib.moe_layer_forward(_fake(A), _fake(A), None, ctypes.byref(ex_bad), None, s, 0, 0,
                                 _fake(A), None, None, _fake(A), 1 << 30,
                                 None) == moe.MOE_ERR_INVALID_ARG
    # shapes
    for bad in [(0, 256, 128, 8, 2), (4, 250, 128, 8, 2), (4, 256, 128, 8, 0), (4, 256, 128, 4, 8)]:
        assert lib.moe_layer_forward(_fake(A), _fake(A), None, ctypes.byref(ex), None,
                                     moe.shape_of(*bad), 0, 0, _fake(A), None, None, _fake(A),
                                     1 << 30, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    # bad enums
    assert lib.moe_layer_forward(_fake(A), _fake(A), None, ctypes.byref(ex), None, s, 9, 0,
                                 _fake(A), None, None, _fake(A), 1 << 30,
                                 None) == moe.MOE_ERR_INVALID_ARG
    # workspace too small
    assert lib.moe_layer_forward(_fake(A), _fake(A), None, ctypes.byref(ex), None, s, 1, 0,
                                 _fake(A), None, None, _fake(A), 64, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_route_topk(_fake(A), _fake(A), None, s, None, _fake(A), _fake(A), _fake(A), 64,
                              None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_bucket(_fake(A), s, _fake(A), _fake(A), None, _fake(A), 1 << 20,
                          None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(_fake(A), None, s, 0, _fake(A), None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_act_quant_mxfp4(_fake(A), 4, 48, _fake(A), _fake(A),
                                   None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_decode_mxfp4(_fake(A), None, 4, 64, _fake(A), None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_get_error(None, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_workspace_init(_fake(A + 8), 1024, None) == moe.MOE_ERR_INVALID_ARG
    # routing needs k <= E; the expert FFN only needs k <= 16 (pair layout)
    k_gt_e = moe.shape_of(4, 256, 128, 4, 8)
    assert lib.moe_route_topk(_fake(A), _fake(A), None, k_gt_e, None, _fake(A), _fake(A), _fake(A),
                              1 << 30, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert moe.moe_workspace_bytes(k_gt_e, moe.MOE_PATH_GEMV) > 0
    assert moe.moe_workspace_bytes(moe.shape_of(4, 256, 128, 4, 17), moe.MOE_PATH_GEMV) == 0
    # expert-parallel pieces
    assert lib.moe_combine_range(_fake(A), _fake(A), _fake(A), 2, 9, s, 0, _fake(A),
                                 None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_combine_range(_fake(A), _fake(A), None, 0, 8, s, 0, _fake(A),
                                 None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_round_bf16(_fake(A), 6, _fake(A), None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_round_bf16(_fake(A), 0, _fake(A), None) == moe.MOE_OK
