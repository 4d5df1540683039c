"""The allocation-free entry point (moe_layer_forward_static).

Callers that may not allocate device memory use this variant: a host
application that owns every device allocation through its own pool, a
real-time loop in which cudaMalloc/cudaFree would synchronise the device and
stall other streams, or plug-in code that only ever sees the tensors it is
handed.  It takes no workspace and runs on a fixed scratch array inside the
library.  Its output must match the regular entry point's within the
tolerance the other layer tests use, on two calls in a row (the second call
finds the array as the first one left it), and calls of different shapes in
a row must each match the oracle.  This file is collected last on purpose.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle as O
from routed_expert_ffn_fp32_b200 import build, moe, synth

from helpers import TOL_Y, bits_np, check_routing, check_y, dev_layer, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load_library()


def _static_call(lib, x, D, shape, y, idx, w=None):
    """moe_layer_forward_static through the C ABI directly."""
    return lib.moe_layer_forward_static(
        ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(D["W_r"].data_ptr()),
        None if D["bias"] is None else ctypes.c_void_p(D["bias"].data_ptr()),
        ctypes.byref(D["experts"].cstruct()),
        None if D["shared"] is None else ctypes.byref(D["shared"].cstruct()),
        shape, moe.MOE_ACT_EXACT, ctypes.c_void_p(y.data_ptr()),
        ctypes.c_void_p(idx.data_ptr()), None if w is None else ctypes.c_void_p(w.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,T", [("decode_h4096_i1408_e64_k2", 5),
                                    ("finegrained_h4096_i2048_e256_k8_shared", 5)])
def test_static_scratch_matches_workspace_entry(name, T):
    cfg = synth.CONFIGS[name]
    lib = moe.load_library()
    shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = moe.make_workspace(shape, moe.MOE_PATH_GEMV, moe.MOE_ACT_EXACT, cfg.shared)
    L = synth.layer(cfg, 11, T)
    D = dev_layer(L)
    for call in range(2):
        x = torch.from_numpy(synth.activations(cfg, 100 + call, T).view(np.int16)).cuda()
        y_ref = torch.empty((T, cfg.H), dtype=torch.int16, device="cuda")
        idx_ref = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
        y = torch.full((T, cfg.H), -1, dtype=torch.int16, device="cuda")
        idx = torch.full((T, cfg.k), -1, dtype=torch.int32, device="cuda")
        moe.moe_layer_forward(x, D["W_r"], D["bias"], D["experts"], D["shared"], shape, y_ref, ws,
                              moe.MOE_PATH_GEMV, moe.MOE_ACT_EXACT, idx_ref)
        st = _static_call(lib, x, D, shape, y, idx)
        assert st == moe.MOE_OK, moe.status_string(st)
        assert lib.moe_get_error_static(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
        torch.cuda.synchronize()
        got = O.bf16_bits_to_f64(bits_np(y))
        want = O.bf16_bits_to_f64(bits_np(y_ref))
        assert rel_l2(got, want) < TOL_Y
        assert np.isfinite(got).all()
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy())


def test_static_scratch_across_shapes_matches_oracle():
    """Shapes in the order that puts a small shape's scratch on a large
    shape's leftovers: fine-grained T=5, decode64 T=1, decode64 T=5,
    fine-grained T=1.  Each call matches the oracle (routing bit-exact,
    per-token output within 2e-3), latches no error and finishes well inside
    any wait limit."""
    lib = moe.load_library()
    fg, d64 = synth.FINEGRAINED, synth.DECODE64
    layers = {}
    for cfg, T in [(fg, 5), (d64, 1), (d64, 5), (fg, 1)]:
        if cfg.name not in layers:
            L = synth.layer(cfg, 12, 5)
            layers[cfg.name] = (L, dev_layer(L))
        L, D = layers[cfg.name]
        shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
        x = D["x"][:T].contiguous()
        y = torch.full((T, cfg.H), -1, dtype=torch.int16, device="cuda")
        idx = torch.full((T, cfg.k), -1, dtype=torch.int32, device="cuda")
        w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        st = _static_call(lib, x, D, shape, y, idx, w)
        assert st == moe.MOE_OK, moe.status_string(st)
        assert moe.moe_get_error_static() == moe.MOE_OK, (cfg.name, T)
        assert time.perf_counter() - t0 < 0.5, (cfg.name, T)
        ref = O.layer_forward(L["x"][:T], L["W_r"], L["bias"], L["experts"], L["shared"], cfg.k)
        check_routing({"x": L["x"][:T], "W_r": L["W_r"], "bias": L["bias"]}, ref,
                      idx.cpu().numpy(), w.cpu().numpy(), cfg.k, cfg.H)
        check_y(bits_np(y), ref)


def test_static_scratch_rejects_oversized_shape():
    lib = moe.load_library()
    big = moe.shape_of(4096, 4096, 2048, 256, 8)
    A = ctypes.c_void_p(0x100000)  # never dereferenced: the size check comes first
    ex = moe.moe_mxfp4_experts_t(0x100000, 0x100000, 0x100000, 0x100000, 0x100000, 0x100000, 256)
    st = lib.moe_layer_forward_static(A, A, None, ctypes.byref(ex), None, big, 0, A, None, None,
                                      None)
    assert st == moe.MOE_ERR_WORKSPACE
