"""Tensor-core (tcgen05 block-scaled MXFP4) expert path vs the oracle.

The path quantises each projection input to MXFP4, so it is compared with the
oracle in mode "mxfp4_act" (same quantisation rule, fp64 arithmetic):
bf16 layer output within rel-L2 2e-3 of the oracle rounded to bf16.
"""
import numpy as np
import pytest
import torch

import oracle as O
from routed_expert_ffn_fp32_b200 import build, moe, synth

from helpers import TOL_Y, bits_np, dev_layer, gpu_layer, rel_l2, to_dev_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load_library()


def _cfg(H, I, E, k, T, shared, bias=True, std=0.05):
    return synth.LayerConfig("gemm", H, I, E, k, T, std, 1.0 if bias else None, shared)


GEMM_CASES = [
    # H, I, E, k, T, shared
    (256, 128, 8, 2, 64, False),      # smallest tiles, one K stage in down
    (1024, 512, 16, 4, 200, True),    # several M tiles, shared expert
    (512, 256, 4, 2, 300, False),     # buckets above 128 tokens: two token tiles
    (512, 1408, 8, 2, 96, True),      # I = 1408: a half-filled last K stage in down
    (256, 384, 3, 3, 7, False),       # k == E, tiny ragged buckets
]


@pytest.mark.parametrize("H,I,E,k,T,shared", GEMM_CASES)
def test_gemm_layer_vs_oracle(H, I, E, k, T, shared):
    cfg = _cfg(H, I, E, k, T, shared)
    L = synth.layer(cfg, 21)
    ref = O.layer_forward(L["x"], L["W_r"], L["bias"], L["experts"], L["shared"], k, "mxfp4_act")
    out = gpu_layer(L, dev_layer(L), cfg, moe.MOE_PATH_GEMM, moe.MOE_ACT_MXFP4)
    got = O.bf16_bits_to_f64(out["y"])
    assert rel_l2(got, O.bf16_bits_to_f64(ref["y_bf16"])) < TOL_Y
    assert rel_l2(got, ref["y"]) < TOL_Y


def test_gemm_partials_match_gemv_mxfp4():
    cfg = _cfg(1024, 512, 16, 4, 150, True)
    L = synth.layer(cfg, 3)
    ref = O.layer_forward(L["x"], L["W_r"], L["bias"], L["experts"], L["shared"], cfg.k, "mxfp4_act")
    D = dev_layer(L)
    shape = moe.shape_of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    rows = cfg.T * cfg.k + cfg.T
    outs = {}
    for path in (moe.MOE_PATH_GEMV, moe.MOE_PATH_GEMM):
        ws = moe.make_workspace(shape, path, moe.MOE_ACT_MXFP4, True)
        partial = torch.zeros((rows, cfg.H), dtype=torch.float32, device="cuda")
        moe.moe_expert_ffn_mxfp4(D["experts"], D["shared"], D["x"],
                                 torch.from_numpy(ref["offsets"]).cuda(),
                                 torch.from_numpy(ref["entries"]).cuda(), shape, partial, ws, path,
                                 moe.MOE_ACT_MXFP4)
        torch.cuda.synchronize()
        assert moe.moe_get_error(ws) == 0
        outs[path] = partial.cpu().numpy()
    for r in range(rows):
        assert rel_l2(outs[moe.MOE_PATH_GEMM][r], ref["partial"][r]) < 5e-3, r
        assert rel_l2(outs[moe.MOE_PATH_GEMV][r], ref["partial"][r]) < 5e-3, r
    assert rel_l2(outs[moe.MOE_PATH_GEMM], outs[moe.MOE_PATH_GEMV]) < 2e-3


def test_gemm_rejects_exact_precision():
    cfg = _cfg(256, 128, 8, 2, 64, False)
    L = synth.layer(cfg, 1)
    D = dev_layer(L)
    shape = moe.shape_of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = moe.make_workspace(shape, moe.MOE_PATH_GEMM, moe.MOE_ACT_MXFP4)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.int16, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_layer_forward(D["x"], D["W_r"], D["bias"], D["experts"], None, shape, y, ws,
                              moe.MOE_PATH_GEMM, moe.MOE_ACT_EXACT)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE


def test_gemm_graph_replay_deterministic():
    cfg = _cfg(512, 256, 8, 2, 128, True)
    L = synth.layer(cfg, 4)
    D = dev_layer(L)
    shape = moe.shape_of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = moe.make_workspace(shape, moe.MOE_PATH_GEMM, moe.MOE_ACT_MXFP4, True)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.int16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        moe.moe_layer_forward(D["x"], D["W_r"], D["bias"], D["experts"], D["shared"], shape, y, ws,
                              moe.MOE_PATH_GEMM, moe.MOE_ACT_MXFP4)
        torch.cuda.synchronize()
        first = bits_np(y).copy()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            moe.moe_layer_forward(D["x"], D["W_r"], D["bias"], D["experts"], D["shared"], shape,
                                  y, ws, moe.MOE_PATH_GEMM, moe.MOE_ACT_MXFP4)
    for _ in range(3):
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(bits_np(y), first)
    assert moe.moe_get_error(ws) == 0
