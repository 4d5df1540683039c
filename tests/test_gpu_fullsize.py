"""Full-size layers in the bench's launch configuration, checked on sampled
tokens (the layer is per-token, so the oracle recomputes only those rows).

Workloads: the fine-grained layer (H 4096, I 2048, 256 experts, top-8, shared
expert) with the prefill Zipf s = 1.2 routing at T = 2048 (tensor-core path,
MXFP4 activations, and the CUDA-core path in exact mode) and at the sweep's
batch sizes.  Tolerance as everywhere: bf16 outputs within rel-L2 2e-3 of the
oracle rounded to bf16; routing bit-exact outside near-ties.
"""
import numpy as np
import pytest
import torch

import oracle as O
from routed_expert_ffn_fp32_b200 import build, moe, synth

from helpers import TOL_Y, check_routing, dev_layer, gpu_layer, rel_l2

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def big():
    build.build()
    moe.load_library()
    cfg = synth.PREFILL
    L = synth.layer(cfg, 0)
    return cfg, L, dev_layer(L)


def _sample(T, n, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(T, size=min(n, T), replace=False))


def _check(cfg, L, out, tokens, mode):
    T = L["x"].shape[0]
    ref = O.layer_forward(L["x"], L["W_r"], L["bias"], L["experts"], L["shared"], cfg.k, mode,
                          tokens=tokens)
    sub = {"x": L["x"][tokens], "W_r": L["W_r"], "bias": L["bias"]}
    check_routing(sub, ref, out["idx"][tokens], out["w"][tokens], cfg.k, cfg.H, T_route=T)
    got = O.bf16_bits_to_f64(out["y"][tokens])
    assert rel_l2(got, O.bf16_bits_to_f64(ref["y_bf16"])) < TOL_Y
    assert np.isfinite(got).all()


def test_prefill_2048_tensor_core_path(big):
    cfg, L, D = big
    out = gpu_layer(L, D, cfg, moe.MOE_PATH_GEMM, moe.MOE_ACT_MXFP4)
    _check(cfg, L, out, _sample(cfg.T, 10, 1), "mxfp4_act")


def test_prefill_2048_cuda_core_path_exact(big):
    cfg, L, D = big
    out = gpu_layer(L, D, cfg, moe.MOE_PATH_GEMV, moe.MOE_ACT_EXACT)
    _check(cfg, L, out, _sample(cfg.T, 6, 2), "exact")


@pytest.mark.parametrize("T", synth.SWEEP_T)
def test_sweep_batch_sizes(big, T):
    cfg, L, D = big
    Lt = dict(L)
    Lt["x"] = synth.activations(cfg, 7, T)
    Dt = dict(D)
    Dt["x"] = torch.from_numpy(Lt["x"].view(np.int16)).cuda()
    out = gpu_layer(Lt, Dt, cfg.with_T(T), moe.MOE_PATH_GEMV, moe.MOE_ACT_EXACT)
    _check(cfg.with_T(T), Lt, out, _sample(T, 3, T), "exact")
    out = gpu_layer(Lt, Dt, cfg.with_T(T), moe.MOE_PATH_GEMM, moe.MOE_ACT_MXFP4)
    _check(cfg.with_T(T), Lt, out, _sample(T, 3, T + 1), "mxfp4_act")
