"""Full-size layers in the bench's launch configuration, checked against the
oracle: the routing of every token of the batch, and the layer output on
sampled tokens (the layer is per-token, so the oracle recomputes only those
rows).

Workloads: the fine-grained layer (H 4096, I 2048, 256 experts, top-8, shared
expert) with the prefill Zipf s = 1.2 routing at T = 2048 and 4096 (tensor-core
path, MXFP4 activations; at 2048 also the CUDA-core path in exact mode) and at
the sweep's batch sizes.  Tolerance as everywhere: the largest per-token
relative L2 error of the bf16 outputs within 2e-3 of the oracle rounded to
bf16; routing bit-exact with no near-ties.
"""
import numpy as np
import pytest
import torch

import oracle as O
from routed_expert_ffn_fp32_b200 import build, moe, synth

from helpers import check_routing, check_y, dev_layer, gpu_layer, route_depth

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
    # near-ties among the sampled tokens are checked for validity; their count
    # over whole prefill batches is bounded in _check_all_routing
    check_routing(sub, ref, out["idx"][tokens], out["w"][tokens], cfg.k, cfg.H, T_route=T,
                  max_ties=len(tokens))
    check_y(out["y"][tokens], ref)


def _check_all_routing(cfg, L, D, out):
    """Routing of every token of the batch (the router is cheap in fp64 even
    at prefill sizes):
    * the GPU's float32 logits (the layer's router kernels, through
      moe_route_topk) lie within the float32 summation bound of the exact ones;
    * every token's indices are exactly the top-k of those float32 logits
      (ties to the lower index) and its weights their renormalised softmax;
    * tokens whose exact top-k + 1 logits are farther apart than the bound
      (all but a few percent: each token has k adjacent gaps, each must clear
      a bound of about 1e-3) get the exact top-k, bit for bit."""
    T = L["x"].shape[0]
    x = O.bf16_bits_to_f64(L["x"])
    logits = O.router_logits(x, L["W_r"], L["bias"])
    idx, w = O.route_topk(logits, cfg.k)
    shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = moe.make_workspace(shape, moe.MOE_PATH_GEMV)
    gidx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    glog = torch.empty((T, cfg.E), dtype=torch.float32, device="cuda")
    moe.moe_route_topk(D["x"], D["W_r"], D["bias"], shape, gidx, gw, ws, logits_out=glog)
    lg = glog.cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(gidx.cpu().numpy(), out["idx"])
    u = 2.0 ** -24
    d = route_depth(cfg.H, T)
    bound = d * u / (1 - d * u) * (np.abs(x) @ np.abs(L["W_r"].astype(np.float64)).T) \
        + 2 * u * np.abs(logits)
    if L["bias"] is not None:
        bound += u * np.abs(L["bias"].astype(np.float64))
    assert (np.abs(lg - logits) <= bound).all()
    fi, fw = O.route_topk(lg, cfg.k)
    np.testing.assert_array_equal(out["idx"], fi)
    np.testing.assert_allclose(out["w"], fw, atol=1e-5, rtol=0)
    check_routing(L, {"logits": logits, "idx": idx, "w": w}, out["idx"], out["w"], cfg.k, cfg.H,
                  max_ties=T // 10)


def test_prefill_2048_tensor_core_path(big):
    cfg, L, D = big
    out = gpu_layer(L, D, cfg, moe.MOE_PATH_GEMM, moe.MOE_ACT_MXFP4)
    _check_all_routing(cfg, L, D, out)
    _check(cfg, L, out, _sample(cfg.T, 10, 1), "mxfp4_act")


def test_prefill_4096_tensor_core_path(big):
    """The 4096-token prefill chunk: buckets reach about 400 tokens, so work
    items span up to four token tiles."""
    cfg, L, D = big
    cfg4 = cfg.with_T(4096)
    L4 = dict(L)
    L4["x"] = synth.activations(cfg, 0, 4096)
    D4 = dict(D)
    D4["x"] = torch.from_numpy(L4["x"].view(np.int16)).cuda()
    out = gpu_layer(L4, D4, cfg4, moe.MOE_PATH_GEMM, moe.MOE_ACT_MXFP4)
    counts = np.bincount(out["idx"].reshape(-1), minlength=cfg.E)
    assert counts.max() > 3 * 128
    _check_all_routing(cfg4, L4, D4, out)
    # the tokens of the largest bucket plus a random sample
    big_e = int(counts.argmax())
    in_big = np.nonzero((out["idx"] == big_e).any(axis=1))[0]
    toks = np.union1d(in_big[:: max(1, in_big.size // 6)][:6], _sample(4096, 6, 5))
    _check(cfg4, L4, out, toks, "mxfp4_act")


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
