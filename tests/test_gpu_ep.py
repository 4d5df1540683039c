"""Expert parallelism with the CUDA kernels, the ranks emulated one after the
other on one GPU.

Each emulated rank runs ep_partial (router, bucket, the expert FFNs of its
experts -- and the shared expert on rank 0 -- and the range-restricted
float32 combine) with the library's kernels; the float32 partial outputs are
added as the all-reduce would add them, and ep_finish rounds the sum to bf16.
The result must match the single-device fp64 oracle like the single-device
layer: routing bit-exact, the largest per-token relative L2 within 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle as O
from routed_expert_ffn_fp32_b200 import build, ep, moe, synth

from helpers import bits_np, check_y, dev_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load_library()


CASES = [
    # workload (or H, I, E, k, shared), T, ranks, precision
    ("decode_h4096_i1408_e64_k2", 5, 2, moe.MOE_ACT_EXACT),
    ("finegrained_h4096_i2048_e256_k8_shared", 5, 4, moe.MOE_ACT_EXACT),
    ("finegrained_h4096_i2048_e256_k8_shared", 3, 8, moe.MOE_ACT_MXFP4),
    ((512, 256, 16, 8, True), 6, 4, moe.MOE_ACT_EXACT),     # 4 experts per rank, k = 8
    ((256, 128, 12, 3, False), 40, 2, moe.MOE_ACT_EXACT),   # unequal shards, unfused router
]


@pytest.mark.parametrize("wl,T,world,precision", CASES)
def test_expert_parallel_ranks_emulated(wl, T, world, precision):
    if isinstance(wl, str):
        cfg = synth.CONFIGS[wl]
    else:
        H, I, E, k, shared = wl
        cfg = synth.LayerConfig("ep", H, I, E, k, T, 0.05, 1.0, shared)
    L = synth.layer(cfg, 51, T)
    D = dev_layer(L)
    mode = "mxfp4_act" if precision == moe.MOE_ACT_MXFP4 else "exact"
    ref = O.layer_forward(L["x"], L["W_r"], L["bias"], L["experts"], L["shared"], cfg.k, mode)
    shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
    total = torch.zeros((T, cfg.H), dtype=torch.float32, device="cuda")
    for r in range(world):
        shard = ep.ExpertShard.from_full(D["experts"], D["shared"], world, r)
        ws = torch.empty(ep.ep_workspace_bytes(shape, shard, precision=precision),
                         dtype=torch.uint8, device="cuda")
        moe.moe_workspace_init(ws)
        y32, idx, w = ep.ep_partial(D["x"], D["W_r"], D["bias"], shard, shape, ws,
                                    precision=precision)
        torch.cuda.synchronize()
        assert moe.moe_get_error(ws) == 0
        np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
        total += y32          # the all-reduce's sum over ranks
    y = torch.empty((T, cfg.H), dtype=torch.int16, device="cuda")
    ep.ep_finish(total, y)
    torch.cuda.synchronize()
    check_y(bits_np(y), ref)
