"""Shared test helpers: device upload of synthetic layers and comparisons."""
import numpy as np
import torch

import oracle as O
from routed_expert_ffn_fp32_b200 import moe, synth

#: bf16 layer output vs the oracle rounded to bf16 (relative L2)
TOL_Y = 2e-3
#: combine weights, absolute
TOL_W = 1e-5


def route_depth(H: int, T: int = 1) -> int:
    """Roundings any router product meets in the route kernels: up to 32
    tokens, a lane chain of H/128 products, 5 shuffle levels, 3 quarter sums
    and the bias; above 32 tokens, a 32-product chunk, H/32 chunk sums and the
    bias."""
    return H // 128 + 9 if T <= 32 else 32 + H // 32 + 1


def to_dev_bits(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def dev_layer(L: dict) -> dict:
    return {
        "x": to_dev_bits(L["x"]),
        "W_r": torch.from_numpy(L["W_r"]).cuda(),
        "bias": None if L["bias"] is None else torch.from_numpy(L["bias"]).cuda(),
        "experts": moe.Experts.from_numpy(L["experts"]),
        "shared": None if L["shared"] is None else moe.Experts.from_numpy(L["shared"]),
    }


def bits_np(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def rel_l2_rows(a, b) -> np.ndarray:
    """Relative L2 error of each row (token) of a against b."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    num = np.linalg.norm(a - b, axis=-1)
    den = np.linalg.norm(b, axis=-1)
    return num / np.where(den > 0, den, 1.0)


def check_y(got_bits, ref, tol=TOL_Y):
    """Layer output against the oracle: the largest per-token relative L2
    error within tol (against the oracle rounded to bf16 and against its
    unrounded value), every value finite.  Returns (max per token, batch)."""
    got = O.bf16_bits_to_f64(got_bits)
    want = O.bf16_bits_to_f64(ref["y_bf16"])
    assert np.isfinite(got).all()
    per_tok = rel_l2_rows(got, want)
    assert per_tok.max() < tol, (int(per_tok.argmax()), float(per_tok.max()))
    assert rel_l2_rows(got, ref["y"]).max() < tol
    return float(per_tok.max()), rel_l2(got, want)


def gpu_layer(L: dict, D: dict, cfg, path=moe.MOE_PATH_AUTO, precision=moe.MOE_ACT_EXACT):
    T = L["x"].shape[0]
    shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
    has_sh = D["shared"] is not None
    ws = moe.make_workspace(shape, path, precision, has_sh)
    y = torch.empty((T, cfg.H), dtype=torch.int16, device="cuda")
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    moe.moe_layer_forward(D["x"], D["W_r"], D["bias"], D["experts"], D["shared"], shape, y, ws,
                          path, precision, idx, w)
    torch.cuda.synchronize()
    assert moe.moe_get_error(ws) == 0
    return {"y": bits_np(y), "idx": idx.cpu().numpy(), "w": w.cpu().numpy(), "ws": ws}


def check_routing(L, ref, idx, w, k, H, T_route=None, max_ties=0):
    """idx bit-exact except near-ties (which must still be a valid top-k);
    w within TOL_W where idx agrees.  T_route: the batch size the GPU routed
    (selects the kernel's summation bound; default idx rows).  At most
    max_ties near-ties are expected (none on the seeded workloads).  Returns
    the near-tie token indices."""
    x = O.bf16_bits_to_f64(L["x"])
    T_route = idx.shape[0] if T_route is None else T_route
    ties = O.near_tie_tokens(x, L["W_r"], L["bias"], ref["logits"], k, route_depth(H, T_route))
    assert len(ties) <= max_ties, f"{len(ties)} near-tie tokens: {ties[:10]}"
    clear = np.setdiff1d(np.arange(idx.shape[0]), ties)
    np.testing.assert_array_equal(idx[clear], ref["idx"][clear])
    np.testing.assert_allclose(w[clear], ref["w"][clear], atol=TOL_W, rtol=0)
    for t in ties:
        assert len(set(idx[t].tolist())) == k
        kth = np.sort(ref["logits"][t])[::-1][k - 1]
        assert (ref["logits"][t, idx[t]] >= kth - 1e-3).all()
    return ties
