"""Edge inputs of the CUDA path against the fp64 oracle, through the C ABI.

* token rows of extreme magnitude (2^-40 .. 2^56) and of wide dynamic range
  within a row, on the row-block GEMV, the K-split GEMV and the tensor-core
  path: per-token relative L2 within 2e-3 of the oracle rounded to bf16;
* token rows holding an infinity or a NaN: that token's output is non-finite,
  every other token still matches the oracle;
* the special E8M0 scale bytes (0 = 2^-127, 1, 254 = 2^127, 255 = NaN) through
  the expert kernels: expert partial rows within 1e-4 (exact activations) /
  2e-3 (MXFP4 activations) of the oracle, NaN exactly where the oracle has NaN;
* one workspace, sized for the largest shape, reused across shapes in the
  order that puts a small shape's counters on a large shape's leftovers;
* the bounded-wait error path: a wait that nothing satisfies latches
  MOE_ERR_TIMEOUT within its limit, and the next call is correct again.
"""
import time

import numpy as np
import pytest
import torch

import oracle as O
from routed_expert_ffn_fp32_b200 import build, moe, synth

from helpers import (bits_np, check_routing, check_y, dev_layer, gpu_layer, rel_l2,
                     rel_l2_rows, to_dev_bits)

pytestmark = pytest.mark.gpu

EXACT, MXFP4 = moe.MOE_ACT_EXACT, moe.MOE_ACT_MXFP4
GEMV, GEMM = moe.MOE_PATH_GEMV, moe.MOE_PATH_GEMM


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load_library()


def _cfg(H, I, E, k, T, shared=False, bias=False, std=0.05):
    return synth.LayerConfig("edge", H, I, E, k, T, std, 1.0 if bias else None, shared)


def _mode(precision):
    return "mxfp4_act" if precision == MXFP4 else "exact"


# --------------------------------------------------- token magnitudes ---
#: log2 of the scale of each token row
ROW_SCALES = [-40, -20, 0, 20, 40, 56]


def _extreme_rows(x_bits, H):
    """Rows of N(0,1) scaled by 2^s for s in ROW_SCALES, a row whose 32-value
    blocks alternate between 2^24 and 2^-24, and a row with exact zeros."""
    x = O.bf16_bits_to_f64(x_bits)
    rows = [x[i] * 2.0 ** s for i, s in enumerate(ROW_SCALES)]
    blk = np.repeat((np.arange(H // 32) % 2) * 48.0 - 24.0, 32)
    rows.append(x[len(ROW_SCALES)] * np.exp2(blk))
    r = x[len(ROW_SCALES) + 1].copy()
    r[::3] = 0.0
    rows.append(r)
    return O.f64_to_bf16_bits(np.stack(rows))


@pytest.mark.parametrize("H,I,E,k,shared,path,precision", [
    (256, 128, 8, 2, False, GEMV, EXACT),    # row-block GEMV (mma.sync)
    (256, 128, 8, 2, True, GEMV, MXFP4),     # row-block GEMV, MXFP4 activations
    (160, 96, 4, 2, True, GEMV, EXACT),      # K-split GEMV (H, I not multiples of 128)
    (256, 128, 8, 2, True, GEMM, MXFP4),     # tcgen05 block-scaled path
])
def test_extreme_token_magnitudes(H, I, E, k, shared, path, precision):
    T = len(ROW_SCALES) + 2
    cfg = _cfg(H, I, E, k, T, shared)
    L = synth.layer(cfg, 31)
    L["x"] = _extreme_rows(L["x"], H)
    ref = O.layer_forward(L["x"], L["W_r"], L["bias"], L["experts"], L["shared"], k,
                          _mode(precision))
    assert np.isfinite(O.bf16_bits_to_f64(ref["y_bf16"])).all()
    out = gpu_layer(L, dev_layer(L), cfg, path, precision)
    check_routing(L, ref, out["idx"], out["w"], k, H)
    check_y(out["y"], ref)


def test_nonfinite_token_rows_stay_local():
    cfg = _cfg(256, 128, 8, 2, 5, shared=True)
    L = synth.layer(cfg, 32)
    x = L["x"].copy()
    x[1, 17] = 0x7F80   # +inf
    x[3, 200] = 0xFFC0  # NaN
    L["x"] = x
    out = gpu_layer(L, dev_layer(L), cfg, GEMV, EXACT)
    y = O.bf16_bits_to_f64(out["y"])
    assert (~np.isfinite(y[1])).all() and (~np.isfinite(y[3])).all()
    good = [0, 2, 4]
    ref = O.layer_forward(x, L["W_r"], L["bias"], L["experts"], L["shared"], cfg.k, tokens=good)
    assert (~np.isfinite(O.layer_forward(x, L["W_r"], L["bias"], L["experts"], L["shared"],
                                         cfg.k, tokens=[1, 3])["y"])).all()
    check_routing({"x": x[good], "W_r": L["W_r"], "bias": L["bias"]}, ref, out["idx"][good],
                  out["w"][good], cfg.k, cfg.H, T_route=cfg.T)
    check_y(out["y"][good], ref)


# ------------------------------------------------- E8M0 special bytes ---
def _special_scale_case(case, with_nan):
    """Experts of a 4-expert layer with special scale bytes, and the layer
    inputs (x bits) that keep the oracle's results finite apart from NaN."""
    H, I, E, k, T = 256, 128, 4, 2, 8
    cfg = _cfg(H, I, E, k, T)
    L = synth.layer(cfg, 33)
    ex = {n: a.copy() for n, a in L["experts"].items()}
    x = O.bf16_bits_to_f64(L["x"])
    if case == "byte0":
        # every gate weight scaled by 2^-127 (the subnormal): small but
        # nonzero outputs; the tokens are scaled up so they stay float32-normal
        ex["gate_s"][:] = 0
        x = x * 2.0 ** 10
    elif case == "byte1":
        ex["up_s"][:] = 1
        x = x * 2.0 ** 10
    elif case == "byte254":
        # one up block per expert at 2^127 holding a single 0.5 (element 6 of
        # row 5): u[5] is about 8.5e37 times that token value
        ex["up_s"][:, 5, 0] = 254
        ex["up_q"][:, 5, :16] = 0
        ex["up_q"][:, 5, 3] = 0x01
        x[:, 6] = 1.0
    if with_nan:
        ex["gate_s"][3, 2, 1] = 255   # expert 3: gate row 2, block 1 is NaN
    L["experts"] = ex
    L["x"] = O.f64_to_bf16_bits(x)
    return cfg, L


@pytest.mark.parametrize("case", ["byte0", "byte1", "byte254"])
@pytest.mark.parametrize("path,precision", [(GEMV, EXACT), (GEMV, MXFP4), (GEMM, MXFP4)])
def test_special_scale_bytes_through_expert_kernels(case, path, precision):
    # NaN (byte 255) with exact activations only: quantising a block that
    # holds a NaN to MXFP4 has no defined result
    with_nan = path == GEMV and precision == EXACT
    cfg, L = _special_scale_case(case, with_nan)
    ref = O.layer_forward(L["x"], L["W_r"], None, L["experts"], None, cfg.k, _mode(precision))
    assert (ref["counts"] > 0).all()
    D = dev_layer(L)
    shape = moe.shape_of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = moe.make_workspace(shape, path, precision, False)
    rows = cfg.T * cfg.k
    partial = torch.zeros((rows, cfg.H), dtype=torch.float32, device="cuda")
    moe.moe_expert_ffn_mxfp4(D["experts"], None, D["x"], torch.from_numpy(ref["offsets"]).cuda(),
                             torch.from_numpy(ref["entries"]).cuda(), shape, partial, ws, path,
                             precision)
    torch.cuda.synchronize()
    assert moe.moe_get_error(ws) == 0
    got = partial.cpu().numpy().astype(np.float64)
    want = ref["partial"]
    nan_rows = np.isnan(want).all(axis=1)
    assert nan_rows.sum() == (ref["idx"] == 3).sum() if with_nan else not nan_rows.any()
    assert np.isnan(got[nan_rows]).all()
    fin = ~nan_rows
    assert np.isfinite(want[fin]).all()
    tol = 1e-4 if precision == EXACT else 2e-3
    err = rel_l2_rows(got[fin], want[fin])
    assert err.max() < tol, (case, int(err.argmax()), float(err.max()))


def test_decode_scale_bytes_match_hardware_conversion():
    """Every E8M0 byte through moe_decode_mxfp4 (the conversion the row-block
    GEMV uses) with one code of each magnitude: 2^(s-127) times the code,
    byte 0 the subnormal 2^-127, byte 255 NaN."""
    q = np.tile(np.array([0x21, 0x43, 0x65, 0x07] * 4, np.uint8), (256, 1))  # codes 1..7, 0
    s = np.arange(256, dtype=np.uint8).reshape(256, 1)
    out = torch.empty((256, 32), dtype=torch.float32, device="cuda")
    moe.moe_decode_mxfp4(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), 32, out)
    got = out.cpu().numpy()
    with np.errstate(over="ignore"):
        want = O.decode_mxfp4(q, s, 32).astype(np.float32)
    assert np.isnan(got[255]).all() and np.isnan(want[255]).all()
    np.testing.assert_array_equal(got[:255], want[:255])
    assert got[0, 0] == np.float32(0.5 * 2.0 ** -127)


# ------------------------------------------------ workspace across shapes ---
def test_one_workspace_across_shapes_regular_entry():
    """One workspace sized for the largest of the shapes, reused in the order
    fine-grained T=5 -> decode64 T=5 -> decode64 T=1 -> fine-grained T=1: each
    output matches the oracle and no call runs into a wait limit."""
    fg, d64 = synth.FINEGRAINED, synth.DECODE64
    order = [(fg, 5), (d64, 5), (d64, 1), (fg, 1)]
    size = max(moe.moe_workspace_bytes(moe.shape_of(T, c.H, c.I, c.E, c.k), GEMV, EXACT, c.shared)
               for c, T in order)
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    moe.moe_workspace_init(ws)
    # leftovers everywhere: a call's scratch must not depend on the bytes it finds
    ws.fill_(0x5A)
    moe.moe_workspace_init(ws.narrow(0, 0, 512))
    layers = {}
    for c, T in order:
        if c.name not in layers:
            L = synth.layer(c, 3, 5)
            layers[c.name] = (L, dev_layer(L))
        L, D = layers[c.name]
        x = L["x"][:T]
        shape = moe.shape_of(T, c.H, c.I, c.E, c.k)
        y = torch.empty((T, c.H), dtype=torch.int16, device="cuda")
        idx = torch.empty((T, c.k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, c.k), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        moe.moe_layer_forward(D["x"][:T].contiguous(), D["W_r"], D["bias"], D["experts"],
                              D["shared"], shape, y, ws, GEMV, EXACT, idx, w)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
        assert moe.moe_get_error(ws) == 0, (c.name, T)
        assert dt < 0.5, (c.name, T, dt)
        ref = O.layer_forward(x, L["W_r"], L["bias"], L["experts"], L["shared"], c.k)
        check_routing({"x": x, "W_r": L["W_r"], "bias": L["bias"]}, ref, idx.cpu().numpy(),
                      w.cpu().numpy(), c.k, c.H)
        check_y(bits_np(y), ref)


# --------------------------------------------------- bounded-wait path ---
def test_expired_wait_latches_timeout_and_next_call_recovers():
    cfg = synth.DECODE64
    T = 5
    L = synth.layer(cfg, 4, T)
    D = dev_layer(L)
    shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = moe.make_workspace(shape, GEMV, EXACT)
    y = torch.empty((T, cfg.H), dtype=torch.int16, device="cuda")
    # a 1 ms limit, and the first warp's first stage left without copies
    moe.moe_workspace_set_limits(ws, 1000, moe.MOE_DEBUG_STARVE_FIRST_WAIT)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    moe.moe_layer_forward(D["x"], D["W_r"], None, D["experts"], None, shape, y, ws, GEMV, EXACT)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 1.0
    assert moe.moe_get_error(ws) == moe.MOE_ERR_TIMEOUT
    assert moe.moe_get_error(ws) == moe.MOE_OK          # read once, then cleared
    moe.moe_workspace_set_limits(ws, 0, 0)
    moe.moe_layer_forward(D["x"], D["W_r"], None, D["experts"], None, shape, y, ws, GEMV, EXACT)
    torch.cuda.synchronize()
    assert moe.moe_get_error(ws) == moe.MOE_OK
    ref = O.layer_forward(L["x"], L["W_r"], None, L["experts"], None, cfg.k)
    check_y(bits_np(y), ref)


def test_expired_wait_on_tensor_core_path_latches_timeout():
    """The same on the tcgen05 GEMM: its first CTA's first stage gets no tile
    copies, the MMA thread's wait on it runs out within the 1 ms limit, the
    other roles give up too and free TMEM; the next call is correct."""
    T = 200
    cfg = _cfg(1024, 512, 16, 4, T, shared=True, bias=True)
    L = synth.layer(cfg, 6)
    D = dev_layer(L)
    shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = moe.make_workspace(shape, GEMM, MXFP4, True)
    y = torch.empty((T, cfg.H), dtype=torch.int16, device="cuda")
    moe.moe_workspace_set_limits(ws, 1000, moe.MOE_DEBUG_STARVE_FIRST_WAIT)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    moe.moe_layer_forward(D["x"], D["W_r"], D["bias"], D["experts"], D["shared"], shape, y, ws,
                          GEMM, MXFP4)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 1.0
    assert moe.moe_get_error(ws) == moe.MOE_ERR_TIMEOUT
    moe.moe_workspace_set_limits(ws, 0, 0)
    moe.moe_layer_forward(D["x"], D["W_r"], D["bias"], D["experts"], D["shared"], shape, y, ws,
                          GEMM, MXFP4)
    torch.cuda.synchronize()
    assert moe.moe_get_error(ws) == moe.MOE_OK
    ref = O.layer_forward(L["x"], L["W_r"], L["bias"], L["experts"], L["shared"], cfg.k,
                          "mxfp4_act")
    check_y(bits_np(y), ref)
