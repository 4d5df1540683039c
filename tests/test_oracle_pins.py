"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test checks the oracle against an independent source: a library routine
(ml_dtypes, scipy, torch), a closed form, a special case of the layer that
reduces to a dense computation written differently (einsum), an invariant, or
a brute-force pure-Python recomputation.  A plausible slip in the oracle (a
dropped term, a wrong sign, a transposed operand, a swapped nibble, a wrong
renormalisation) fails at least one of them.
"""
import math
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import scipy.special
import torch

import oracle as O
from routed_expert_ffn_fp32_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_table():
    e2m1, e8m0 = {}, {}
    with open(os.path.join(GOLDEN, "e2m1_e8m0_ocp_mx_v1.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kind, a, b = line.split()
            if kind == "e2m1":
                e2m1[int(a)] = float(b)
            else:
                e8m0[int(a)] = float(b)
    return e2m1, e8m0


# ---------------------------------------------------------------- decode ---
def test_e2m1_table_matches_ocp_golden():
    e2m1, _ = _golden_table()
    assert len(e2m1) == 16
    for c, v in e2m1.items():
        assert O.E2M1_TABLE[c] == v
        assert math.copysign(1.0, O.E2M1_TABLE[c]) == math.copysign(1.0, v)


def test_e8m0_matches_ocp_golden():
    _, e8m0 = _golden_table()
    for s, lg in e8m0.items():
        got = O.e8m0_to_f64(np.array([s]))[0]
        if math.isnan(lg):
            assert math.isnan(got)
        else:
            assert got == 2.0 ** lg


def test_decode_exhaustive_against_ml_dtypes():
    """All 16 codes x 256 scale bytes, in both nibble positions."""
    codes = np.arange(16, dtype=np.uint8)
    elem = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    scales = np.arange(256, dtype=np.uint8)
    sc = scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    # one 32-element row per (scale, code-pair): element 2b = lo, 2b+1 = hi
    for s in range(256):
        lo = np.tile(codes, 2)                 # 32 codes
        hi = np.roll(lo, 5)
        q = (lo[0::2] | (hi[1::2] << 4)).astype(np.uint8)  # packs lo[2b], hi[2b+1]
        nib = np.empty(32, np.uint8)
        nib[0::2] = lo[0::2]
        nib[1::2] = hi[1::2]
        got = O.decode_mxfp4(q[None, :], np.array([[s]], np.uint8), 32)[0]
        want = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64) * sc[s]
        if s == 255:
            assert np.isnan(got).all()
        else:
            np.testing.assert_array_equal(got, want)
            np.testing.assert_array_equal(np.signbit(got), np.signbit(want))
    assert elem[1] == 0.5 and elem[7] == 6.0 and elem[9] == -0.5


def test_decode_closed_form_bitfields():
    """value = (-1)^s 2^(E-1) (1 + m/2) for E > 0, (-1)^s m/2 for E = 0."""
    for c in range(16):
        s, E, m = c >> 3, (c >> 1) & 3, c & 1
        mag = (2.0 ** (E - 1)) * (1 + m / 2) if E else m / 2
        v = -mag if s else mag
        for sb in (0, 1, 120, 127, 140, 254):
            q = np.full((1, 16), c | (c << 4), np.uint8)
            got = O.decode_mxfp4(q, np.array([[sb]], np.uint8), 32)[0]
            assert (got == v * 2.0 ** (sb - 127)).all()


def test_decode_row_layout_blocks_follow_K():
    """Scale byte q multiplies elements 32q..32q+31 only."""
    q = np.full((1, 64), 0x22, np.uint8)        # every element 1.0, K = 128
    s = np.array([[127, 128, 126, 130]], np.uint8)
    got = O.decode_mxfp4(q, s, 128)[0]
    for b, sb in enumerate(s[0]):
        assert (got[32 * b:32 * b + 32] == 2.0 ** (int(sb) - 127)).all()


# ------------------------------------------------------------------ bf16 ---
def _bf16_nearest_brute(v: float) -> int:
    """Bits of the bf16 nearest to v (ties to even mantissa) by exact search."""
    f = np.float32(v)
    base = int(np.array([f], np.float32).view(np.uint32)[0] >> 16)
    cands = []
    for b in range(max(0, base - 2), min(0xFFFF, base + 3) + 1):
        for bits in (b, b | 0x8000, b & 0x7FFF):
            val = np.array([bits << 16], np.uint32).view(np.float32)[0]
            if np.isfinite(val):
                cands.append((abs(Fraction(float(val)) - Fraction(v)), bits & 1, bits))
    cands.sort()
    best = cands[0]
    ties = [c for c in cands if c[0] == best[0]]
    even = [c for c in ties if c[1] == 0]
    return (even or ties)[0][2]


def test_bf16_rounding_brute_force():
    rng = np.random.default_rng(5)
    vals = list(rng.normal(size=300) * 10.0 ** rng.integers(-30, 30, 300))
    # exact halfway cases between bf16 neighbours (tie -> even)
    for b in (0x3F80, 0x3F81, 0x4049, 0xC2F7):
        lo = np.array([b << 16], np.uint32).view(np.float32)[0]
        hi = np.array([(b + 1) << 16], np.uint32).view(np.float32)[0]
        vals.append((float(lo) + float(hi)) / 2)
    # f64 values just off the f32 grid (would double-round via f32)
    vals.append(1.0 + 2.0 ** -8 + 2.0 ** -40)
    vals.append(-(1.0 + 2.0 ** -8 - 2.0 ** -40))
    got = O.f64_to_bf16_bits(np.array(vals))
    for v, g in zip(vals, got):
        assert int(g) == _bf16_nearest_brute(v), v


def test_bf16_rounding_matches_torch_on_f32_inputs():
    rng = np.random.default_rng(6)
    v32 = rng.normal(size=4096).astype(np.float32)
    want = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.f64_to_bf16_bits(v32.astype(np.float64)), want)
    back = O.bf16_bits_to_f64(want)
    np.testing.assert_array_equal(back, torch.from_numpy(v32).to(torch.bfloat16).double().numpy())


# ---------------------------------------------------------------- router ---
def test_route_matches_scipy_softmax_and_torch_topk():
    rng = np.random.default_rng(7)
    logits = rng.normal(size=(64, 32)) * 1.3
    k = 5
    idx, w = O.route_topk(logits, k)
    p = scipy.special.softmax(logits, axis=1)
    tv, ti = torch.topk(torch.from_numpy(logits), k, dim=1)
    np.testing.assert_array_equal(idx, ti.numpy())
    chosen = np.take_along_axis(p, ti.numpy(), 1)
    np.testing.assert_allclose(w, chosen / chosen.sum(1, keepdims=True), rtol=1e-14)


def test_renormalised_topk_equals_softmax_over_topk_logits():
    rng = np.random.default_rng(8)
    logits = rng.normal(size=(40, 256)) * 2.0
    idx, w = O.route_topk(logits, 8)
    top = np.take_along_axis(logits, idx.astype(np.int64), 1)
    np.testing.assert_allclose(w, scipy.special.softmax(top, axis=1), rtol=1e-13, atol=0)


def test_route_invariants_and_ties():
    rng = np.random.default_rng(9)
    logits = rng.normal(size=(50, 64))
    idx, w = O.route_topk(logits, 6)
    for t in range(50):
        assert len(set(idx[t].tolist())) == 6
        assert np.all(np.diff(logits[t, idx[t]]) <= 0)
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-12)
    tied = np.zeros((1, 8))
    tied[0, [6, 2, 5]] = 1.0
    idx, w = O.route_topk(tied, 2)
    assert idx.tolist() == [[2, 5]]
    assert (w == 0.5).all()


def test_router_logits_bias_and_layout():
    rng = np.random.default_rng(10)
    x = rng.normal(size=(3, 16))
    W = rng.normal(size=(5, 16))
    b = rng.normal(size=5)
    got = O.router_logits(x, W, b)
    want = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(W), torch.from_numpy(b))
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-13)


# ---------------------------------------------------------------- bucket ---
def test_bucket_matches_stable_argsort_and_invariants():
    rng = np.random.default_rng(11)
    T, E, k = 97, 16, 4
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, entries = O.bucket_by_expert(idx, E)
    want = torch.argsort(torch.from_numpy(idx.reshape(-1).astype(np.int64)), stable=True).numpy()
    np.testing.assert_array_equal(entries, want)
    assert counts.sum() == T * k and offsets[-1] == T * k and offsets[0] == 0
    np.testing.assert_array_equal(np.sort(entries), np.arange(T * k))
    np.testing.assert_array_equal(np.bincount(idx.reshape(-1), minlength=E), counts)
    for e in range(E):
        seg = entries[offsets[e]:offsets[e + 1]]
        assert (idx.reshape(-1)[seg] == e).all()
        assert np.all(np.diff(seg // k) > 0)          # ascending token


# ----------------------------------------------------- MXFP4 activations ---
def test_act_quantiser_matches_ml_dtypes_and_scale_rule():
    rng = np.random.default_rng(12)
    v = rng.normal(size=(16, 256)) * 10.0 ** rng.integers(-3, 3, size=(16, 1))
    v[3, 32:64] = 0.0                                  # an all-zero block
    v[4, :32] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.9] * 4) * 1.0  # amax 7.9 -> X = 0
    q, s = O.quantise_mxfp4_rows(v)
    X = s.astype(np.int64) - 127
    for r in range(16):
        for b in range(8):
            blk = v[r, 32 * b:32 * b + 32]
            amax = np.abs(blk).max()
            if amax == 0:
                assert s[r, b] == 0
                continue
            assert 2.0 ** (X[r, b] + 2) <= amax < 2.0 ** (X[r, b] + 3)
            want = (blk / 2.0 ** X[r, b]).astype(np.float32).astype(ml_dtypes.float4_e2m1fn)
            got = O.decode_mxfp4(q[r:r + 1, 16 * b:16 * b + 16], s[r:r + 1, b:b + 1], 32)[0]
            np.testing.assert_array_equal(got, want.astype(np.float64) * 2.0 ** X[r, b])
    ties = O.dequantise_mxfp4_rows(v[4:5, :32])[0, :8]
    np.testing.assert_array_equal(ties, [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0])


def test_act_quantiser_nearest_brute_force():
    rng = np.random.default_rng(13)
    v = rng.normal(size=(4, 64))
    deq = O.dequantise_mxfp4_rows(v)
    q, s = O.quantise_mxfp4_rows(v)
    grid = np.array(sorted(set(O.E2M1_TABLE.tolist())))
    for r in range(4):
        for i in range(64):
            sc = 2.0 ** (int(s[r, i // 32]) - 127)
            best = min(abs(v[r, i] - g * sc) for g in grid)
            assert abs(v[r, i] - deq[r, i]) <= best + 1e-300 or abs(v[r, i]) > 6 * sc


# ------------------------------------------------------- whole layer -------
def _small_layer(seed=0, H=64, I=32, E=6, k=2, T=5, shared=False, bias=False):
    cfg = synth.LayerConfig("t", H, I, E, k, T, 0.1, 1.0 if bias else None, shared, 0.05)
    return synth.layer(cfg, seed)


def _dense_ffn(Wg, Wu, Wd, x):
    g = np.einsum("ih,th->ti", Wg, x)
    u = np.einsum("ih,th->ti", Wu, x)
    h = g * scipy.special.expit(g) * u
    return np.einsum("di,ti->td", Wd, h)


@pytest.mark.parametrize("shared", [False, True])
def test_k_equals_E_is_dense_softmax_mixture(shared):
    L = _small_layer(seed=3, E=5, k=5, shared=shared, bias=True)
    r = O.layer_forward(L["x"], L["W_r"], L["bias"], L["experts"], L["shared"], 5)
    x = L["x"].astype(np.uint32) << 16
    x = x.view(np.float32).astype(np.float64)
    logits = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(L["W_r"].astype(np.float64)),
                                        torch.from_numpy(L["bias"].astype(np.float64))).numpy()
    p = scipy.special.softmax(logits, axis=1)
    H, I = 64, 32
    y = np.zeros_like(r["y"])
    ex = L["experts"]
    for e in range(5):
        Wg = ex["gate_q"][e]
        mats = [np.asarray(ml_dtypes_decode(ex[n + "_q"][e], ex[n + "_s"][e])) for n in ("gate", "up", "down")]
        y += p[:, e:e + 1] * _dense_ffn(*mats, x)
    if shared:
        sh = L["shared"]
        mats = [ml_dtypes_decode(sh[n + "_q"][0], sh[n + "_s"][0]) for n in ("gate", "up", "down")]
        y += _dense_ffn(*mats, x)
    np.testing.assert_allclose(r["y"], y, rtol=1e-11, atol=1e-14)


def ml_dtypes_decode(q, s):
    """Independent MXFP4 decode through ml_dtypes (rows [R, K/2] -> [R, K])."""
    R, half = q.shape
    nib = np.stack([q & 0xF, q >> 4], axis=-1).reshape(R, 2 * half).astype(np.uint8)
    vals = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sc = s.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    return vals * np.repeat(sc, 32, axis=1)


def test_one_hot_routing_is_single_expert():
    L = _small_layer(seed=4, E=6, k=1, T=3)
    W_r = np.zeros_like(L["W_r"])
    bias = np.zeros(6, np.float32)
    bias[4] = 50.0
    r = O.layer_forward(L["x"], W_r, bias, L["experts"], None, 1)
    assert (r["idx"][:, 0] == 4).all() and (r["w"] == 1.0).all()
    x = (L["x"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ex = L["experts"]
    mats = [ml_dtypes_decode(ex[n + "_q"][4], ex[n + "_s"][4]) for n in ("gate", "up", "down")]
    np.testing.assert_allclose(r["y"], _dense_ffn(*mats, x), rtol=1e-12, atol=1e-15)


def test_zero_experts_leave_shared_only():
    L = _small_layer(seed=5, shared=True)
    ex = {n: np.zeros_like(a) for n, a in L["experts"].items()}
    r = O.layer_forward(L["x"], L["W_r"], None, ex, L["shared"], 2)
    x = (L["x"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    sh = L["shared"]
    mats = [ml_dtypes_decode(sh[n + "_q"][0], sh[n + "_s"][0]) for n in ("gate", "up", "down")]
    np.testing.assert_allclose(r["y"], _dense_ffn(*mats, x), rtol=1e-12, atol=1e-15)
    r0 = O.layer_forward(L["x"], L["W_r"], None, ex, None, 2)
    assert (r0["y"] == 0).all()


def test_token_permutation_equivariance():
    L = _small_layer(seed=6, T=9, E=8, k=3, shared=True, bias=True)
    r = O.layer_forward(L["x"], L["W_r"], L["bias"], L["experts"], L["shared"], 3)
    perm = np.random.default_rng(1).permutation(9)
    rp = O.layer_forward(L["x"][perm], L["W_r"], L["bias"], L["experts"], L["shared"], 3)
    np.testing.assert_array_equal(rp["idx"], r["idx"][perm])
    np.testing.assert_allclose(rp["w"], r["w"][perm], rtol=1e-15)
    np.testing.assert_allclose(rp["y"], r["y"][perm], rtol=1e-12, atol=1e-16)
    np.testing.assert_array_equal(rp["counts"], r["counts"])


def _brute_layer(x_bits, W_r, bias, ex, k):
    """Pure-Python loops: bit-field decode, explicit sums, math.exp."""
    def dec(qrow, srow, K):
        out = []
        for i in range(K):
            byte = int(qrow[i // 2])
            c = (byte & 0xF) if i % 2 == 0 else (byte >> 4)
            s, E, m = c >> 3, (c >> 1) & 3, c & 1
            mag = (2.0 ** (E - 1)) * (1 + m / 2) if E else m / 2
            out.append((-mag if s else mag) * 2.0 ** (int(srow[i // 32]) - 127))
        return out

    T, H = x_bits.shape
    E, I = ex["gate_q"].shape[:2]
    xs = [[float(np.array([int(b) << 16], np.uint32).view(np.float32)[0]) for b in row] for row in x_bits]
    W = {n: [[dec(ex[n + "_q"][e][r], ex[n + "_s"][e][r], H if n != "down" else I)
              for r in range(I if n != "down" else H)] for e in range(E)] for n in ("gate", "up", "down")}
    ys = []
    for t in range(T):
        lg = [sum(xs[t][h] * float(W_r[e][h]) for h in range(H)) + (float(bias[e]) if bias is not None else 0.0)
              for e in range(E)]
        order = sorted(range(E), key=lambda e: (-lg[e], e))[:k]
        z = [math.exp(lg[e] - lg[order[0]]) for e in order]
        ws = [v / sum(z) for v in z]
        y = [0.0] * H
        for j, e in enumerate(order):
            g = [sum(W["gate"][e][i][h] * xs[t][h] for h in range(H)) for i in range(I)]
            u = [sum(W["up"][e][i][h] * xs[t][h] for h in range(H)) for i in range(I)]
            hh = [g[i] / (1 + math.exp(-g[i])) * u[i] for i in range(I)]
            for d in range(H):
                y[d] += ws[j] * sum(W["down"][e][d][i] * hh[i] for i in range(I))
        ys.append(y)
    return np.array(ys)


def test_brute_force_small_layer():
    L = _small_layer(seed=7, H=64, I=32, E=4, k=2, T=3, bias=True)
    r = O.layer_forward(L["x"], L["W_r"], L["bias"], L["experts"], None, 2)
    want = _brute_layer(L["x"], L["W_r"], L["bias"], L["experts"], 2)
    np.testing.assert_allclose(r["y"], want, rtol=1e-11, atol=1e-15)


def test_mxfp4_act_mode_quantises_both_projection_inputs():
    L = _small_layer(seed=8, H=64, I=64, E=3, k=1, T=4)
    ex = L["experts"]
    r = O.layer_forward(L["x"], L["W_r"], None, ex, None, 1, mode="mxfp4_act")
    x = (L["x"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(4):
        e = int(r["idx"][t, 0])
        Wg, Wu, Wd = (ml_dtypes_decode(ex[n + "_q"][e], ex[n + "_s"][e]) for n in ("gate", "up", "down"))
        xq = _ml_quant(x[t:t + 1])
        g, u = xq @ Wg.T, xq @ Wu.T
        h = g * scipy.special.expit(g) * u
        o = _ml_quant(h) @ Wd.T
        np.testing.assert_allclose(r["y"][t], o[0], rtol=1e-12, atol=1e-15)


def _ml_quant(v):
    """MX quantise-dequantise through ml_dtypes' float4_e2m1fn conversion."""
    out = np.empty_like(v)
    for r in range(v.shape[0]):
        for b in range(v.shape[1] // 32):
            blk = v[r, 32 * b:32 * b + 32]
            amax = np.abs(blk).max()
            X = -127 if amax == 0 else max(-127, min(127, math.floor(math.log2(amax)) - 2))
            q = (blk / 2.0 ** X).astype(np.float32).astype(ml_dtypes.float4_e2m1fn)
            out[r, 32 * b:32 * b + 32] = q.astype(np.float64) * 2.0 ** X
    return out


# ------------------------------------------------------------ byte model ---
def test_expert_byte_model():
    assert O.expert_bytes(256, 128) == 3 * 256 * 128 * 17 // 32
    assert O.expert_bytes(4096, 1408) == 9_191_424
    assert O.expert_bytes(4096, 2048) == 13_369_344
    ex = synth.experts(synth.TINY)
    assert sum(a.nbytes for a in ex.values()) == 8 * O.expert_bytes(256, 128)
    # 4.25 bits per routed weight: a 284B-parameter model in MXFP4 is ~151 GB of
    # routed experts, the order of the ~156 GB native package ("ds4-ssd" README,
    # "Run SSD Sidecar Mode"; 284B MoE per the pawin.top ds4 guide).
    assert 140e9 < 284e9 * 4.25 / 8 < 160e9


def test_near_tie_bound_flags_exact_ties_only_when_close():
    x = np.ones((2, 4))
    W = np.array([[1.0, 0, 0, 0], [1.0, 0, 0, 0], [0.5, 0, 0, 0]])
    logits = O.router_logits(x, W, None)
    ties = O.near_tie_tokens(x, W, None, logits, 1, depth=8)
    assert ties.tolist() == [0, 1]
    W2 = np.array([[1.0, 0, 0, 0], [0.5, 0, 0, 0], [0.25, 0, 0, 0]])
    assert O.near_tie_tokens(x, W2, None, O.router_logits(x, W2, None), 1, depth=8).size == 0


def _tie_threshold(depth, la, sa, sb, ba, bb):
    """Exact gap g at which logits la and la - g (with sum|x W| of sa and sb,
    biases ba and bb) meet the bound: g (1 + 2u) = gamma (sa + sb)
    + 4u la + u (|ba| + |bb|), u = 2^-24, gamma = depth u / (1 - depth u)."""
    u = Fraction(1, 2 ** 24)
    gamma = depth * u / (1 - depth * u)
    return (gamma * (Fraction(sa) + Fraction(sb)) + 4 * u * Fraction(la)
            + u * (abs(Fraction(ba)) + abs(Fraction(bb)))) / (1 + 2 * u)


@pytest.mark.parametrize("depth", [8, 41])
@pytest.mark.parametrize("bias", [None, (0.5, 0.25, 0.0)])
def test_near_tie_bound_magnitude_exact(depth, bias):
    """The near-tie bound is Higham's gamma_depth * sum|x W| plus 2u|logit|
    (plus u|b|) per logit, u = 2^-24: a gap just below the exact bound (as a
    rational) is a near-tie, one just above is not.  A wrong unit roundoff, a
    dropped gamma or a scaled bound moves one of the two cases across."""
    x = np.array([[1.0, 0.0, 0.0, 0.0]])
    W = np.array([[1.0, 0, 0, 0], [-1.0, 0, 0, 0], [0.125, 0, 0, 0]])
    b = None if bias is None else np.array(bias)
    bz = (0.0, 0.0, 0.0) if bias is None else bias
    eps = Fraction(1, 10 ** 6)
    # k = 1: the top two logits 1 and 1 - g
    g01 = _tie_threshold(depth, 1, 1, 1, bz[0], bz[1])
    for scale, expect_tie in ((1 - eps, True), (1 + eps, False)):
        logits = np.array([[1.0, 1.0 - float(g01 * scale), -10.0]])
        assert (O.near_tie_tokens(x, W, b, logits, 1, depth).size == 1) == expect_tie
    # k = 2: the order among the top k + 1 counts too; logits 1, 0.5 and
    # 0.5 - g (experts 1 and 2: sum|x W| 1 and 0.125)
    g12 = _tie_threshold(depth, 0.5, 1, 0.125, bz[1], bz[2])
    for scale, expect_tie in ((1 - eps, True), (1 + eps, False)):
        logits = np.array([[1.0, 0.5, 0.5 - float(g12 * scale)]])
        assert (O.near_tie_tokens(x, W, b, logits, 2, depth).size == 1) == expect_tie
