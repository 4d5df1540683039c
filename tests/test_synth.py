"""The seeded input generator: determinism, layouts and value distributions."""
import numpy as np
import ml_dtypes

from routed_expert_ffn_fp32_b200 import synth


def test_deterministic_and_prefix_stable():
    a = synth.layer(synth.TINY, seed=0)
    b = synth.layer(synth.TINY, seed=0)
    for key in ("x", "W_r"):
        np.testing.assert_array_equal(a[key], b[key])
    for n in a["experts"]:
        np.testing.assert_array_equal(a["experts"][n], b["experts"][n])
    x8 = synth.activations(synth.TINY, 0, T=8)
    np.testing.assert_array_equal(x8[:4], a["x"])
    c = synth.layer(synth.TINY, seed=1)
    assert not np.array_equal(a["experts"]["gate_q"], c["experts"]["gate_q"])


def test_layouts():
    cfg = synth.TINY
    L = synth.layer(cfg)
    ex = L["experts"]
    assert ex["gate_q"].shape == (cfg.E, cfg.I, cfg.H // 2)
    assert ex["gate_s"].shape == (cfg.E, cfg.I, cfg.H // 32)
    assert ex["down_q"].shape == (cfg.E, cfg.H, cfg.I // 2)
    assert ex["down_s"].shape == (cfg.E, cfg.H, cfg.I // 32)
    assert L["x"].dtype == np.uint16 and L["x"].shape == (cfg.T, cfg.H)
    assert L["W_r"].dtype == np.float32 and L["bias"] is None and L["shared"] is None


def test_weight_distribution_matches_normal():
    """Decoded weights (via ml_dtypes) have the drawn N(0, 0.02) spread."""
    q, s = synth.mxfp4_matrices(np.random.default_rng(0), 4, 64, 256, 0.02)
    nib = np.stack([q & 0xF, q >> 4], -1).reshape(4, 64, 256).astype(np.uint8)
    v = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    v = v * np.repeat(s.view(ml_dtypes.float8_e8m0fnu).astype(np.float64), 32, axis=-1)
    assert abs(v.std() - 0.02) < 0.002
    assert abs(v.mean()) < 0.001
    assert s.min() > 100 and s.max() < 130          # no 0 / 255 scale bytes
    # the largest element of each block encodes to magnitude 4 or 6 (OCP scale rule)
    mags = np.abs(v.reshape(-1, 32)) / np.repeat(
        s.view(ml_dtypes.float8_e8m0fnu).astype(np.float64).reshape(-1, 1), 1, axis=1)
    assert set(np.unique(mags.max(axis=1))) <= {4.0, 6.0}


def test_pool_path_distribution():
    old = synth.POOL_BLOCKS
    synth.POOL_BLOCKS = 1 << 12
    try:
        q, s = synth.mxfp4_matrices(np.random.default_rng(1), 2, 256, 512, 0.02)
    finally:
        synth.POOL_BLOCKS = old
    assert q.shape == (2, 256, 256) and s.shape == (2, 256, 16)
    assert 110 < np.median(s) < 125


def test_zipf_bias():
    W_r, b = synth.router(synth.FINEGRAINED)
    assert W_r.shape == (256, 4096) and abs(W_r.std() - 0.02) < 1e-3
    ranks = np.round(np.exp(-b / (synth.ZIPF_ALPHA * 1.0))).astype(int)
    assert sorted(ranks.tolist()) == list(range(1, 257))
    _, b0 = synth.router(synth.DECODE64)
    assert b0 is None


def test_bf16_rne():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5], np.float32)
    bits = synth.bf16_bits_rne(v)
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020]
