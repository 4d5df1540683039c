"""Seeded synthetic inputs for the routed MoE layer (shared by tests and bench).

This module only draws random inputs and stores them in the layouts the
library reads; it holds none of the layer's arithmetic (no routing, no
decoding, no FFN).  Weights are drawn N(0, std) and stored as MXFP4 with the
OCP scale choice 2^(floor(log2 amax) - 2) per 32-value block and the nearest
E2M1 magnitude (midpoint thresholds); activations are N(0, 1) rounded to bf16.

Large weight sets are filled from a pool of 2^20 independently drawn and
encoded blocks, each block of the output picked uniformly from the pool: every
block has the distribution of an encoded N(0, std) block while generation
stays a few seconds per GB.

Workloads (the decode64 shape is the 64-expert, top-2 model of the ainews.cool
"antirez ds4 DeepSeek Metal inference" page; the fine-grained shape stands for
the 284B DeepSeek-V4-Flash layer of the pawin.top ds4 guide and the ds4-ssd
README, with its shared expert; the pages print no per-layer dimensions, so
H, I and E are readings):
  tiny          H 256,  I 128,  E 8,   k 2, T 4,   router N(0,.05), no bias
  decode64      H 4096, I 1408, E 64,  k 2, T 1|5, router N(0,.02), no bias
  finegrained   H 4096, I 2048, E 256, k 8, T 1|5, shared expert, Zipf s=1.0 bias
  prefill       finegrained layer, T 2048|4096, Zipf s=1.2 bias
  sweep         8 finegrained layers, T in {1,2,4,5,8,16,32,64,128,512}, Zipf s=1.2
"""
from __future__ import annotations

import dataclasses

import numpy as np

ZIPF_ALPHA = 0.13          # bias scale giving prefill buckets of ~30..200 tokens
POOL_BLOCKS = 1 << 20


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    H: int
    I: int
    E: int
    k: int
    T: int
    router_std: float
    zipf_s: float | None      # None: no router bias (uniform routing)
    shared: bool
    weight_std: float = 0.02

    def with_T(self, T: int) -> "LayerConfig":
        return dataclasses.replace(self, T=T)


TINY = LayerConfig("tiny_h256_i128_e8_k2", 256, 128, 8, 2, 4, 0.05, None, False)
DECODE64 = LayerConfig("decode_h4096_i1408_e64_k2", 4096, 1408, 64, 2, 5, 0.02, None, False)
FINEGRAINED = LayerConfig("finegrained_h4096_i2048_e256_k8_shared", 4096, 2048, 256, 8, 5,
                          0.02, 1.0, True)
PREFILL = LayerConfig("prefill_h4096_i2048_e256_k8_shared_zipf1.2", 4096, 2048, 256, 8, 2048,
                      0.02, 1.2, True)
SWEEP = LayerConfig("sweep_h4096_i2048_e256_k8_shared_zipf1.2", 4096, 2048, 256, 8, 1,
                    0.02, 1.2, True)
SWEEP_T = (1, 2, 4, 5, 8, 16, 32, 64, 128, 512)
SWEEP_LAYERS = 8

CONFIGS = {c.name: c for c in (TINY, DECODE64, FINEGRAINED, PREFILL, SWEEP)}

# 16 E2M1 magnitudes (codes 0..7) and the midpoints between neighbours
_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
_MIDS = (_MAGS[:-1] + _MAGS[1:]) / 2.0


def _encode_blocks(v: np.ndarray):
    """[nb, 32] float -> codes [nb, 16] u8 (element 2i low nibble) and scales [nb] u8."""
    v = np.asarray(v, dtype=np.float32)
    amax = np.abs(v).max(axis=1)
    _, e = np.frexp(np.where(amax > 0, amax, np.float32(1.0)))   # amax = m 2^e, m in [.5,1)
    X = np.where(amax > 0, np.clip(e.astype(np.int64) - 1 - 2, -127, 127), -127)
    y = np.abs(v) * np.exp2(-X.astype(np.float32))[:, None]       # exact power-of-two scaling
    mag_code = np.zeros(v.shape, dtype=np.uint8)
    for mid in _MIDS.astype(np.float32):                           # nearest magnitude
        mag_code += (y > mid)
    nib = mag_code | (np.signbit(v).astype(np.uint8) << 3)
    q = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return q, (X + 127).astype(np.uint8)


def _encoded_normal_blocks(rng: np.random.Generator, nb: int, std: float):
    """nb independent N(0, std) blocks of 32, encoded (in chunks to bound temporaries)."""
    q = np.empty((nb, 16), dtype=np.uint8)
    s = np.empty(nb, dtype=np.uint8)
    step = 1 << 16
    for a in range(0, nb, step):
        b = min(nb, a + step)
        v = rng.standard_normal(size=(b - a, 32), dtype=np.float32) * np.float32(std)
        q[a:b], s[a:b] = _encode_blocks(v)
    return q, s


def mxfp4_matrices(rng: np.random.Generator, n: int, rows: int, K: int, std: float):
    """n matrices [rows, K] of N(0, std) stored as MXFP4: q [n,rows,K/2], s [n,rows,K/32]."""
    assert K % 32 == 0
    nb_mat = rows * K // 32
    total = n * nb_mat
    if total <= POOL_BLOCKS:
        q, s = _encoded_normal_blocks(rng, total, std)
        return q.reshape(n, rows, K // 2), s.reshape(n, rows, K // 32)
    pq, ps = _encoded_normal_blocks(rng, POOL_BLOCKS, std)
    q = np.empty((n, rows, K // 2), dtype=np.uint8)
    s = np.empty((n, rows, K // 32), dtype=np.uint8)
    for m in range(n):
        pick = rng.integers(0, POOL_BLOCKS, size=nb_mat, dtype=np.int64)
        q[m] = pq[pick].reshape(rows, K // 2)
        s[m] = ps[pick].reshape(rows, K // 32)
    return q, s


def bf16_bits_rne(v: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def activations(cfg: LayerConfig, seed: int = 0, T: int | None = None) -> np.ndarray:
    """x [T, H] bf16 bits, N(0, 1); the first rows do not depend on T."""
    T = cfg.T if T is None else T
    rng = np.random.default_rng(np.random.SeedSequence([seed, 1]))
    return bf16_bits_rne(rng.standard_normal(size=(T, cfg.H), dtype=np.float32))


def router(cfg: LayerConfig, seed: int = 0):
    """W_r [E, H] f32 ~ N(0, router_std); bias [E] f32 or None.

    Bias: b_e = ZIPF_ALPHA * (-s * ln r_e), r_e a seeded permutation rank 1..E,
    so expert popularity falls off like a Zipf law of exponent s.
    """
    rng = np.random.default_rng(np.random.SeedSequence([seed, 2]))
    W_r = rng.normal(0.0, cfg.router_std, size=(cfg.E, cfg.H)).astype(np.float32)
    if cfg.zipf_s is None:
        return W_r, None
    rank = rng.permutation(cfg.E).astype(np.float64) + 1.0
    bias = (ZIPF_ALPHA * (-cfg.zipf_s * np.log(rank))).astype(np.float32)
    return W_r, bias


def experts(cfg: LayerConfig, seed: int = 0, n: int | None = None, stream: int = 3) -> dict:
    """MXFP4 expert weights: gate/up [n, I, H], down [n, H, I] as codes + scales."""
    n = cfg.E if n is None else n
    ss = np.random.SeedSequence([seed, stream])
    r_gate, r_up, r_down = (np.random.default_rng(c) for c in ss.spawn(3))
    gq, gs = mxfp4_matrices(r_gate, n, cfg.I, cfg.H, cfg.weight_std)
    uq, us = mxfp4_matrices(r_up, n, cfg.I, cfg.H, cfg.weight_std)
    dq, ds = mxfp4_matrices(r_down, n, cfg.H, cfg.I, cfg.weight_std)
    return {"gate_q": gq, "gate_s": gs, "up_q": uq, "up_s": us,
            "down_q": dq, "down_s": ds}


def layer(cfg: LayerConfig, seed: int = 0, T: int | None = None) -> dict:
    """All inputs of one layer call."""
    W_r, bias = router(cfg, seed)
    return {
        "cfg": cfg if T is None else cfg.with_T(T),
        "x": activations(cfg, seed, T),
        "W_r": W_r,
        "bias": bias,
        "experts": experts(cfg, seed),
        "shared": experts(cfg, seed, n=1, stream=4) if cfg.shared else None,
    }
