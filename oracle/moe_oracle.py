"""fp64 CPU oracle: routed mixture-of-SwiGLU-experts layer over MXFP4 weights.

TEST INFRASTRUCTURE ONLY -- imported by tests/, __graft_entry__.smoke() and the
CPU-baseline / reference arm of bench.py, never by the product path.  It shares
no code with the CUDA library (no kernels, headers, tables or helpers).

What the layer computes, and where the pages say so
---------------------------------------------------
* Only the experts a token activates are read and run -- "ds4-ssd" README,
  intro ("SSD-streamed routed-MoE sidecar path") and ainews.cool "antirez ds4
  DeepSeek Metal inference", section 技术深度解析 (block-sparse MoE matmul that
  loads only the activated experts' weights; fine-grained experts, top-k
  routing).
* Routed experts are stored as MXFP4 -- "ds4-ssd" README, "Run SSD Sidecar
  Mode" (native package with bit-exact MXFP4 routed experts); the element
  format (E2M1 codes, one E8M0 power-of-two scale per 32 values) is the OCP
  Microscaling Formats (MX) v1.0 specification's.
* ``--moe-expert-topk`` changes the number of routed experts per token
  ("ds4-ssd" README, "Experimental Pro Support"), i.e. k is a parameter.
* A shared (always-on) expert with its own down projection exists ("ds4-ssd"
  README, "Experimental Pro Support": shared-down decode prefetch).
* ``--quality`` / ``--no-int8`` select exact, non-accelerated arithmetic
  ("ds4-ssd" README, "Experimental Pro Support"); the fast prefill path on
  the pages quantises activations for an accelerator ("ds4-ssd" README,
  "Attribution": GPU int8 dequant/packing feeding the ANE).  Here: mode
  ``"exact"`` and mode ``"mxfp4_act"``.

The pages print no formula for the router, softmax, top-k, SwiGLU or combine;
the plainest reading is taken for each and written next to the function.

Readings where the pages are silent (the CUDA library takes the same ones):
  R1 nibble order: byte b of a row holds element 2b in its low nibble and 2b+1
     in its high nibble; scale byte q covers elements 32q..32q+31 along the
     row's contiguous (input) dimension.
  R2 router bias b is added to the logits before the softmax and used for both
     selection and weights.
  R3 top-k ties break towards the lower expert index; indices are listed in
     descending logit order.
  R4 no routed scaling factor (1.0); renormalised weights sum to one.
  R5 SwiGLU: h = silu(g) * u with silu(z) = z / (1 + e^-z); g from the gate
     projection, u from the up projection.
  R6 the shared expert is added with weight 1.
  R7 mode "mxfp4_act": each projection's input is quantised per row in
     32-element blocks with the OCP rule (scale 2^(floor(log2 amax) - 2)),
     round-to-nearest-even onto the E2M1 grid with saturation at +-6.
  R8 combine sums routed slots in slot order j = 0..k-1, then the shared
     expert; the reported output is that sum rounded to bf16 (RNE).
  R9 E8M0 byte 255 decodes to NaN.

Parity is pinned by tests/test_oracle_pins.py (exhaustive decode against
ml_dtypes, k = E dense mixture, one-hot routing, invariants, brute force).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "E2M1_TABLE", "e8m0_to_f64", "decode_mxfp4", "bf16_bits_to_f64",
    "f64_to_bf16_bits", "router_logits", "route_topk", "bucket_by_expert",
    "silu", "quantise_mxfp4_rows", "dequantise_mxfp4_rows", "expert_ffn",
    "decode_expert", "layer_forward", "near_tie_tokens", "expert_bytes",
]

# --------------------------------------------------------------------------
# MXFP4 element and scale decode (OCP MX v1.0, FP4 E2M1 and E8M0 tables)
# --------------------------------------------------------------------------
#: value of each 4-bit E2M1 code: bit 3 sign, bits 2..1 exponent (bias 1),
#: bit 0 mantissa; code 1 is the subnormal 0.5.
E2M1_TABLE = np.array(
    [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
     -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0], dtype=np.float64)


def e8m0_to_f64(s):
    """E8M0 scale byte -> 2^(s-127); byte 255 is NaN (reading R9)."""
    s = np.asarray(s, dtype=np.int64)
    out = np.ldexp(1.0, s - 127).astype(np.float64)
    return np.where(s == 255, np.nan, out)


def decode_mxfp4(q: np.ndarray, s: np.ndarray, K: int) -> np.ndarray:
    """Decode MXFP4 rows: codes q [..., K/2] u8, scales s [..., K/32] u8 -> [..., K] f64.

    Element value = E2M1_TABLE[code] * 2^(scale - 127) (OCP MX v1.0); nibble
    order and block axis per reading R1.
    """
    assert K % 32 == 0
    q = np.asarray(q, dtype=np.uint8)
    s = np.asarray(s, dtype=np.uint8)
    assert q.shape[-1] == K // 2 and s.shape[-1] == K // 32
    codes = np.empty(q.shape[:-1] + (K,), dtype=np.uint8)
    codes[..., 0::2] = q & 0x0F
    codes[..., 1::2] = q >> 4
    vals = E2M1_TABLE[codes]
    scale = np.repeat(e8m0_to_f64(s), 32, axis=-1)
    with np.errstate(invalid="ignore"):
        return vals * scale


def expert_bytes(H: int, I: int) -> int:
    """Bytes of one MXFP4 expert (gate, up: [I,H]; down: [H,I]): codes + scales."""
    per_matrix = H * I // 2 + H * I // 32
    return 3 * per_matrix


# --------------------------------------------------------------------------
# bf16 <-> f64
# --------------------------------------------------------------------------
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact f64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round f64 to bf16 with round-to-nearest-even in one step (no double rounding).

    bf16: 8 significant bits, normal exponents -126..127, subnormal spacing 2^-133.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.float64)
    finite = np.isfinite(v)
    a = np.abs(np.where(finite, v, 0.0))
    m, e = np.frexp(a)                       # a = m * 2^e, m in [0.5, 1)
    # quantum (spacing) of bf16 at this magnitude: 2^(e - 8), floored at 2^-133
    qexp = np.maximum(e - 8, -133)
    r = np.round(np.ldexp(a, -qexp)) * 1.0    # np.round: half to even
    mag = np.ldexp(r, qexp)
    mag = np.where(mag > 3.3895313892515355e38, np.inf, mag)  # above bf16 max
    out[...] = np.where(finite, np.copysign(mag, v), v)
    f32 = out.astype(np.float32)              # exact: every bf16 value is an f32
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# --------------------------------------------------------------------------
# Router, softmax, top-k, renormalise  (readings R2, R3, R4)
# --------------------------------------------------------------------------
def router_logits(x: np.ndarray, W_r: np.ndarray, bias=None) -> np.ndarray:
    """logits[t, e] = sum_h x[t,h] * W_r[e,h] + b[e], in f64."""
    logits = np.asarray(x, np.float64) @ np.asarray(W_r, np.float64).T
    if bias is not None:
        logits = logits + np.asarray(bias, np.float64)[None, :]
    return logits


def route_topk(logits: np.ndarray, k: int):
    """softmax over all experts, pick the k largest, renormalise the chosen k.

    Returns idx [T,k] int32 (descending logit, ties -> lower index) and w [T,k].
    """
    logits = np.asarray(logits, np.float64)
    T, E = logits.shape
    assert 1 <= k <= E
    zmax = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - zmax)
    p = p / p.sum(axis=1, keepdims=True)
    # stable sort of the negated logits keeps the lower index first among ties
    order = np.argsort(-logits, axis=1, kind="stable")
    idx = order[:, :k].astype(np.int32)
    chosen = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    w = chosen / chosen.sum(axis=1, keepdims=True)
    return idx, w


def near_tie_tokens(x: np.ndarray, W_r: np.ndarray, bias, logits: np.ndarray,
                    k: int, depth: int) -> np.ndarray:
    """Tokens whose fp32 top-(k+1) order is not decided by the exact logits.

    A float32 sum in which every product meets at most ``depth`` roundings has
    error at most gamma_depth * sum_h |x_h W_r[e,h]| (+ |b_e| u for the bias),
    gamma_n = n u / (1 - n u), u = 2^-24 (Higham, Accuracy and Stability of
    Numerical Algorithms, sec. 3.1/4.2).  A token is a near-tie when two of its
    k+1 largest logits, adjacent in order, are closer than the sum of their
    bounds, or when the (k+1)-th is that close to the k-th.
    """
    u = 2.0 ** -24
    g = depth * u / (1.0 - depth * u)
    absdot = np.abs(np.asarray(x, np.float64)) @ np.abs(np.asarray(W_r, np.float64)).T
    err = g * absdot + (2 * u) * np.abs(logits)
    if bias is not None:
        err = err + u * np.abs(np.asarray(bias, np.float64))[None, :]
    T, E = logits.shape
    kk = min(k + 1, E)
    order = np.argsort(-logits, axis=1, kind="stable")[:, :kk]
    top = np.take_along_axis(logits, order, axis=1)
    te = np.take_along_axis(err, order, axis=1)
    gaps = top[:, :-1] - top[:, 1:]
    bound = te[:, :-1] + te[:, 1:]
    return np.nonzero((gaps <= bound).any(axis=1))[0] if kk > 1 else np.zeros(0, np.int64)


# --------------------------------------------------------------------------
# Bucket: stable counting sort of (token, slot) pairs by expert
# --------------------------------------------------------------------------
def bucket_by_expert(idx: np.ndarray, E: int):
    """Pairs p = t*k + j sorted by expert idx[t, j], ascending p within an expert.

    Returns counts [E], offsets [E+1] (exclusive scan, offsets[E] = T*k) and
    entries [T*k] holding pair indices.
    """
    flat = np.asarray(idx, np.int64).reshape(-1)
    counts = np.zeros(E, dtype=np.int32)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int32)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    cursor = offsets[:-1].copy()
    entries = np.empty(flat.size, dtype=np.int32)
    for p, e in enumerate(flat):          # ascending p keeps the sort stable
        entries[cursor[e]] = p
        cursor[e] += 1
    return counts, offsets, entries


# --------------------------------------------------------------------------
# MXFP4 activation quantisation (mode "mxfp4_act", reading R7)
# --------------------------------------------------------------------------
_E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def quantise_mxfp4_rows(v: np.ndarray):
    """Quantise rows [R, K] to MXFP4 codes [R, K/2] u8 and scales [R, K/32] u8.

    Per 32-element block: amax = max|v|; scale exponent
    X = clamp(floor(log2 amax) - 2, -127, 127) (OCP MX v1.0, emax of E2M1 is 2);
    amax = 0 gives X = -127 and all codes 0.  Each element v / 2^X goes to the
    nearest E2M1 magnitude; an exact tie goes to the code with mantissa bit 0;
    magnitudes above 6 saturate to 6.  Negative inputs keep the sign bit.
    """
    v = np.asarray(v, np.float64)
    R, K = v.shape
    assert K % 32 == 0
    blocks = v.reshape(R, K // 32, 32)
    amax = np.abs(blocks).max(axis=2)
    X = np.full(amax.shape, -127, dtype=np.int64)
    nz = amax > 0
    _, e = np.frexp(np.where(nz, amax, 1.0))        # amax = m 2^e, m in [0.5,1)
    X = np.where(nz, np.clip((e - 1) - 2, -127, 127), X)
    scaled = blocks / np.ldexp(1.0, X)[:, :, None]
    mag = np.abs(scaled)
    dist = np.abs(mag[..., None] - _E2M1_MAGS)      # [R, nb, 32, 8]
    best = dist.min(axis=-1, keepdims=True)
    cand = dist == best
    # among equal distances prefer an even code (mantissa bit 0); codes 0..7
    # are ordered by magnitude, so ties are two neighbours: pick the even one.
    even = (np.arange(8) % 2 == 0)
    pick_even = cand & even
    has_even = pick_even.any(axis=-1)
    code = np.where(has_even, np.argmax(pick_even, axis=-1), np.argmax(cand, axis=-1))
    sign = (np.signbit(scaled)).astype(np.int64)
    nib = (code + 8 * sign).astype(np.uint8).reshape(R, K)
    q = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    s = (X + 127).astype(np.uint8)
    return q, s


def dequantise_mxfp4_rows(v: np.ndarray) -> np.ndarray:
    """v -> decode(quantise(v)): the values a projection sees in mode mxfp4_act."""
    v = np.asarray(v, np.float64)
    q, s = quantise_mxfp4_rows(v)
    return decode_mxfp4(q, s, v.shape[1])


# --------------------------------------------------------------------------
# Expert FFN (reading R5) and the whole layer
# --------------------------------------------------------------------------
def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z / (1 + e^-z), f64."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def decode_expert(experts: dict, e: int, H: int, I: int):
    """Decoded f64 matrices (gate [I,H], up [I,H], down [H,I]) of expert e."""
    Wg = decode_mxfp4(experts["gate_q"][e], experts["gate_s"][e], H)
    Wu = decode_mxfp4(experts["up_q"][e], experts["up_s"][e], H)
    Wd = decode_mxfp4(experts["down_q"][e], experts["down_s"][e], I)
    return Wg, Wu, Wd


def expert_ffn(Wg, Wu, Wd, X, mode: str = "exact"):
    """o = W_down (silu(W_gate x) * (W_up x)) for each row x of X [R, H]."""
    X = np.asarray(X, np.float64)
    xin = dequantise_mxfp4_rows(X) if mode == "mxfp4_act" else X
    g = xin @ Wg.T
    u = xin @ Wu.T
    h = silu(g) * u
    hin = dequantise_mxfp4_rows(h) if mode == "mxfp4_act" else h
    return hin @ Wd.T


def layer_forward(x_bits, W_r, bias, experts: dict, shared, k: int,
                  mode: str = "exact", tokens=None):
    """The whole routed layer for the rows of x_bits (bf16 bits [T, H]).

    experts: dict of gate_q [E,I,H/2], gate_s [E,I,H/32], up_q, up_s (same),
    down_q [E,H,I/2], down_s [E,H,I/32] (uint8); shared: same with E = 1, or None.
    ``tokens`` restricts the computation to those rows (the layer is per-token).

    Returns a dict with logits, idx, w, counts, offsets, entries, partial
    [T*k + S*T, H] (rows p = t*k + j, then T*k + t for the shared expert),
    y (f64, reading R8) and y_bf16 (uint16 bits).
    """
    x_bits = np.asarray(x_bits, np.uint16)
    if tokens is not None:
        x_bits = x_bits[np.asarray(tokens)]
    x = bf16_bits_to_f64(x_bits)
    T, H = x.shape
    E = experts["gate_q"].shape[0]
    I = experts["gate_q"].shape[1]
    logits = router_logits(x, np.asarray(W_r, np.float64), bias)
    idx, w = route_topk(logits, k)
    counts, offsets, entries = bucket_by_expert(idx, E)
    S = 1 if shared is not None else 0
    partial = np.zeros((T * k + S * T, H), dtype=np.float64)
    for e in range(E):
        rows = entries[offsets[e]:offsets[e + 1]]
        if rows.size == 0:
            continue
        Wg, Wu, Wd = decode_expert(experts, e, H, I)
        toks = rows // k
        partial[rows] = expert_ffn(Wg, Wu, Wd, x[toks], mode)
    if S:
        Wg, Wu, Wd = decode_expert(shared, 0, H, I)
        partial[T * k:] = expert_ffn(Wg, Wu, Wd, x, mode)
    y = np.zeros((T, H), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            y[t] += w[t, j] * partial[t * k + j]
        if S:
            y[t] += partial[T * k + t]
    return {
        "logits": logits, "idx": idx, "w": w, "counts": counts,
        "offsets": offsets, "entries": entries, "partial": partial,
        "y": y, "y_bf16": f64_to_bf16_bits(y),
    }
