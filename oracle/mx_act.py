"""O1 oracle of the layer's block-scaled numerics variant -- TEST INFRASTRUCTURE ONLY.

The MXFP4 layer (GPT-OSS expert weights in E2M1 codes with an E8M0 scale per 32
elements along K: "GPT-OSS 20B GGUF with MoE CPU Offloading", Model
Specifications; group size 32 for the 4-bit and MXFP8 formats: "Ollama
glm4_moe_lite.go", ``quantizationParams``) can also run with its *activations*
in MXFP8 -- the inputs of both expert projections, x_perm and h, quantized to
E4M3 elements with one E8M0 scale per 32 consecutive elements along K -- so that
the tensor cores multiply the 8-bit activations by the 4-bit weights directly,
each product scaled by the two blocks' scales.  The pages name the format and
its group size, not how a layer quantizes to it; the readings here are:

  * E4M3 (OCP 8-bit floating point, the "fn" form): sign bit 7, exponent bits
    6..3 with bias 7, mantissa bits 2..0; exponent field 0 is subnormal
    (m * 2^-9); no infinities; S.1111.111 is NaN; the largest finite value is
    1.75 * 2^8 = 448;
  * the scale of a block is 2^X with X the smallest integer for which the
    block's largest magnitude is at most 448 * 2^X, so no element saturates
    (X = -127, the smallest E8M0 scale, for an all-zero block; X is clamped to
    [-127, 127]);
  * each element is v / 2^X rounded to the nearest E4M3 value, ties to the
    value with an even mantissa;
  * the quantized value is that E4M3 value times 2^X; everything else is the
    plain layer (``moe_oracle``) in float64.

All arithmetic is float64 on exact values: v / 2^X is exact (a power of two),
and the rounding is done on the exact quotient.
"""
from __future__ import annotations

from typing import Dict, Tuple

import numpy as np

from . import moe_oracle as O

E4M3_MAX = 448.0
BLOCK = 32


def e4m3_value(code) -> np.ndarray:
    """Value of 8-bit E4M3 codes (NaN for S.1111.111)."""
    c = np.asarray(code).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    man = c & 0x7
    mag = np.where(ex == 0, man * 2.0 ** -9, np.ldexp(1.0 + man / 8.0, ex - 7))
    mag = np.where((ex == 0xF) & (man == 0x7), np.nan, mag)
    return sign * mag


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest E4M3 value, ties to an even mantissa.

    Magnitudes above 448 saturate to 448 (the scale rule never produces them).
    The grid near |v|: spacing 2^(e-3) for normal values in [2^e, 2^(e+1)),
    e >= -6; spacing 2^-9 below 2^-6 (subnormals).
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    # exact binade: correct floor(log2) where it is off by one at powers of two
    e = np.where(np.ldexp(1.0, e.astype(np.int64)) > a, e - 1, e)
    e = np.where(np.ldexp(1.0, (e + 1).astype(np.int64)) <= a, e + 1, e)
    e = np.maximum(e, -6.0)
    step = np.ldexp(1.0, (e - 3).astype(np.int64))
    q = a / step                       # exact: a power-of-two divisor
    r = np.floor(q)
    frac = q - r
    up = (frac > 0.5) | ((frac == 0.5) & (np.mod(r, 2) == 1))
    r = r + up
    out = np.minimum(r * step, E4M3_MAX)
    return np.where(v < 0, -out, out)


def scale_exponent(amax: np.ndarray) -> np.ndarray:
    """X: the smallest integer with amax <= 448 * 2^X (-127 for amax = 0), clamped to [-127, 127]."""
    amax = np.asarray(amax, dtype=np.float64)
    pos = amax > 0
    m, e = np.frexp(np.where(pos, amax, 1.0))   # amax = m * 2^e, m in [0.5, 1)
    # amax = (2m) * 2^(e-1) with 2m in [1, 2); 448 = 1.75 * 2^8
    X = (e - 1) - 8 + (2.0 * m > 1.75)
    X = np.where(pos, X, -127)
    return np.clip(X, -127, 127).astype(np.int64)


def quantize(a: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """MXFP8 along the last axis (length a multiple of 32).

    Returns (the dequantized values, float64 like ``a``; the scale exponents X
    [..., K/32]).  Block j covers elements 32 j .. 32 j + 31.
    """
    a = np.asarray(a, dtype=np.float64)
    K = a.shape[-1]
    if K % BLOCK:
        raise ValueError("MXFP8 needs the reduction length to be a multiple of 32")
    blocks = a.reshape(*a.shape[:-1], K // BLOCK, BLOCK)
    X = scale_exponent(np.max(np.abs(blocks), axis=-1))
    s = np.ldexp(1.0, X)[..., None]
    q = e4m3_round(blocks / s) * s
    return q.reshape(a.shape), X


def layer_tokens(layer: Dict[str, np.ndarray], tokens: np.ndarray, k: int, limit: float,
                 alpha: float = 1.702) -> Dict[str, np.ndarray]:
    """The layer for selected tokens with MXFP8 activations in both expert projections.

    Router, top-k and softmax as in ``moe_oracle`` (bf16 x, exact).  For each
    chosen expert: g, u = q(x) W^T + b, h = clipped SwiGLU(g, u),
    o = q(h) W_d^T + b_d with q the MXFP8 quantizer above; y = sum_j w_j o_j.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    x = O.decode(layer["x"][tokens])
    logits = x @ O.decode(layer["w_router"]).T + O.decode(layer["b_router"])[None, :]
    ids, w = O.topk_softmax(logits, k)
    xq, _ = quantize(x)
    D = layer["b_down"].shape[1]
    F = layer["b_gate"].shape[1]
    h = np.zeros((tokens.size, k, F))
    o = np.zeros((tokens.size, k, D))
    for e in np.unique(ids):
        e = int(e)
        ii, jj = np.nonzero(ids == e)
        xs = xq[ii]
        g = xs @ O.expert_weights(layer, "gate", e).T + O.decode(layer["b_gate"][e])
        u = xs @ O.expert_weights(layer, "up", e).T + O.decode(layer["b_up"][e])
        hh = O.clipped_swiglu(g, u, limit, alpha)
        h[ii, jj] = hh
        o[ii, jj] = quantize(hh)[0] @ O.expert_weights(layer, "down", e).T + O.decode(layer["b_down"][e])
    y = np.zeros((tokens.size, D))
    for j in range(k):
        y += w[:, j:j + 1] * o[:, j]
    return dict(logits=logits, ids=ids, w=w, h=h, y=y)
