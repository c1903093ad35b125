"""O1 oracle: the GPT-OSS MoE FFN layer as its plain definition, numpy fp64.

TEST INFRASTRUCTURE ONLY -- see the package docstring.

Sources (page title, section):
  * "Ollama Imagegen GPT OSS" (leeroopedia), Description: the SwiGLU clips the
    gate to [0, limit] and the up projection to [-limit, limit] and uses a fixed
    alpha = 1.702 in the sigmoid; Signature: ``Config`` fields hidden_size,
    num_local_experts, num_experts_per_tok, swiglu_limit; ``swiGLU(gate, up,
    alpha, limit)``.
  * "maxtext gpt_oss weight mapping", "MoE Router" block: a router kernel and a
    router bias; "MOE EXPERTS" block: separate gate (wi_0) and up (wi_1)
    projections with biases, a down projection (wo) with a bias.
  * "GPT-OSS 20B GGUF with MoE CPU Offloading", Key Features / Model
    Specifications: 32 experts with 4 active per token; MXFP4 expert weights.
  * "Ollama glm4_moe_lite.go", ``SwitchMLP.Forward``: tokens are dispatched by
    an argsort of the flattened expert ids and un-permuted with the inverse
    order; ``MoE.Forward``: the output is the score-weighted sum of the k expert
    outputs.  (Its sigmoid router and plain SiLU are a different model and are
    not used here.)

Readings where the pages are silent (each is listed in the design notes):
  * top-k: the k largest logits, ties broken by the lower expert index; the
    selected ids are listed in descending-logit order;
  * routing weights: softmax over the k selected (biased) logits;
  * the down bias is part of each expert's output, i.e. it is weighted;
  * dispatch order: a *stable* sort by expert id, so rows of one expert are in
    increasing token order;
  * MXFP4: E2M1 code (sign bit 3, exponent bits 2..1 with bias 1, mantissa bit
    0), E8M0 scale 2^(s-127), 32-element blocks along the reduction dim,
    element 2i in the low nibble of byte i.

All arithmetic is float64 on the exact values of the (bf16 / fp32) inputs.
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import numpy as np


# --------------------------------------------------------------------------- #
# input decoding
# --------------------------------------------------------------------------- #
def decode(a: np.ndarray) -> np.ndarray:
    """Exact float64 values of an input array.

    uint16 arrays hold bf16 bit patterns; float32/float64 arrays are taken as is.
    """
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if a.dtype in (np.float32, np.float64):
        return a.astype(np.float64)
    raise TypeError(f"unsupported input dtype {a.dtype}")


def e2m1_value(code: np.ndarray) -> np.ndarray:
    """Value of 4-bit E2M1 codes: sign bit 3, two exponent bits (bias 1), one mantissa bit.

    exponent field 0 is subnormal: value = mantissa * 0.5; otherwise
    value = 2^(exp - 1) * (1 + mantissa / 2).
    """
    code = np.asarray(code).astype(np.int64)
    sign = np.where(code & 0x8, -1.0, 1.0)
    ex = (code >> 1) & 0x3
    man = code & 0x1
    mag = np.where(ex == 0, man * 0.5, np.ldexp(1.0 + man / 2.0, ex - 1))
    return sign * mag


def mxfp4_dequant(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Dequantise packed MXFP4 weights.

    q [..., N, K/2] uint8: element 2i of a row is the low nibble of byte i,
    element 2i+1 the high nibble.  s [..., N, K/32] uint8 E8M0 scale bytes:
    element j of a row is multiplied by 2^(s[j // 32] - 127).
    """
    lo = q & 0x0F
    hi = q >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(*q.shape[:-1], q.shape[-1] * 2)
    vals = e2m1_value(codes)
    scale = np.ldexp(1.0, s.astype(np.int64) - 127)
    return vals * np.repeat(scale, 32, axis=-1)


def expert_weights(layer: Dict[str, np.ndarray], name: str, e: Optional[int] = None) -> np.ndarray:
    """float64 weights of ``w_<name>`` (all experts, or expert e), dense or MXFP4."""
    w = layer[f"w_{name}"]
    if w.dtype == np.uint8:
        s = layer[f"s_{name}"]
        return mxfp4_dequant(w if e is None else w[e], s if e is None else s[e])
    return decode(w if e is None else w[e])


# --------------------------------------------------------------------------- #
# the layer, step by step
# --------------------------------------------------------------------------- #
def router_logits(x: np.ndarray, w_router: np.ndarray, b_router: np.ndarray) -> np.ndarray:
    """l[t, e] = sum_d x[t, d] * Wr[e, d] + br[e]  (router kernel + router bias)."""
    return decode(x) @ decode(w_router).T + decode(b_router)[None, :]


def topk_softmax(logits: np.ndarray, k: int) -> Tuple[np.ndarray, np.ndarray]:
    """The k largest logits per token and the softmax over them.

    ids[t, 0..k-1] are the selected experts in descending-logit order (ties:
    lower expert index first); w[t, j] = exp(l_j - l_max) / sum_i exp(l_i - l_max)
    over the selected logits only.
    """
    T, E = logits.shape
    # lexsort: the last key is the primary one -> by descending logit, then by expert index
    idx = np.broadcast_to(np.arange(E)[None, :], (T, E))
    order = np.lexsort((idx, -logits), axis=1)
    ids = order[:, :k]
    sel = np.take_along_axis(logits, ids, axis=1)
    m = sel[:, :1]
    ex = np.exp(sel - m)
    w = ex / ex.sum(axis=1, keepdims=True)
    return ids.astype(np.int32), w


def clipped_swiglu(g: np.ndarray, u: np.ndarray, limit: float, alpha: float = 1.702) -> np.ndarray:
    """h = gc * sigmoid(alpha * gc) * uc, gc = clip(g, 0, limit), uc = clip(u, -limit, limit)."""
    gc = np.minimum(np.maximum(g, 0.0), limit)
    uc = np.minimum(np.maximum(u, -limit), limit)
    return gc * (1.0 / (1.0 + np.exp(-alpha * gc))) * uc


def dispatch(ids: np.ndarray, E: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Stable sort of the (token, slot) pairs by expert id.

    Returns expert_off [E+1] (segment starts, expert_off[E] = T*k),
    row_of_slot [T, k] (the permuted row of pair (t, j)) and
    slot_of_row [T*k] (the flat slot t*k + j held by each permuted row);
    slot_of_row is the argsort ``order`` of the flattened ids, row_of_slot its
    inverse.
    """
    T, k = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")
    inv = np.empty_like(order)
    inv[order] = np.arange(order.size)
    counts = np.bincount(flat, minlength=E)
    off = np.zeros(E + 1, dtype=np.int64)
    off[1:] = np.cumsum(counts)
    return off.astype(np.int32), inv.reshape(T, k).astype(np.int32), order.astype(np.int32)


def permute_rows(x: np.ndarray, slot_of_row: np.ndarray, k: int) -> np.ndarray:
    """x_perm[r] = x[slot_of_row[r] // k]."""
    return x[slot_of_row // k]


def expert_ffn(x_perm: np.ndarray, expert_off: np.ndarray, layer: Dict[str, np.ndarray],
               limit: float, alpha: float = 1.702) -> Tuple[np.ndarray, np.ndarray]:
    """Per-expert gate/up projections, clipped SwiGLU and down projection.

    For the rows r of expert e's segment: g = x W_g[e]^T + b_g[e],
    u = x W_u[e]^T + b_u[e], h = swiglu(g, u), y = h W_d[e]^T + b_d[e].
    Returns h [R, F] and y_perm [R, D] in float64.
    """
    xp = decode(x_perm) if x_perm.dtype != np.float64 else x_perm
    E = expert_off.size - 1
    R = xp.shape[0]
    F = layer["b_gate"].shape[1]
    D = layer["b_down"].shape[1]
    h = np.zeros((R, F))
    y = np.zeros((R, D))
    for e in range(E):
        a, b = int(expert_off[e]), int(expert_off[e + 1])
        if a == b:
            continue
        xs = xp[a:b]
        g = xs @ expert_weights(layer, "gate", e).T + decode(layer["b_gate"][e])
        u = xs @ expert_weights(layer, "up", e).T + decode(layer["b_up"][e])
        he = clipped_swiglu(g, u, limit, alpha)
        h[a:b] = he
        y[a:b] = he @ expert_weights(layer, "down", e).T + decode(layer["b_down"][e])
    return h, y


def combine(y_perm: np.ndarray, row_of_slot: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y[t] = sum_j w[t, j] * y_perm[row_of_slot[t, j]]."""
    T, k = row_of_slot.shape
    out = np.zeros((T, y_perm.shape[1]))
    for j in range(k):
        out += w[:, j:j + 1] * y_perm[row_of_slot[:, j]]
    return out


def layer_forward(layer: Dict[str, np.ndarray], k: int, limit: float, alpha: float = 1.702) -> Dict[str, np.ndarray]:
    """The whole layer: router -> top-k/softmax -> dispatch -> experts -> combine."""
    E = layer["w_router"].shape[0]
    logits = router_logits(layer["x"], layer["w_router"], layer["b_router"])
    ids, w = topk_softmax(logits, k)
    off, row_of_slot, slot_of_row = dispatch(ids, E)
    x_perm = permute_rows(decode(layer["x"]), slot_of_row, k)
    h, y_perm = expert_ffn(x_perm, off, layer, limit, alpha)
    y = combine(y_perm, row_of_slot, w)
    return dict(logits=logits, ids=ids, w=w, expert_off=off, row_of_slot=row_of_slot,
                slot_of_row=slot_of_row, x_perm=x_perm, h=h, y_perm=y_perm, y=y)


def layer_tokens(layer: Dict[str, np.ndarray], tokens: np.ndarray, k: int, limit: float,
                 alpha: float = 1.702) -> Dict[str, np.ndarray]:
    """The layer output for selected tokens only, one token at a time.

    Used where the whole layer is too large for the CPU: each token's output
    needs only its own row, the router and the k selected experts.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    x = decode(layer["x"][tokens])
    logits = x @ decode(layer["w_router"]).T + decode(layer["b_router"])[None, :]
    ids, w = topk_softmax(logits, k)
    D = layer["b_down"].shape[1]
    F = layer["b_gate"].shape[1]
    h = np.zeros((tokens.size, k, F))
    o = np.zeros((tokens.size, k, D))
    # each selected expert's weights are decoded once, for all the tokens that chose it
    for e in np.unique(ids):
        e = int(e)
        ii, jj = np.nonzero(ids == e)
        xs = x[ii]
        g = xs @ expert_weights(layer, "gate", e).T + decode(layer["b_gate"][e])
        u = xs @ expert_weights(layer, "up", e).T + decode(layer["b_up"][e])
        hh = clipped_swiglu(g, u, limit, alpha)
        h[ii, jj] = hh
        o[ii, jj] = hh @ expert_weights(layer, "down", e).T + decode(layer["b_down"][e])
    y = np.zeros((tokens.size, D))
    for j in range(k):
        y += w[:, j:j + 1] * o[:, j]
    return dict(logits=logits, ids=ids, w=w, h=h, y=y)
