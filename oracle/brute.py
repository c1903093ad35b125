"""O0 oracle: scalar-loop brute force for tiny inputs -- TEST INFRASTRUCTURE ONLY.

Plain Python floats (IEEE double) and explicit loops, written independently of
``moe_oracle`` so that each pins the other.  Same sources and readings as
``moe_oracle`` (GPT-OSS SwiGLU clip and alpha from "Ollama Imagegen GPT OSS",
router/expert parameters from the MaxText GPT-OSS weight map, argsort
dispatch and weighted combine from "Ollama glm4_moe_lite.go").

Top-k here is found by enumerating every k-subset of experts, not by sorting;
the dispatch permutation by counting, not by a library sort.

The last section does the same for the GLM4-MoE-Lite variant of the layer
(sigmoid router with a selection-only correction bias, SiLU experts without
biases, a shared expert), pinning ``glm_moe``.
"""
from __future__ import annotations

import itertools
import math
import struct
from typing import Dict, List, Optional, Sequence, Tuple


def bf16_value(bits: int) -> float:
    """Value of one bf16 bit pattern (the top half of an IEEE single)."""
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def value(a) -> float:
    """Scalar input value: numpy uint16 -> bf16, anything else -> float()."""
    if getattr(a, "dtype", None) is not None and str(a.dtype) == "uint16":
        return bf16_value(int(a))
    return float(a)


def e2m1(code: int) -> float:
    """4-bit E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa."""
    s = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        return s * (m / 2.0)
    return s * (2.0 ** (e - 1)) * (1.0 + m / 2.0)


def mxfp4_row(qrow, srow) -> List[float]:
    """One dequantised weight row from packed bytes and E8M0 scale bytes."""
    out = []
    for i in range(len(qrow)):
        byte = int(qrow[i])
        for nib in (byte & 0xF, byte >> 4):
            j = len(out)
            out.append(e2m1(nib) * 2.0 ** (int(srow[j // 32]) - 127))
    return out


def weight_row(layer, name: str, e: int, n: int) -> List[float]:
    w = layer[f"w_{name}"]
    if str(w.dtype) == "uint8":
        return mxfp4_row(w[e, n], layer[f"s_{name}"][e, n])
    return [value(v) for v in w[e, n]]


def sigmoid(z: float) -> float:
    return 1.0 / (1.0 + math.exp(-z))


def swiglu(g: float, u: float, limit: float, alpha: float = 1.702) -> float:
    gc = g
    if gc < 0.0:
        gc = 0.0
    if gc > limit:
        gc = limit
    uc = u
    if uc < -limit:
        uc = -limit
    if uc > limit:
        uc = limit
    return gc * sigmoid(alpha * gc) * uc


def dot(a: Sequence[float], b: Sequence[float]) -> float:
    s = 0.0
    for i in range(len(a)):
        s += a[i] * b[i]
    return s


def router_logits(layer, t: int) -> List[float]:
    x = [value(v) for v in layer["x"][t]]
    E = layer["w_router"].shape[0]
    return [dot(x, [value(v) for v in layer["w_router"][e]]) + value(layer["b_router"][e]) for e in range(E)]


def topk_bruteforce(logits: Sequence[float], k: int) -> Tuple[List[int], List[float]]:
    """The k-subset whose every member beats every non-member (ties: lower index wins).

    Enumerates all subsets; returns the ids by descending logit and the softmax
    over them.
    """
    E = len(logits)

    def beats(a: int, b: int) -> bool:
        return logits[a] > logits[b] or (logits[a] == logits[b] and a < b)

    found = None
    for sub in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in sub]
        if all(beats(a, b) for a in sub for b in rest):
            found = list(sub)
            break
    assert found is not None
    # order the chosen ids with a selection pass (no library sort)
    ordered: List[int] = []
    pool = list(found)
    while pool:
        best = pool[0]
        for c in pool[1:]:
            if beats(c, best):
                best = c
        ordered.append(best)
        pool.remove(best)
    m = max(logits[e] for e in ordered)
    ex = [math.exp(logits[e] - m) for e in ordered]
    z = sum(ex)
    return ordered, [v / z for v in ex]


def dispatch_counting(ids: Sequence[Sequence[int]], E: int) -> Tuple[List[int], List[List[int]], List[int]]:
    """Counting-sort dispatch: segment offsets, row of each (t, j), slot of each row."""
    T = len(ids)
    k = len(ids[0]) if T else 0
    cnt = [0] * E
    for t in range(T):
        for j in range(k):
            cnt[ids[t][j]] += 1
    off = [0] * (E + 1)
    for e in range(E):
        off[e + 1] = off[e] + cnt[e]
    fill = list(off[:E])
    row_of_slot = [[-1] * k for _ in range(T)]
    slot_of_row = [-1] * (T * k)
    for t in range(T):            # increasing token order -> stable by token
        for j in range(k):
            e = ids[t][j]
            r = fill[e]
            fill[e] += 1
            row_of_slot[t][j] = r
            slot_of_row[r] = t * k + j
    return off, row_of_slot, slot_of_row


def expert_output(layer, e: int, x: Sequence[float], limit: float, alpha: float = 1.702) -> Tuple[List[float], List[float]]:
    """(h, o) of expert e for one activation row, by scalar loops."""
    F = layer["b_gate"].shape[1]
    D = layer["b_down"].shape[1]
    h = []
    for f in range(F):
        g = dot(x, weight_row(layer, "gate", e, f)) + value(layer["b_gate"][e, f])
        u = dot(x, weight_row(layer, "up", e, f)) + value(layer["b_up"][e, f])
        h.append(swiglu(g, u, limit, alpha))
    o = []
    for d in range(D):
        o.append(dot(h, weight_row(layer, "down", e, d)) + value(layer["b_down"][e, d]))
    return h, o


def layer_token(layer, t: int, k: int, limit: float, alpha: float = 1.702) -> Dict[str, list]:
    """The whole layer for token t, by scalar loops."""
    lg = router_logits(layer, t)
    ids, w = topk_bruteforce(lg, k)
    x = [value(v) for v in layer["x"][t]]
    D = layer["b_down"].shape[1]
    y = [0.0] * D
    hs = []
    for j in range(k):
        h, o = expert_output(layer, ids[j], x, limit, alpha)
        hs.append(h)
        for d in range(D):
            y[d] += w[j] * o[d]
    return dict(logits=lg, ids=ids, w=w, h=hs, y=y)


# --------------------------------------------------------------------------- #
# GLM4-MoE-Lite variant ("Ollama glm4_moe_lite.go": MoEGate.Forward,
# SwitchMLP.Forward, SharedExperts.Forward, MoE.Forward), by scalar loops
# --------------------------------------------------------------------------- #
def silu(z: float) -> float:
    return z * sigmoid(z)


def glm_route_bruteforce(logits: Sequence[float], k: int, correction: Optional[Sequence[float]],
                         norm_topk_prob: bool, routed_scaling_factor: float) -> Tuple[List[int], List[float]]:
    """Experts chosen by enumerating k-subsets on the corrected sigmoid scores.

    The chosen subset is the one whose every member beats every non-member
    (larger corrected score, equal scores: lower index); the weights are the
    uncorrected scores of the chosen experts, normalised by their sum when
    k > 1 and ``norm_topk_prob``, then scaled.
    """
    E = len(logits)
    score = [sigmoid(v) for v in logits]
    sel = [score[e] + (correction[e] if correction is not None else 0.0) for e in range(E)]
    ids, _ = topk_bruteforce(sel, k)      # subset enumeration, ordered by a selection pass
    w = [score[e] for e in ids]
    if k > 1 and norm_topk_prob:
        z = 0.0
        for v in w:
            z += v
        w = [v / z for v in w]
    return ids, [v * routed_scaling_factor for v in w]


def silu_mlp_row(x: Sequence[float], wg_rows, wu_rows, wd_rows) -> List[float]:
    """o = W_d (SiLU(W_g x) * (W_u x)) for one activation row; weights given as row lists."""
    h = [silu(dot(x, wg_rows[f])) * dot(x, wu_rows[f]) for f in range(len(wg_rows))]
    return [dot(h, wd_rows[d]) for d in range(len(wd_rows))]


def glm_layer_token(layer, t: int, k: int, norm_topk_prob: bool, routed_scaling_factor: float) -> Dict[str, list]:
    """The GLM4-MoE-Lite layer for token t, by scalar loops."""
    x = [value(v) for v in layer["x"][t]]
    E = layer["w_router"].shape[0]
    lg = []
    for e in range(E):
        v = dot(x, [value(q) for q in layer["w_router"][e]])
        if layer.get("b_router") is not None:
            v += value(layer["b_router"][e])
        lg.append(v)
    corr = layer.get("e_score_correction_bias")
    corr = None if corr is None else [value(v) for v in corr]
    ids, w = glm_route_bruteforce(lg, k, corr, norm_topk_prob, routed_scaling_factor)
    D = layer["w_down"].shape[1]
    y = [0.0] * D
    for j in range(k):
        e = ids[j]
        o = silu_mlp_row(x, [[value(q) for q in r] for r in layer["w_gate"][e]],
                         [[value(q) for q in r] for r in layer["w_up"][e]],
                         [[value(q) for q in r] for r in layer["w_down"][e]])
        for d in range(D):
            y[d] += w[j] * o[d]
    if "ws_gate" in layer:
        o = silu_mlp_row(x, [[value(q) for q in r] for r in layer["ws_gate"]],
                         [[value(q) for q in r] for r in layer["ws_up"]],
                         [[value(q) for q in r] for r in layer["ws_down"]])
        for d in range(D):
            y[d] += o[d]
    return dict(logits=lg, ids=ids, w=w, y=y)


# --------------------------------------------------------------------------- #
# MXFP8 activations (the block-scaled numerics variant, pins ``mx_act``)
# --------------------------------------------------------------------------- #
def e4m3_table() -> List[Tuple[int, float]]:
    """(code, value) of every finite E4M3 code, built bit field by bit field."""
    out = []
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            continue                                   # NaN
        if e == 0:
            val = s * m * 2.0 ** -9
        else:
            val = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
        out.append((code, val))
    return out


def e4m3_nearest(v: float) -> float:
    """The finite E4M3 value nearest to v (ties: the code with an even mantissa), by search."""
    best, best_code = None, None
    for code, val in e4m3_table():
        if best is None or abs(val - v) < abs(best - v) or (
                abs(val - v) == abs(best - v) and (code & 1) == 0 and (best_code & 1) == 1):
            best, best_code = val, code
    return best + 0.0   # -0.0 -> 0.0


def mx8_exponent(amax: float) -> int:
    """Smallest X in [-127, 127] with amax <= 448 * 2^X (searching upwards)."""
    for X in range(-127, 128):
        if amax <= 448.0 * 2.0 ** X:
            return X
    return 127


def mx8_row(v: Sequence[float]) -> List[float]:
    """One row quantized to MXFP8 and dequantized, 32-element blocks."""
    out = []
    for b in range(0, len(v), 32):
        blk = list(v[b:b + 32])
        X = mx8_exponent(max(abs(t) for t in blk))
        out.extend(e4m3_nearest(t / 2.0 ** X) * 2.0 ** X for t in blk)
    return out


def layer_token_mx8(layer, t: int, k: int, limit: float, alpha: float = 1.702) -> Dict[str, list]:
    """One token through the layer with MXFP8 activations in both expert projections."""
    logits = router_logits(layer, t)
    ids, w = topk_bruteforce(logits, k)
    x = mx8_row([value(v) for v in layer["x"][t]])
    D = len(layer["b_down"][0])
    y = [0.0] * D
    for e, wt in zip(ids, w):
        F = len(layer["b_gate"][e])
        h = []
        for f in range(F):
            g = dot(x, weight_row(layer, "gate", e, f)) + value(layer["b_gate"][e][f])
            u = dot(x, weight_row(layer, "up", e, f)) + value(layer["b_up"][e][f])
            h.append(swiglu(g, u, limit, alpha))
        hq = mx8_row(h)
        for d in range(D):
            y[d] += wt * (dot(hq, weight_row(layer, "down", e, d)) + value(layer["b_down"][e][d]))
    return {"ids": ids, "w": w, "y": y}
