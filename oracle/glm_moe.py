"""O1 oracle for the GLM4-MoE-Lite variant of the MoE layer, numpy fp64.

TEST INFRASTRUCTURE ONLY -- see the package docstring.

This is the second router and expert form the pages show, on the same
dispatch and combine as the GPT-OSS layer.  Source: "Ollama glm4_moe_lite.go"
(the MLX Go model file):

  * ``MoEGate.Forward``: the gate linear gives logits; the scores are their
    logistic sigmoid.  An optional per-expert ``e_score_correction_bias`` is
    added to the scores for the *choice* of experts only: the k experts with
    the largest corrected scores are picked, and their weights are the
    uncorrected scores.  When k > 1 and ``norm_topk_prob`` is set, the k
    weights are divided by their sum; finally every weight is multiplied by
    ``routed_scaling_factor``.
  * ``SwitchMLP.Forward``: each chosen expert applies SiLU(x W_g^T) * (x W_u^T)
    and then W_d; no biases and no clipping.  Tokens reach their experts by
    the same sort of the flattened expert ids as in the GPT-OSS layer.
  * ``SharedExperts.Forward``: one dense SiLU-gated MLP applied to every token.
  * ``MoE.Forward``: y = sum_j w[t, j] * expert_{ids[t, j]}(x[t]) + shared(x[t]).
  * ``Config``: n_routed_experts, n_shared_experts, num_experts_per_tok,
    routed_scaling_factor, norm_topk_prob.

Readings where the page is silent (each is listed in the design notes):
  * the choice among equal corrected scores goes to the lower expert index, and
    ids are listed by descending corrected score (``Argpartition`` leaves both
    open);
  * the gate linear carries no bias unless the layer supplies ``b_router``;
  * SiLU(z) = z * sigmoid(z), the standard definition;
  * the shared expert is present when the layer holds ``ws_gate``/``ws_up``/
    ``ws_down`` (n_shared_experts experts of one dense MLP, as the page loads them).
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import numpy as np

from .moe_oracle import decode, dispatch


def sigmoid(z: np.ndarray) -> np.ndarray:
    """Logistic function 1 / (1 + e^-z), elementwise (e^-z overflowing to inf gives 0)."""
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-np.asarray(z, dtype=np.float64)))


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z)."""
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def gate_logits(x: np.ndarray, w_router: np.ndarray, b_router: Optional[np.ndarray] = None) -> np.ndarray:
    """l[t, e] = sum_d x[t, d] * Wr[e, d] (+ br[e] when the gate has a bias)."""
    lg = decode(x) @ decode(w_router).T
    if b_router is not None:
        lg = lg + decode(b_router)[None, :]
    return lg


def route(logits: np.ndarray, k: int, correction_bias: Optional[np.ndarray] = None,
          norm_topk_prob: bool = True, routed_scaling_factor: float = 1.0
          ) -> Tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """``MoEGate.Forward``: returns ids [T, k], weights [T, k], scores [T, E], corrected scores [T, E].

    scores = sigmoid(logits); choice by scores + correction_bias; weights are the
    uncorrected scores of the chosen experts, normalised to sum 1 when k > 1 and
    ``norm_topk_prob``, then times ``routed_scaling_factor``.
    """
    scores = sigmoid(logits)
    chosen_by = scores if correction_bias is None else scores + decode(correction_bias)[None, :]
    # a stable sort of the negated values: descending, equal values by lower index
    ids = np.argsort(-chosen_by, axis=1, kind="stable")[:, :k]
    w = np.take_along_axis(scores, ids, axis=1)
    if k > 1 and norm_topk_prob:
        w = w / w.sum(axis=1, keepdims=True)
    w = w * routed_scaling_factor
    return ids.astype(np.int32), w, scores, chosen_by


def silu_mlp(x: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray
             ) -> Tuple[np.ndarray, np.ndarray]:
    """h = SiLU(x W_g^T) * (x W_u^T), o = h W_d^T; weights already float64."""
    h = silu(x @ w_gate.T) * (x @ w_up.T)
    return h, h @ w_down.T


def shared_expert(layer: Dict[str, np.ndarray], x: np.ndarray) -> np.ndarray:
    """``SharedExperts.Forward`` on float64 rows x; zeros when the layer has no shared expert."""
    if "ws_gate" not in layer:
        return np.zeros((x.shape[0], layer["w_down"].shape[1]))
    return silu_mlp(x, decode(layer["ws_gate"]), decode(layer["ws_up"]), decode(layer["ws_down"]))[1]


def layer_forward(layer: Dict[str, np.ndarray], k: int, norm_topk_prob: bool = True,
                  routed_scaling_factor: float = 1.0) -> Dict[str, np.ndarray]:
    """The whole variant layer: gate -> sigmoid choice -> dispatch -> SiLU experts -> combine + shared."""
    E = layer["w_router"].shape[0]
    x = decode(layer["x"])
    logits = gate_logits(layer["x"], layer["w_router"], layer.get("b_router"))
    ids, w, scores, chosen_by = route(logits, k, layer.get("e_score_correction_bias"), norm_topk_prob,
                                      routed_scaling_factor)
    off, row_of_slot, slot_of_row = dispatch(ids, E)
    x_perm = x[slot_of_row // k]
    D = layer["w_down"].shape[1]
    F = layer["w_gate"].shape[1]
    h = np.zeros((x_perm.shape[0], F))
    y_perm = np.zeros((x_perm.shape[0], D))
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if a == b:
            continue
        h[a:b], y_perm[a:b] = silu_mlp(x_perm[a:b], decode(layer["w_gate"][e]), decode(layer["w_up"][e]),
                                       decode(layer["w_down"][e]))
    y_routed = np.zeros((x.shape[0], D))
    for j in range(k):
        y_routed += w[:, j:j + 1] * y_perm[row_of_slot[:, j]]
    y_shared = shared_expert(layer, x)
    return dict(logits=logits, scores=scores, chosen_by=chosen_by, ids=ids, w=w, expert_off=off,
                row_of_slot=row_of_slot, slot_of_row=slot_of_row, h=h, y_perm=y_perm, y_routed=y_routed,
                y_shared=y_shared, y=y_routed + y_shared)
