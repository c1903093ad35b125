"""Pins for the GLM4-MoE-Lite variant oracle (``oracle.glm_moe``), without a GPU.

Source: "Ollama glm4_moe_lite.go" (MoEGate.Forward, SwitchMLP.Forward,
SharedExperts.Forward, MoE.Forward).  The numpy oracle is tied to things other
than itself: router cases worked by hand as exact fractions
(``tests/golden/glm_router_worked.txt``), the choice of experts by subset
enumeration, the scalar-loop layer of ``oracle.brute``, closed forms of SiLU,
invariants (normalised weights sum to the scaling factor, the correction bias
moves the choice and never the weights), the shared expert on its own, and
planted mistakes that each of these catches.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from conftest import golden_lines
from oracle import brute, glm_moe as G
import workloads as W

LN3 = math.log(3.0)


# --------------------------------------------------------------------------- #
# router
# --------------------------------------------------------------------------- #
def _router_golden():
    for line in golden_lines("glm_router_worked.txt"):
        m, corr, k, norm, scale, ids, w = line.split()
        yield ([int(v) * LN3 for v in m.split(",")],
               None if corr == "-" else [float(v) for v in corr.split(",")],
               int(k), bool(int(norm)), float(scale),
               [int(v) for v in ids.split(",")], [float(Fraction(v)) for v in w.split(",")])


def test_router_golden_oracle():
    n = 0
    for lg, corr, k, norm, scale, ids, w in _router_golden():
        got_ids, got_w, _, _ = G.route(np.array([lg]), k, None if corr is None else np.array(corr), norm, scale)
        assert got_ids[0].tolist() == ids
        np.testing.assert_allclose(got_w[0], w, rtol=1e-14)
        n += 1
    assert n == 7


def test_router_golden_brute():
    for lg, corr, k, norm, scale, ids, w in _router_golden():
        got_ids, got_w = brute.glm_route_bruteforce(lg, k, corr, norm, scale)
        assert got_ids == ids
        np.testing.assert_allclose(got_w, w, rtol=1e-14)


@pytest.mark.parametrize("E,k", [(2, 1), (4, 2), (5, 3), (8, 2), (8, 4), (6, 6), (7, 1)])
@pytest.mark.parametrize("norm", [True, False])
def test_router_vs_subset_enumeration(E, k, norm):
    rng = np.random.default_rng(E * 10 + k + 100 * norm)
    lg = rng.standard_normal((40, E)) * 2
    corr = rng.standard_normal(E) * 0.2
    # equal scores: logits 0 give the score 1/2 exactly, so ties between experts are exact
    lg[::5, : E // 2] = 0.0
    for c in (None, corr):
        ids, w, _, _ = G.route(lg, k, c, norm, 1.8)
        for t in range(lg.shape[0]):
            bids, bw = brute.glm_route_bruteforce(lg[t].tolist(), k, None if c is None else c.tolist(), norm, 1.8)
            assert ids[t].tolist() == bids
            np.testing.assert_allclose(w[t], bw, rtol=1e-13)


def test_router_invariants():
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((400, 32)) * 2
    corr = rng.standard_normal(32) * 0.3
    scale = 2.5
    ids, w, scores, chosen_by = G.route(lg, 4, corr, True, scale)
    # k distinct experts; normalised weights sum to the scaling factor
    assert all(len(set(r)) == 4 for r in ids.tolist())
    np.testing.assert_allclose(w.sum(axis=1), scale, rtol=1e-14)
    # the weights are the uncorrected scores of the chosen experts, renormalised
    s = 1.0 / (1.0 + np.exp(-np.take_along_axis(lg, ids, axis=1)))
    np.testing.assert_allclose(w, scale * s / s.sum(axis=1, keepdims=True), rtol=1e-14)
    # every chosen expert beats every other on the corrected score
    for t in range(lg.shape[0]):
        rest = np.setdiff1d(np.arange(32), ids[t])
        assert chosen_by[t, ids[t]].min() > chosen_by[t, rest].max()
    # without normalisation each weight is scale * sigmoid(logit), inside (0, scale)
    _, w2, _, _ = G.route(lg, 4, corr, False, scale)
    np.testing.assert_allclose(w2, scale * s, rtol=1e-14)
    assert np.all((w2 > 0) & (w2 < scale))


def test_correction_bias_moves_the_choice_only():
    """A large bias on one expert makes every token choose it, with the weight its own score earns."""
    rng = np.random.default_rng(4)
    lg = rng.standard_normal((200, 8))
    corr = np.zeros(8)
    corr[5] = 10.0
    ids, w, scores, _ = G.route(lg, 2, corr, False, 1.0)
    assert np.all(ids[:, 0] == 5)
    np.testing.assert_allclose(w[:, 0], scores[:, 5], rtol=1e-15)
    # the second choice is the best of the others, by the uncorrected score
    others = np.delete(np.arange(8), 5)
    assert np.all(ids[:, 1] == others[np.argmax(scores[:, others], axis=1)])


def test_k1_is_not_normalised():
    """With k = 1 the page skips the normalisation: the weight is scale * sigmoid(logit), not scale."""
    lg = np.array([[0.3, -1.2, 2.0]])
    ids, w, _, _ = G.route(lg, 1, None, True, 3.0)
    assert ids[0].tolist() == [2]
    assert w[0, 0] == pytest.approx(3.0 / (1.0 + math.exp(-2.0)), rel=1e-15)


# --------------------------------------------------------------------------- #
# SiLU
# --------------------------------------------------------------------------- #
def test_silu_closed_forms():
    # sigmoid(m ln 3) = 3^m / (1 + 3^m)
    z = np.array([0.0, LN3, -LN3, 2 * LN3])
    np.testing.assert_allclose(G.silu(z), [0.0, 0.75 * LN3, -0.25 * LN3, 0.9 * 2 * LN3], rtol=1e-15, atol=0)
    # large arguments: SiLU(z) -> z, SiLU(-z) -> -z e^-z
    np.testing.assert_allclose(G.silu(np.array([40.0])), [40.0], rtol=1e-15)
    np.testing.assert_allclose(G.silu(np.array([-40.0])), [-40.0 * math.exp(-40.0)], rtol=1e-12)
    assert G.silu(np.array([-1000.0]))[0] == 0.0
    for v in (-3.0, -0.5, 0.25, 1.5, 6.0):
        assert brute.silu(v) == pytest.approx(float(G.silu(np.array([v]))[0]), rel=1e-15)


# --------------------------------------------------------------------------- #
# the whole variant layer
# --------------------------------------------------------------------------- #
def _scores_fn(spec):
    def f(layer):
        lg = G.gate_logits(layer["x"], layer["w_router"], layer.get("b_router"))
        return G.route(lg, spec.k, layer.get("e_score_correction_bias"))[3]
    return f


def _layer(spec, seed=0):
    return W.make_glm_layer(spec, seed=seed, scores_fn=_scores_fn(spec))


TINY = [W.glm_tiny_spec(T=7, D=16, E=6, k=2, F=8, F_shared=8, dtype="f32", expert_w_std=0.3, router_w_std=0.4),
        W.glm_tiny_spec(T=5, D=32, E=4, k=3, F=16, F_shared=0, dtype="bf16", expert_w_std=0.3, router_w_std=0.4,
                        norm_topk_prob=False, routed_scaling_factor=1.0, cfg_id=311),
        W.glm_tiny_spec(T=6, D=16, E=5, k=1, F=16, F_shared=32, dtype="bf16", expert_w_std=0.3, router_w_std=0.4,
                        correction_b_std=None, cfg_id=312),
        W.glm_tiny_spec(T=4, D=16, E=3, k=3, F=8, F_shared=8, dtype="f32", expert_w_std=0.3, router_w_std=0.4,
                        cfg_id=313)]


@pytest.mark.parametrize("spec", TINY, ids=lambda s: s.name)
def test_layer_vs_scalar_loops_tiny(spec):
    layer = _layer(spec)
    got = G.layer_forward(layer, spec.k, spec.norm_topk_prob, spec.routed_scaling_factor)
    for t in range(spec.T):
        want = brute.glm_layer_token(layer, t, spec.k, spec.norm_topk_prob, spec.routed_scaling_factor)
        assert got["ids"][t].tolist() == want["ids"]
        np.testing.assert_allclose(got["w"][t], want["w"], rtol=1e-13)
        np.testing.assert_allclose(got["y"][t], want["y"], rtol=1e-11, atol=1e-12 * np.max(np.abs(want["y"])))


def test_shared_expert_alone():
    """With every routed down projection zero the layer is the shared expert alone."""
    spec = TINY[0]
    layer = _layer(spec)
    layer["w_down"] = np.zeros_like(layer["w_down"])
    got = G.layer_forward(layer, spec.k, spec.norm_topk_prob, spec.routed_scaling_factor)
    for t in range(spec.T):
        x = [float(v) for v in layer["x"][t]]
        want = brute.silu_mlp_row(x, layer["ws_gate"].astype(float).tolist(), layer["ws_up"].astype(float).tolist(),
                                  layer["ws_down"].astype(float).tolist())
        np.testing.assert_allclose(got["y"][t], want, rtol=1e-12, atol=1e-15)
    assert np.all(got["y_routed"] == 0.0)


def test_dispatch_is_the_gptoss_permutation():
    """SwitchMLP.Forward sorts the flattened expert ids as the GPT-OSS layer does:
    rows of one expert in increasing token order, offsets counting each expert's rows."""
    spec = TINY[0]
    layer = _layer(spec)
    got = G.layer_forward(layer, spec.k, spec.norm_topk_prob, spec.routed_scaling_factor)
    off, ros, sor = brute.dispatch_counting(got["ids"].tolist(), spec.E)
    assert got["expert_off"].tolist() == off
    assert got["row_of_slot"].tolist() == ros
    assert got["slot_of_row"].tolist() == sor


def test_pins_catch_planted_mistakes():
    """Plausible mistakes in the variant, each written out as a numpy variant of the layer,
    all disagree with the scalar-loop layer where the oracle agrees to 1e-12: weights from
    the corrected scores, a softmax instead of the sigmoid scores, normalising at k = 1,
    choosing by the uncorrected scores, a dropped shared expert, a dropped scaling factor,
    and the GPT-OSS clipped activation in place of SiLU."""
    specs = [W.glm_tiny_spec(T=8, D=12, E=6, k=2, F=12, F_shared=12, dtype="f32", expert_w_std=0.5,
                             router_w_std=0.6, correction_b_std=0.3, cfg_id=314),
             W.glm_tiny_spec(T=8, D=12, E=6, k=1, F=12, F_shared=12, dtype="f32", expert_w_std=0.5,
                             router_w_std=0.6, correction_b_std=0.3, cfg_id=315)]
    caught = set()
    for spec in specs:
        layer = _layer(spec)
        x = layer["x"].astype(np.float64)
        lg = x @ layer["w_router"].astype(np.float64).T
        cb = layer["e_score_correction_bias"].astype(np.float64)
        Wg, Wu, Wd = (layer[f"w_{n}"].astype(np.float64) for n in ("gate", "up", "down"))
        Sg, Su, Sd = (layer[f"ws_{n}"].astype(np.float64) for n in ("gate", "up", "down"))
        k, scale = spec.k, spec.routed_scaling_factor

        def variant(weights="score", choose="corrected", norm_k1=False, shared=True, scaled=True, act="silu"):
            ys = np.zeros((spec.T, spec.D))
            for t in range(spec.T):
                s = 1.0 / (1.0 + np.exp(-lg[t]))
                by = s + cb if choose == "corrected" else s
                ids = np.argsort(-by, kind="stable")[:k]
                if weights == "score":
                    w = s[ids]
                elif weights == "corrected":
                    w = by[ids]
                else:
                    e = np.exp(lg[t, ids] - lg[t, ids].max())
                    w = e / e.sum()
                if (k > 1 or norm_k1) and weights != "softmax":
                    w = w / w.sum()
                if scaled:
                    w = w * scale
                for j, ex in enumerate(ids):
                    g, u = Wg[ex] @ x[t], Wu[ex] @ x[t]
                    if act == "silu":
                        h = g / (1.0 + np.exp(-g)) * u
                    else:
                        gc, uc = np.clip(g, 0.0, 7.0), np.clip(u, -7.0, 7.0)
                        h = gc / (1.0 + np.exp(-1.702 * gc)) * uc
                    ys[t] += w[j] * (Wd[ex] @ h)
                if shared:
                    g, u = Sg @ x[t], Su @ x[t]
                    ys[t] += Sd @ (g / (1.0 + np.exp(-g)) * u)
            return ys

        want = np.array([brute.glm_layer_token(layer, t, k, spec.norm_topk_prob, scale)["y"] for t in range(spec.T)])
        np.testing.assert_allclose(G.layer_forward(layer, k, spec.norm_topk_prob, scale)["y"], want,
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(variant(), want, rtol=1e-12, atol=1e-12)
        kws = [dict(weights="corrected"), dict(weights="softmax"), dict(choose="uncorrected"), dict(shared=False),
               dict(scaled=False), dict(act="clipped")]
        if k == 1:
            kws.append(dict(norm_k1=True))
        for kw in kws:
            if not np.allclose(variant(**kw), want, rtol=1e-6, atol=1e-9):
                caught.add(tuple(sorted(kw.items())))
    # every planted mistake is caught by at least one of the two layers
    assert len(caught) == 7, caught


# --------------------------------------------------------------------------- #
# input recipe
# --------------------------------------------------------------------------- #
def test_recipe_near_tie_gap_and_optional_parts():
    spec = W.glm_tiny_spec(T=300, D=32, E=16, k=4, F=16, F_shared=0, dtype="bf16", router_w_std=0.3,
                           correction_b_std=0.05, cfg_id=316)
    layer = _layer(spec)
    by = _scores_fn(spec)(layer)
    srt = -np.sort(-by, axis=1)
    assert np.all(srt[:, spec.k - 1] - srt[:, spec.k] >= 1e-3)
    assert "ws_gate" not in layer and "b_gate" not in layer
    nobias = W.glm_tiny_spec(T=4, D=16, E=4, k=2, F=16, F_shared=16, correction_b_std=None, cfg_id=317)
    layer2 = W.make_glm_layer(nobias)
    assert "e_score_correction_bias" not in layer2 and layer2["ws_down"].shape == (16, 16)
