"""Pins for the CPU oracle: golden hand-worked values, brute force, invariants.

These run without a GPU.  They tie ``oracle.moe_oracle`` (numpy, fp64) to
things other than itself: hand-worked values of the clipped SwiGLU and of the
top-k softmax, the OCP E2M1 / E8M0 code tables, subset-enumeration top-k,
counting-sort dispatch, a scalar-loop layer, the E = k = 1 dense reduction,
and invariants (weights sum to 1, the permutation is a bijection, token
permutation equivariance, unused experts contribute nothing).
"""
import math

import numpy as np
import pytest

from conftest import golden_lines
from oracle import brute, moe_oracle as O
import workloads as W


# --------------------------------------------------------------------------- #
# clipped SwiGLU
# --------------------------------------------------------------------------- #
def _swiglu_golden():
    rows = []
    for line in golden_lines("swiglu_worked.txt"):
        g, u, h = (float(v) for v in line.split())
        rows.append((g, u, h))
    return rows


def test_swiglu_golden_oracle():
    rows = _swiglu_golden()
    g = np.array([r[0] for r in rows])
    u = np.array([r[1] for r in rows])
    want = np.array([r[2] for r in rows])
    got = O.clipped_swiglu(g, u, 7.0, 1.702)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-14)


def test_swiglu_golden_brute():
    for g, u, h in _swiglu_golden():
        assert brute.swiglu(g, u, 7.0, 1.702) == pytest.approx(h, rel=1e-11, abs=1e-14)


def test_swiglu_gate_nonpositive_is_zero():
    g = -np.abs(np.random.default_rng(0).standard_normal(1000)) * 10
    u = np.random.default_rng(1).standard_normal(1000) * 10
    assert np.all(O.clipped_swiglu(g, u, 7.0) == 0.0)


def test_swiglu_saturates_at_limit():
    # beyond the limit both clips are active: h = L * sigmoid(alpha L) * (+-L)
    L = 7.0
    g = np.array([7.0, 8.0, 1e6])
    u = np.array([-7.5, 7.0, 1e9])
    want = L * (1 / (1 + math.exp(-1.702 * L))) * np.array([-L, L, L])
    np.testing.assert_allclose(O.clipped_swiglu(g, u, L), want, rtol=1e-15)


# --------------------------------------------------------------------------- #
# top-k + softmax
# --------------------------------------------------------------------------- #
def _topk_golden():
    for line in golden_lines("topk_worked.txt"):
        lg, k, ids, w = (p.strip() for p in line.split("|"))
        yield ([float(v) for v in lg.split()], int(k), [int(v) for v in ids.split()], [float(v) for v in w.split()])


def test_topk_golden_oracle():
    for lg, k, ids, w in _topk_golden():
        got_ids, got_w = O.topk_softmax(np.array([lg]), k)
        assert got_ids[0].tolist() == ids
        np.testing.assert_allclose(got_w[0], w, rtol=1e-14)


def test_topk_golden_brute():
    for lg, k, ids, w in _topk_golden():
        got_ids, got_w = brute.topk_bruteforce(lg, k)
        assert got_ids == ids
        np.testing.assert_allclose(got_w, w, rtol=1e-14)


@pytest.mark.parametrize("E,k", [(2, 1), (4, 2), (5, 3), (8, 2), (8, 4), (6, 6), (7, 1)])
def test_topk_vs_subset_enumeration(E, k):
    rng = np.random.default_rng(E * 10 + k)
    # integer-valued logits force many exact ties (exercises the tie-break)
    lg = np.concatenate([rng.standard_normal((40, E)), rng.integers(-2, 3, size=(40, E)).astype(float)])
    ids, w = O.topk_softmax(lg, k)
    for t in range(lg.shape[0]):
        bids, bw = brute.topk_bruteforce(lg[t].tolist(), k)
        assert ids[t].tolist() == bids
        np.testing.assert_allclose(w[t], bw, rtol=1e-13)


def test_topk_invariants():
    rng = np.random.default_rng(7)
    lg = rng.standard_normal((500, 32)) * 3
    ids, w = O.topk_softmax(lg, 4)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-12)
    assert all(len(set(r)) == 4 for r in ids.tolist())
    assert np.all(np.diff(np.take_along_axis(lg, ids.astype(np.int64), 1), axis=1) <= 0)
    assert np.all(w[:, :-1] >= w[:, 1:])
    # k = E selects every expert
    ids_all, w_all = O.topk_softmax(lg[:, :8], 8)
    assert all(sorted(r) == list(range(8)) for r in ids_all.tolist())
    # a uniform shift of the logits changes nothing
    ids2, w2 = O.topk_softmax(lg + 123.0, 4)
    assert np.array_equal(ids, ids2)
    np.testing.assert_allclose(w, w2, rtol=1e-9)


# --------------------------------------------------------------------------- #
# dispatch
# --------------------------------------------------------------------------- #
def _random_ids(rng, T, E, k):
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32) if T else np.zeros((0, k), np.int32)


@pytest.mark.parametrize("T,E,k", [(0, 4, 2), (1, 1, 1), (1, 8, 4), (13, 5, 2), (64, 8, 2), (200, 32, 4), (77, 128, 4)])
def test_dispatch_vs_counting_sort(T, E, k):
    rng = np.random.default_rng(T + E + k)
    ids = _random_ids(rng, T, E, k)
    off, ros, sor = O.dispatch(ids, E)
    boff, bros, bsor = brute.dispatch_counting(ids.tolist(), E)
    assert off.tolist() == boff
    assert ros.tolist() == (bros if T else [])
    assert sor.tolist() == bsor


@pytest.mark.parametrize("T,E,k", [(1, 8, 4), (100, 8, 2), (500, 32, 4), (300, 128, 4)])
def test_dispatch_invariants(T, E, k):
    rng = np.random.default_rng(99)
    ids = _random_ids(rng, T, E, k)
    off, ros, sor = O.dispatch(ids, E)
    R = T * k
    assert off[0] == 0 and off[E] == R and np.all(np.diff(off) >= 0)
    assert np.array_equal(np.sort(ros.reshape(-1)), np.arange(R))            # bijection
    assert np.array_equal(sor[ros.reshape(-1)], np.arange(R))                # inverse
    for e in range(E):
        seg = sor[off[e]:off[e + 1]]
        assert np.all(ids.reshape(-1)[seg] == e)                               # rows of e hold e
        assert np.all(np.diff(seg // k) > 0)                                   # by increasing token
    # the rows are what an argsort of the flattened ids gives (stable), tokens = order // k
    order = np.argsort(ids.reshape(-1), kind="stable")
    assert np.array_equal(sor, order)
    x = rng.standard_normal((T, 3))
    np.testing.assert_array_equal(O.permute_rows(x, sor, k), x[order // k])


# --------------------------------------------------------------------------- #
# MXFP4
# --------------------------------------------------------------------------- #
def _mx_golden():
    sec, e2m1, e8m0 = None, {}, {}
    for line in golden_lines("e2m1_codes.txt"):
        if line in ("E2M1", "E8M0"):
            sec = line
            continue
        a, b = line.split()
        (e2m1 if sec == "E2M1" else e8m0)[int(a)] = float(b)
    return e2m1, e8m0


def test_e2m1_table():
    e2m1, _ = _mx_golden()
    codes = np.arange(16)
    np.testing.assert_array_equal(O.e2m1_value(codes), [e2m1[c] for c in range(16)])
    assert [brute.e2m1(c) for c in range(16)] == [e2m1[c] for c in range(16)]
    assert math.copysign(1.0, O.e2m1_value(np.array([8]))[0]) == -1.0


def test_e8m0_scales_and_nibble_order():
    e2m1, e8m0 = _mx_golden()
    for sbyte, scale in e8m0.items():
        # row of 32 elements: byte i packs element 2i (low nibble) and 2i+1 (high nibble)
        q = np.array([[(c & 0xF) | (((c + 1) & 0xF) << 4) for c in range(0, 32, 2)]], dtype=np.uint8)
        s = np.array([[sbyte]], dtype=np.uint8)
        got = O.mxfp4_dequant(q, s)[0]
        want = []
        for c in range(0, 32, 2):
            want += [e2m1[c & 0xF] * scale, e2m1[(c + 1) & 0xF] * scale]
        np.testing.assert_array_equal(got, want)
    # a single byte 0x21: element 0 = code 1 (0.5), element 1 = code 2 (1.0)
    q = np.zeros((1, 16), np.uint8)
    q[0, 0] = 0x21
    got = O.mxfp4_dequant(q, np.array([[127]], np.uint8))[0]
    assert got[0] == 0.5 and got[1] == 1.0 and np.all(got[2:] == 0)


def test_mxfp4_dequant_vs_brute():
    rng = np.random.default_rng(3)
    q = rng.integers(0, 256, size=(5, 64), dtype=np.uint8)
    s = (127 + rng.integers(-8, 1, size=(5, 4))).astype(np.uint8)
    got = O.mxfp4_dequant(q, s)
    for n in range(5):
        assert got[n].tolist() == brute.mxfp4_row(q[n], s[n])
    # every dequantised weight is exactly representable in bf16
    bits = W.f32_to_bf16_bits(got.astype(np.float32))
    np.testing.assert_array_equal(W.bf16_bits_to_f32(bits).astype(np.float64), got)


# --------------------------------------------------------------------------- #
# the whole layer
# --------------------------------------------------------------------------- #
def _logits_fn(layer):
    return O.router_logits(layer["x"], layer["w_router"], layer["b_router"])


def _check_layer_vs_brute(spec, layer, tokens, tol=1e-9):
    ref = O.layer_forward(layer, spec.k, spec.limit, spec.alpha)
    for t in tokens:
        b = brute.layer_token(layer, int(t), spec.k, spec.limit, spec.alpha)
        np.testing.assert_allclose(ref["logits"][t], b["logits"], rtol=1e-12, atol=1e-12)
        assert ref["ids"][t].tolist() == b["ids"]
        np.testing.assert_allclose(ref["w"][t], b["w"], rtol=1e-12)
        for j in range(spec.k):
            r = ref["row_of_slot"][t, j]
            np.testing.assert_allclose(ref["h"][r], b["h"][j], rtol=tol, atol=tol)
        np.testing.assert_allclose(ref["y"][t], b["y"], rtol=tol, atol=tol)
    return ref


@pytest.mark.parametrize("dtype,wfmt,D,F", [("f32", "dense", 16, 24), ("bf16", "dense", 16, 40), ("bf16", "mxfp4", 32, 64)])
def test_layer_vs_scalar_loops_tiny(dtype, wfmt, D, F):
    spec = W.tiny_spec(T=7, D=D, E=5, k=2, F=F, dtype=dtype, wfmt=wfmt, expert_w_std=0.3, router_w_std=0.5)
    layer = W.make_layer(spec, seed=1, logits_fn=_logits_fn)
    _check_layer_vs_brute(spec, layer, range(spec.T))


def test_layer_vs_scalar_loops_tiny_fp32_config():
    spec = W.TINY_FP32
    layer = W.make_layer(spec, seed=0, logits_fn=_logits_fn)
    _check_layer_vs_brute(spec, layer, [0, 31, 63])


def test_dense_reduction_E1_k1():
    """E = k = 1: the layer is one dense clipped-SwiGLU MLP with routing weight exactly 1."""
    spec = W.tiny_spec(T=5, D=12, E=1, k=1, F=20, dtype="f32", expert_w_std=0.5)
    layer = W.make_layer(spec, seed=4)
    ref = O.layer_forward(layer, 1, spec.limit)
    assert np.all(ref["w"] == 1.0) and np.all(ref["ids"] == 0)
    for t in range(spec.T):
        x = [float(v) for v in layer["x"][t]]
        h, o = brute.expert_output(layer, 0, x, spec.limit)
        np.testing.assert_allclose(ref["y"][t], o, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(ref["h"][t], h, rtol=1e-12, atol=1e-12)


def test_layer_tokens_matches_full_layer():
    spec = W.TINY_FP32
    layer = W.make_layer(spec, seed=0, logits_fn=_logits_fn)
    full = O.layer_forward(layer, spec.k, spec.limit)
    toks = np.array([3, 0, 63, 17])
    part = O.layer_tokens(layer, toks, spec.k, spec.limit)
    np.testing.assert_array_equal(part["ids"], full["ids"][toks])
    np.testing.assert_allclose(part["y"], full["y"][toks], rtol=1e-12, atol=1e-12)


def test_token_permutation_equivariance_and_duplicates():
    spec = W.tiny_spec(T=24, D=32, E=6, k=3, F=48, dtype="bf16")
    layer = W.make_layer(spec, seed=2, logits_fn=_logits_fn)
    layer["x"][5] = layer["x"][11]                       # a duplicate token
    ref = O.layer_forward(layer, spec.k, spec.limit)
    np.testing.assert_array_equal(ref["y"][5], ref["y"][11])
    perm = np.random.default_rng(0).permutation(spec.T)
    l2 = dict(layer)
    l2["x"] = layer["x"][perm]
    ref2 = O.layer_forward(l2, spec.k, spec.limit)
    np.testing.assert_allclose(ref2["y"], ref["y"][perm], rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(ref2["ids"], ref["ids"][perm])


def test_unrouted_expert_contributes_nothing():
    spec = W.tiny_spec(T=16, D=16, E=4, k=2, F=16, dtype="f32")
    layer = W.make_layer(spec, seed=5)
    layer["b_router"] = layer["b_router"].copy()
    layer["b_router"][2] = -1e4                           # expert 2 is never selected
    ref = O.layer_forward(layer, spec.k, spec.limit)
    assert ref["expert_off"][2] == ref["expert_off"][3]
    for name in ("gate", "up", "down"):
        layer[f"w_{name}"] = layer[f"w_{name}"].copy()
        layer[f"w_{name}"][2] = 1e6
    ref2 = O.layer_forward(layer, spec.k, spec.limit)
    np.testing.assert_array_equal(ref2["y"], ref["y"])


def test_swiglu_is_odd_in_up_and_flat_beyond_the_limits():
    """h(g, -u) = -h(g, u) (the up clip is symmetric), h is constant in u beyond +/-L and
    in g beyond L, and scales linearly in u inside the clip range."""
    rng = np.random.default_rng(10)
    g = rng.uniform(-3, 10, 200)
    u = rng.uniform(-10, 10, 200)
    L = 7.0
    np.testing.assert_array_equal(O.clipped_swiglu(g, -u, L), -O.clipped_swiglu(g, u, L))
    np.testing.assert_array_equal(O.clipped_swiglu(g, np.full_like(u, 9.0), L), O.clipped_swiglu(g, np.full_like(u, L), L))
    np.testing.assert_array_equal(O.clipped_swiglu(np.full_like(g, 12.0), u, L), O.clipped_swiglu(np.full_like(g, L), u, L))
    inside = np.abs(u) < L / 2
    np.testing.assert_allclose(O.clipped_swiglu(g[inside], 2 * u[inside], L), 2 * O.clipped_swiglu(g[inside], u[inside], L),
                               rtol=1e-15, atol=0)


def test_mxfp4_scale_step_doubles_every_weight():
    """Raising every E8M0 byte by one doubles every dequantised weight exactly."""
    rng = np.random.default_rng(11)
    q = rng.integers(0, 256, size=(3, 5, 32), dtype=np.uint8)        # [E, N, K/2] = 64 codes per row
    s = rng.integers(100, 140, size=(3, 5, 2), dtype=np.uint8)       # two 32-element blocks per row
    np.testing.assert_array_equal(O.mxfp4_dequant(q, s + 1), 2.0 * O.mxfp4_dequant(q, s))


def test_output_is_linear_in_the_down_projection():
    """Doubling W_down and b_down doubles y exactly (routing and h are untouched)."""
    spec = W.tiny_spec(T=10, D=16, E=4, k=2, F=24, dtype="f32", expert_w_std=0.3)
    layer = W.make_layer(spec, seed=12)
    ref = O.layer_forward(layer, spec.k, spec.limit)
    l2 = dict(layer)
    l2["w_down"] = 2.0 * layer["w_down"]
    l2["b_down"] = 2.0 * layer["b_down"]
    ref2 = O.layer_forward(l2, spec.k, spec.limit)
    np.testing.assert_array_equal(ref2["ids"], ref["ids"])
    np.testing.assert_array_equal(ref2["h"], ref["h"])
    np.testing.assert_allclose(ref2["y"], 2.0 * ref["y"], rtol=1e-14, atol=0)


def test_identical_experts_give_the_dense_mlp():
    """If every expert has the same weights and biases, routing cannot matter: the softmax
    weights sum to 1, so every token's output is that one dense MLP's output (a scalar
    triple loop), whatever the router picks."""
    spec = W.tiny_spec(T=11, D=16, E=5, k=3, F=24, dtype="f32", expert_w_std=0.3)
    layer = W.make_layer(spec, seed=8)
    for name in ("w_gate", "w_up", "w_down", "b_gate", "b_up", "b_down"):
        layer[name] = np.repeat(layer[name][:1], spec.E, axis=0)
    ref = O.layer_forward(layer, spec.k, spec.limit)
    for t in range(spec.T):
        _, o = brute.expert_output(layer, 0, [float(v) for v in layer["x"][t]], spec.limit)
        np.testing.assert_allclose(ref["y"][t], o, rtol=1e-12, atol=1e-12)


def test_router_logits_with_identity_weights():
    """Wr = I (E = D): the logits are the activations plus the router bias."""
    D = 6
    rng = np.random.default_rng(9)
    x = rng.standard_normal((7, D))
    b = rng.standard_normal(D)
    lg = O.router_logits(x, np.eye(D), b)
    np.testing.assert_allclose(lg, x + b, rtol=0, atol=1e-15)


def test_down_bias_is_weighted():
    """With zero expert weights the output is sum_j w_j * b_down[e_j]."""
    spec = W.tiny_spec(T=9, D=8, E=4, k=2, F=8, dtype="f32")
    layer = W.make_layer(spec, seed=6)
    for name in ("gate", "up", "down"):
        layer[f"w_{name}"] = np.zeros_like(layer[f"w_{name}"])
    ref = O.layer_forward(layer, spec.k, spec.limit)
    want = np.zeros((spec.T, spec.D))
    for t in range(spec.T):
        for j in range(spec.k):
            want[t] += ref["w"][t, j] * layer["b_down"][ref["ids"][t, j]].astype(np.float64)
    np.testing.assert_allclose(ref["y"], want, rtol=1e-14, atol=1e-15)


# --------------------------------------------------------------------------- #
# planted mistakes: a wrong oracle must fail the pins above
# --------------------------------------------------------------------------- #
def test_pins_catch_planted_swiglu_mistakes(monkeypatch):
    rows = _swiglu_golden()
    g = np.array([r[0] for r in rows])
    u = np.array([r[1] for r in rows])
    want = np.array([r[2] for r in rows])
    wrong = [
        lambda g, u, L, a: np.clip(g, -L, L) / (1 + np.exp(-a * np.clip(g, -L, L))) * np.clip(u, -L, L),  # gate lower clip -L
        lambda g, u, L, a: np.clip(g, 0, L) / (1 + np.exp(-np.clip(g, 0, L))) * np.clip(u, -L, L),        # alpha dropped
        lambda g, u, L, a: np.clip(g, 0, L) / (1 + np.exp(-a * np.clip(g, 0, L))) * (np.clip(u, -L, L) + 1),  # u + 1
        lambda g, u, L, a: np.clip(g, 0, L) / (1 + np.exp(-a * np.clip(g, 0, L))) * u,                   # up not clipped
    ]
    for f in wrong:
        assert not np.allclose(f(g, u, 7.0, 1.702), want, rtol=1e-6)


def test_pins_catch_planted_dispatch_mistake():
    rng = np.random.default_rng(1)
    ids = _random_ids(rng, 50, 8, 2)
    unstable = np.argsort(ids.reshape(-1), kind="quicksort")[::-1]   # not stable by token
    _, _, sor = brute.dispatch_counting(ids.tolist(), 8)
    assert unstable.tolist() != sor


def test_pins_catch_planted_layer_mistakes():
    """Plausible mistakes in the layer arithmetic, each written out as a variant of the
    layer (numpy, fp64), all disagree with the scalar-loop layer on a tiny case where the
    oracle itself agrees to 1e-12: softmax over all experts, selection of the smallest
    logits, a dropped down bias, an unweighted down bias, a transposed gate weight, gate
    and up swapped, and an unnormalised routing weight."""
    spec = W.tiny_spec(T=6, D=12, E=5, k=2, F=12, dtype="f32", expert_w_std=0.4, router_w_std=0.5)
    layer = W.make_layer(spec, seed=13, logits_fn=_logits_fn)
    L, a = spec.limit, 1.702
    x = O.decode(layer["x"])
    lg = O.router_logits(layer["x"], layer["w_router"], layer["b_router"])
    Wg, Wu, Wd = (O.expert_weights(layer, n) for n in ("gate", "up", "down"))
    bg, bu, bd = (O.decode(layer[f"b_{n}"]) for n in ("gate", "up", "down"))

    def layer_y(select="top", weights="softmax_k", bias="weighted", gate_t=False, swap=False):
        ys = np.zeros((spec.T, spec.D))
        for t in range(spec.T):
            order = np.argsort(-lg[t], kind="stable") if select == "top" else np.argsort(lg[t], kind="stable")
            ids = order[:spec.k]
            if weights == "softmax_k":
                e = np.exp(lg[t, ids] - lg[t, ids].max()); w = e / e.sum()
            elif weights == "softmax_all":
                e = np.exp(lg[t] - lg[t].max()); w = (e / e.sum())[ids]
            else:
                w = np.exp(lg[t, ids] - lg[t, ids].max())
            for j, ex in enumerate(ids):
                wg = Wg[ex].T if gate_t else Wg[ex]
                g = wg @ x[t] + bg[ex]
                u = Wu[ex] @ x[t] + bu[ex]
                if swap:
                    g, u = u, g
                h = O.clipped_swiglu(g, u, L, a)
                o = Wd[ex] @ h
                if bias == "weighted":
                    ys[t] += w[j] * (o + bd[ex])
                elif bias == "unweighted":
                    ys[t] += w[j] * o + bd[ex]
                else:
                    ys[t] += w[j] * o
        return ys

    want = np.array([brute.layer_token(layer, t, spec.k, L)["y"] for t in range(spec.T)])
    np.testing.assert_allclose(O.layer_forward(layer, spec.k, L)["y"], want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(layer_y(), want, rtol=1e-12, atol=1e-12)
    for kw in (dict(weights="softmax_all"), dict(select="bottom"), dict(bias="none"), dict(bias="unweighted"),
               dict(gate_t=True), dict(swap=True), dict(weights="unnormalised")):
        assert not np.allclose(layer_y(**kw), want, rtol=1e-6, atol=1e-9), kw


# --------------------------------------------------------------------------- #
# input recipes
# --------------------------------------------------------------------------- #
def test_bf16_rounding_recipe():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0], np.float32)
    bits = W.f32_to_bf16_bits(v)
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000]    # ties to even


def test_zipf_bias_is_log_probability():
    b = W.zipf_log_bias(128, 1.1)
    assert abs(np.exp(b).sum() - 1.0) < 1e-12
    assert np.all(np.diff(b) < 0)
    np.testing.assert_allclose(b[0] - b[1], 1.1 * math.log(2.0), rtol=1e-12)


def test_near_tie_rejection_meets_gap():
    spec = W.TINY_FP32
    layer = W.make_layer(spec, seed=0, logits_fn=_logits_fn)
    lg = _logits_fn(layer)
    srt = -np.sort(-lg, axis=1)
    assert np.all(srt[:, spec.k - 1] - srt[:, spec.k] >= 1e-3)
    assert layer["x"].dtype == np.float32 and layer["w_gate"].shape == (8, 512, 256)
    assert layer["w_down"].shape == (8, 256, 512)


def test_mxfp4_recipe_ranges():
    spec = W.tiny_spec(T=4, D=64, E=3, k=2, F=32, dtype="bf16", wfmt="mxfp4")
    layer = W.make_layer(spec, seed=0)
    assert layer["w_gate"].shape == (3, 32, 32) and layer["s_gate"].shape == (3, 32, 2)
    assert layer["w_down"].shape == (3, 64, 16) and layer["s_down"].shape == (3, 64, 1)
    for n in ("gate", "up", "down"):
        assert layer[f"s_{n}"].min() >= 119 and layer[f"s_{n}"].max() <= 127
