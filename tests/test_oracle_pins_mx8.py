"""Pins of the MXFP8-activation oracle (``oracle.mx_act``) -- CPU only.

Sources: MXFP4 expert weights ("GPT-OSS 20B GGUF with MoE CPU Offloading", Model
Specifications); group size 32 for the 4-bit and MXFP8 formats ("Ollama
glm4_moe_lite.go", quantizationParams).  The E4M3 element format is the OCP 8-bit
floating point one; its value table and round-to-nearest-even are pinned against
PyTorch's own float8_e4m3fn conversion (a library routine) and against a search
over every code (``oracle.brute``), the scale rule against its closed form and a
search, and the variant layer against a scalar-loop restatement.  Planted
mistakes in the quantizer and in the layer must all be caught.
"""
import numpy as np
import pytest

import workloads as W
from oracle import brute as B
from oracle import moe_oracle as O
from oracle import mx_act as M

torch = pytest.importorskip("torch")


def test_e4m3_table_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ours = M.e4m3_value(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert nan.sum() == 2 and np.array_equal(np.isnan(ours), nan)    # S.1111.111 only
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.nanmax(ours) == 448.0 and np.nanmin(ours) == -448.0
    # and against the field-by-field table of the brute-force module
    table = dict(B.e4m3_table())
    assert all(ours[c] == v for c, v in table.items())


def test_e4m3_round_matches_torch_and_search():
    rng = np.random.default_rng(0)
    grid = M.e4m3_value(np.arange(256))
    grid = np.unique(grid[np.isfinite(grid)])
    mids = (grid[1:] + grid[:-1]) / 2                # exact ties: must go to the even mantissa
    v = np.concatenate([grid, mids, rng.uniform(-448, 448, 4000), rng.normal(0, 1, 4000),
                        rng.normal(0, 1e-2, 2000), np.ldexp(rng.uniform(-1, 1, 500), -8)])
    ours = M.e4m3_round(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)
    for t in v[::97]:
        assert M.e4m3_round(np.array([t]))[0] == B.e4m3_nearest(float(t))


def test_e4m3_round_saturates_and_keeps_grid():
    assert M.e4m3_round(np.array([500.0, -1e6]))[0] == 448.0
    assert M.e4m3_round(np.array([500.0, -1e6]))[1] == -448.0
    assert M.e4m3_round(np.array([464.0]))[0] == 448.0        # above the top of the grid
    assert M.e4m3_round(np.array([2.0 ** -10]))[0] == 0.0     # half the smallest subnormal: tie to 0
    assert M.e4m3_round(np.array([3 * 2.0 ** -10]))[0] == 2.0 ** -8   # tie 1.5 ulp -> even (2)


@pytest.mark.parametrize("amax,X", [(448.0, 0), (448.00001, 1), (1.0, -8), (1.75, -8), (1.7500001, -7),
                                   (0.875, -9), (0.0, -127), (7.0, -6), (49.0, -3), (2.0 ** -140, -127)])
def test_scale_exponent_cases(amax, X):
    """X is the smallest integer with amax <= 448 * 2^X (448 = 1.75 * 2^8)."""
    assert M.scale_exponent(np.array([amax]))[0] == X
    if amax > 2.0 ** -130:
        assert B.mx8_exponent(amax) == X


def test_scale_exponent_matches_search():
    rng = np.random.default_rng(1)
    a = np.concatenate([np.abs(rng.normal(0, 1, 300)), np.ldexp(1.75, np.arange(-20, 20)),
                        np.nextafter(np.ldexp(1.75, np.arange(-20, 20)), np.inf), rng.uniform(0, 60, 100)])
    X = M.scale_exponent(a)
    assert all(int(x) == B.mx8_exponent(float(t)) for x, t in zip(X, a))


def test_quantize_invariants():
    rng = np.random.default_rng(2)
    a = rng.normal(0, 3, (64, 256)) * np.exp(rng.normal(0, 2, (64, 1)))
    q, X = M.quantize(a)
    s = np.ldexp(1.0, X)
    scaled = np.abs(q.reshape(64, 8, 32)) / s[..., None]
    # no element saturates, and no smaller scale would do
    assert np.all(scaled <= 448.0)
    amax = np.max(np.abs(a.reshape(64, 8, 32)), axis=-1)
    assert np.all(amax <= 448.0 * s) and np.all(amax > 448.0 * s / 2)
    # every element within half an E4M3 step of its value (relative 2^-4 for normal values)
    err = np.abs(q - a).reshape(64, 8, 32)
    step = np.maximum(np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(a.reshape(64, 8, 32)) / s[..., None],
                                                                 2.0 ** -6))).astype(int) - 3), 2.0 ** -9)
    assert np.all(err <= step / 2 * s[..., None] * (1 + 1e-12))
    # quantizing twice changes no value (a block whose largest element rounded down to 224 * 2^X
    # may pick the next smaller scale the second time, on which its values are still exact)
    assert np.array_equal(M.quantize(q)[0], q)


def test_quantize_matches_brute_rows():
    rng = np.random.default_rng(3)
    a = rng.normal(0, 2, (3, 96))
    q, _ = M.quantize(a)
    for r in range(3):
        assert np.array_equal(q[r], np.array(B.mx8_row(list(a[r]))))


MX_TINY = W.tiny_spec(T=12, D=64, E=4, k=2, F=64, dtype="bf16", wfmt="mxfp4", cfg_id=501)


@pytest.fixture(scope="module")
def mx_layer():
    return W.make_layer(MX_TINY, seed=0,
                        logits_fn=lambda l: O.router_logits(l["x"], l["w_router"], l["b_router"]))


def test_variant_layer_matches_scalar_loops(mx_layer):
    spec = MX_TINY
    ref = M.layer_tokens(mx_layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
    for t in range(spec.T):
        b = B.layer_token_mx8(mx_layer, t, spec.k, spec.limit, spec.alpha)
        assert sorted(b["ids"]) == sorted(ref["ids"][t].tolist())
        np.testing.assert_allclose(b["y"], ref["y"][t], rtol=1e-12, atol=1e-12)


def test_variant_reduces_to_plain_layer_on_grid_activations(mx_layer):
    """With x already on the MXFP8 grid and h quantization taken out, the variant is the plain
    layer: the only difference between them is the two quantizers."""
    spec = MX_TINY
    lay = dict(mx_layer)
    xq, _ = M.quantize(O.decode(lay["x"]))
    lay["x"] = xq
    plain = O.layer_tokens(lay, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
    orig = M.quantize
    try:
        calls = []

        def q_x_only(a):
            calls.append(a.shape)
            return orig(a) if len(calls) == 1 else (a, None)
        M.quantize = q_x_only
        var = M.layer_tokens(lay, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
    finally:
        M.quantize = orig
    np.testing.assert_allclose(var["y"], plain["y"], rtol=1e-12, atol=1e-13)


def _plant(monkeypatch, name, fn):
    monkeypatch.setattr(M, name, fn)


@pytest.mark.parametrize("mistake", ["floor_scale", "no_h_quant", "truncate", "block16", "scale_off_by_one"])
def test_planted_mistakes_are_caught(mx_layer, monkeypatch, mistake):
    spec = MX_TINY
    good = M.layer_tokens(mx_layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)["y"]
    orig_q, orig_round, orig_exp = M.quantize, M.e4m3_round, M.scale_exponent
    if mistake == "floor_scale":        # the floor-of-log2 rule, which lets the largest elements saturate
        _plant(monkeypatch, "scale_exponent",
               lambda a: np.where(np.asarray(a) > 0, np.floor(np.log2(np.where(np.asarray(a) > 0, a, 1.0))) - 8,
                                  -127).astype(np.int64))
    elif mistake == "no_h_quant":
        calls = []

        def q(a):
            calls.append(1)
            return orig_q(a) if len(calls) == 1 else (a, None)
        _plant(monkeypatch, "quantize", q)
    elif mistake == "truncate":         # round toward zero on the E4M3 grid instead of to nearest
        grid = np.unique(np.abs(M.e4m3_value(np.arange(128))[:-1]))

        def trunc(v):
            v = np.asarray(v, dtype=np.float64)
            i = np.searchsorted(grid, np.minimum(np.abs(v), 448.0), side="right") - 1
            return np.sign(v) * grid[i]
        _plant(monkeypatch, "e4m3_round", trunc)
    elif mistake == "block16":
        def q16(a):
            a = np.asarray(a, dtype=np.float64)
            blocks = a.reshape(*a.shape[:-1], a.shape[-1] // 16, 16)
            X = orig_exp(np.max(np.abs(blocks), axis=-1))
            s = np.ldexp(1.0, X)[..., None]
            return (orig_round(blocks / s) * s).reshape(a.shape), X
        _plant(monkeypatch, "quantize", q16)
    elif mistake == "scale_off_by_one":
        _plant(monkeypatch, "scale_exponent", lambda a: orig_exp(a) + 1)
    bad = M.layer_tokens(mx_layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)["y"]
    assert not np.allclose(bad, good, rtol=1e-9, atol=1e-12)
