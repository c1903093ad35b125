"""CUDA path vs the CPU oracle, through the C ABI (all marked gpu).

Bit-exact: expert ids (as sets; slot order where the logits are separated),
the dispatch maps and x_perm.  Floating point: every whole-layer test runs the
layer with the output in the layer dtype and in fp32 (y_f32), and bf16 layers
with dense weights also with h kept as two bf16 halves (h_split).  Asserted:
  * the acceptance bound as written, max |y - y_ref| / RMS(y_ref) <= 2e-2 (bf16
    and fp32 layers) or 5e-2 (MXFP4), on the fp32 output of the most precise
    form of every layer (h_split where it exists), and on the default form
    (h in one bf16 value) of the configured workloads (tiny fp32, GPT-OSS-20B
    prefill and decode, MXFP4, GPT-OSS-120B skewed);
  * the default form differs from the h_split form by no more than the bf16
    rounding of h can explain (a per-element bound computed from the oracle's
    h and |W_d|);
  * the dtype output is exactly the round-to-nearest-even of the fp32 output.
The intermediates h and y_perm, which are stored in the activation dtype, get the
bound plus their storage rounding (2^-8 |ref| per element for bf16); routing
weights within 2e-5.
Full-size layers are compared on every routing decision and on a sample of
token outputs that the oracle computes one by one.
"""
import numpy as np
import pytest

import workloads as W
from oracle import moe_oracle as O
from parity_util import (TOL_W, check_h_rounding, check_ids, check_output, check_rounding, check_stored, f64,
                         h_rounding_bound, layer_for, rel_rms, tol_for)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api(cuda_ok):
    from mixture_experts_ffn_12_b200 import api as A, build
    build.build()
    return A


RAGGED_BF16 = W.tiny_spec(T=300, D=128, E=7, k=2, F=272, dtype="bf16", cfg_id=201)
RAGGED_F32 = W.tiny_spec(T=77, D=96, E=5, k=3, F=144, dtype="f32", cfg_id=202)
WIDE_K = W.tiny_spec(T=260, D=64, E=16, k=8, F=48, dtype="bf16", cfg_id=203)
ONE_EXPERT = W.tiny_spec(T=40, D=32, E=1, k=1, F=32, dtype="bf16", cfg_id=204)
MXFP4_SMALL = W.tiny_spec(T=280, D=128, E=6, k=2, F=160, dtype="bf16", wfmt="mxfp4", cfg_id=205)

# >= 128 rows per expert on average: runs the CTA-pair kernels; ragged F and D tiles, an expert with no rows
PAIR_RAGGED = W.tiny_spec(T=900, D=256, E=5, k=2, F=272, dtype="bf16", cfg_id=206, dead_experts=(3,),
                          router_w_std=0.2)

# <= 16 rows per expert with F = 64: the decode kernels by default, with fewer down units than
# SMs but a single 64-wide K block, so the down projection must not split K (an empty half
# would add an accumulator no MMA wrote)
DECODE_ONE_KBLOCK = W.tiny_spec(T=24, D=64, E=16, k=4, F=64, dtype="bf16", cfg_id=210, router_w_std=0.2)

SMALL_SPECS = [W.TINY_FP32, RAGGED_BF16, RAGGED_F32, WIDE_K, ONE_EXPERT, MXFP4_SMALL, PAIR_RAGGED, DECODE_ONE_KBLOCK]

# many experts: the K-split router with 16 / 32 threads per token in its top-k (E = 128 / 256),
# 256 expert groups in the GEMMs (the maximum), k = 8 (the maximum)
MANY_EXPERTS = [W.tiny_spec(T=300, D=512, E=128, k=8, F=96, dtype="bf16", cfg_id=207, router_w_std=0.2),
                W.tiny_spec(T=520, D=1024, E=256, k=8, F=64, dtype="bf16", cfg_id=208, router_w_std=0.2)]
DECODE_SPECS = [W.gptoss20b_decode(t) for t in W.GPTOSS20B_DECODE_T]


def dev(layer, api):
    return api.upload_layer(layer)


# --------------------------------------------------------------------------- #
# router + top-k
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("spec", SMALL_SPECS + [W.GPTOSS20B_PREFILL, W.gptoss20b_decode(8), W.GPTOSS120B_SKEWED],
                         ids=lambda s: s.name)
def test_router_topk(api, spec):
    layer = layer_for(spec, experts=False)
    d = dev({k: layer[k] for k in ("x", "w_router", "b_router")}, api)
    cfg = api.config_from_spec(spec)
    ids, w = api.router_topk(cfg, d["x"], d["w_router"], d["b_router"])
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    lg = O.router_logits(layer["x"], layer["w_router"], layer["b_router"])
    rid, rw = O.topk_softmax(lg, spec.k)
    gid = ids.cpu().numpy()
    check_ids(gid, rid, lg)
    # weights: compare on the oracle's order (same sets)
    gw = w.cpu().numpy().astype(np.float64)
    order_map = np.argsort(gid, axis=1)
    ref_sorted = np.take_along_axis(rw, np.argsort(rid, axis=1), axis=1)
    got_sorted = np.take_along_axis(gw, order_map, axis=1)
    assert np.max(np.abs(got_sorted - ref_sorted)) <= TOL_W
    np.testing.assert_allclose(gw.sum(axis=1), 1.0, atol=1e-6)


# --------------------------------------------------------------------------- #
# dispatch
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("T,E,k,D", [(1, 1, 1, 16), (5, 4, 2, 32), (257, 256, 8, 16), (1000, 3, 3, 48),
                                     (4096, 32, 4, 64), (70000, 128, 4, 16)])
def test_permute_bit_exact(api, T, E, k, D):
    rng = np.random.default_rng(T + E)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    x = rng.standard_normal((T, D)).astype(np.float32)
    cfg = api.make_config(D, 32, E, k, dtype="f32")
    out = api.permute(cfg, torch.from_numpy(ids).cuda(), torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    off, ros, sor = O.dispatch(ids, E)
    assert np.array_equal(out["expert_off"].cpu().numpy(), off)
    assert np.array_equal(out["row_of_slot"].cpu().numpy(), ros)
    assert np.array_equal(out["slot_of_row"].cpu().numpy(), sor)
    assert np.array_equal(out["x_perm"].cpu().numpy(), O.permute_rows(x, sor, k))


def test_permute_empty_and_index_only(api):
    cfg = api.make_config(32, 32, 4, 2, dtype="bf16")
    out = api.permute(cfg, torch.zeros((0, 2), dtype=torch.int32, device="cuda"))
    assert out["expert_off"].cpu().numpy().tolist() == [0] * 5
    ids = torch.tensor([[1, 0], [1, 3], [3, 2]], dtype=torch.int32, device="cuda")
    out = api.permute(cfg, ids)
    torch.cuda.synchronize()
    assert out["expert_off"].cpu().numpy().tolist() == [0, 1, 3, 4, 6]
    assert out["slot_of_row"].cpu().numpy().tolist() == [1, 0, 2, 5, 3, 4]


def test_permute_bad_ids_flag_device_error(api):
    from mixture_experts_ffn_12_b200 import _lib
    cfg = api.make_config(32, 32, 4, 2, dtype="bf16")
    ids = torch.tensor([[1, 7], [2, 2]], dtype=torch.int32, device="cuda")   # out of range; repeated
    api.permute(cfg, ids, torch.zeros((2, 32), dtype=torch.bfloat16, device="cuda"))
    assert api.last_device_error() == _lib.MOE_ERR_DEVICE_BOUNDS
    assert api.last_device_error() == 0                                        # cleared, context usable


# --------------------------------------------------------------------------- #
# expert FFN (gate/up + SwiGLU, down) and combine, from the oracle's dispatch
# --------------------------------------------------------------------------- #
def _expert_inputs(spec, layer, api):
    lg = O.router_logits(layer["x"], layer["w_router"], layer["b_router"])
    ids, w = O.topk_softmax(lg, spec.k)
    off, ros, sor = O.dispatch(ids, spec.E)
    xp = layer["x"][sor // spec.k]                          # permuted rows, storage format
    return ids, w, off, ros, sor, xp


@pytest.mark.parametrize("spec", SMALL_SPECS, ids=lambda s: s.name)
def test_expert_ffn(api, spec):
    layer = layer_for(spec)
    ids, w, off, ros, sor, xp = _expert_inputs(spec, layer, api)
    d = dev({k: v for k, v in layer.items() if k not in ("x",)}, api)
    cfg = api.config_from_spec(spec)
    h, yp = api.expert_ffn(cfg, api.to_torch(xp).cuda(), torch.from_numpy(off).cuda(), api.expert_weights_from(d))
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    rh, ry = O.expert_ffn(xp, off, layer, spec.limit, spec.alpha)
    tol = tol_for(spec)
    check_stored(f64(h), rh, tol, spec.dtype == "bf16")
    check_stored(f64(yp), ry, tol, spec.dtype == "bf16")


@pytest.mark.parametrize("variant", [0, 1, 2, 3], ids=["default", "single_cta", "cta_pair", "decode"])
@pytest.mark.parametrize("spec", [RAGGED_BF16, PAIR_RAGGED, DECODE_ONE_KBLOCK], ids=lambda s: s.name)
def test_expert_ffn_h_split(api, spec, variant):
    """h kept as two bf16 halves: hi is the bf16 rounding of h, hi + lo is h to about 16 bits,
    and y_perm (one bf16 value per element) stays within the bound plus its own rounding."""
    layer = layer_for(spec)
    ids, w, off, ros, sor, xp = _expert_inputs(spec, layer, api)
    d = dev({k: v for k, v in layer.items() if k not in ("x",)}, api)
    cfg = api.config_from_spec(spec, h_split=True)
    api.set_expert_gemm_variant(variant)
    try:
        h2, yp = api.expert_ffn(cfg, api.to_torch(xp).cuda(), torch.from_numpy(off).cuda(),
                                api.expert_weights_from(d))
        torch.cuda.synchronize()
    finally:
        api.set_expert_gemm_variant(0)
    assert api.last_device_error() == 0
    rh, ry = O.expert_ffn(xp, off, layer, spec.limit, spec.alpha)
    F = spec.F
    hi, lo = f64(h2[:, :F]), f64(h2[:, F:])
    rms = float(np.sqrt(np.mean(np.square(rh))))
    # hi + lo carries h to about 2^-16 of its size; the rest is the fp32 arithmetic of h
    assert np.all(np.abs(hi + lo - rh) <= 2.0 ** -14 * np.abs(rh) + 1e-6 * rms)
    # hi is h rounded to bf16 once, so |lo| is at most half an ulp of hi
    assert np.all(np.abs(lo) <= 2.0 ** -8 * np.abs(hi))
    check_stored(f64(yp), ry, 2e-2, True)


@pytest.mark.parametrize("variant", [1, 2, 4], ids=["single_cta", "cta_pair", "wm_pair"])
@pytest.mark.parametrize("spec", [RAGGED_BF16, WIDE_K, PAIR_RAGGED], ids=lambda s: s.name)
def test_expert_ffn_each_gemm_variant(api, spec, variant):
    """moe_expert_ffn (bf16 down rows, no weighting) through each prefill GEMM kernel."""
    layer = layer_for(spec)
    ids, w, off, ros, sor, xp = _expert_inputs(spec, layer, api)
    d = dev({k: v for k, v in layer.items() if k not in ("x",)}, api)
    cfg = api.config_from_spec(spec)
    api.set_expert_gemm_variant(variant)
    try:
        h, yp = api.expert_ffn(cfg, api.to_torch(xp).cuda(), torch.from_numpy(off).cuda(),
                               api.expert_weights_from(d))
        torch.cuda.synchronize()
    finally:
        api.set_expert_gemm_variant(0)
    assert api.last_device_error() == 0
    rh, ry = O.expert_ffn(xp, off, layer, spec.limit, spec.alpha)
    check_stored(f64(h), rh, tol_for(spec), True)
    check_stored(f64(yp), ry, tol_for(spec), True)


@pytest.mark.parametrize("variant", [0, 4], ids=["default", "wm_pair"])
@pytest.mark.parametrize("spec", [W.GPTOSS20B_PREFILL], ids=lambda s: s.name)
def test_expert_ffn_full_size_some_experts(api, spec, variant):
    """GPT-OSS-20B-shaped gate/up/down on all 16384 routed rows; the oracle checks three whole experts."""
    layer = layer_for(spec)
    ids, w, off, ros, sor, xp = _expert_inputs(spec, layer, api)
    d = dev({k: v for k, v in layer.items() if k not in ("x",)}, api)
    cfg = api.config_from_spec(spec)
    api.set_expert_gemm_variant(variant)
    try:
        h, yp = api.expert_ffn(cfg, api.to_torch(xp).cuda(), torch.from_numpy(off).cuda(),
                               api.expert_weights_from(d))
        torch.cuda.synchronize()
    finally:
        api.set_expert_gemm_variant(0)
    assert api.last_device_error() == 0
    for e in (0, 13, spec.E - 1):
        a, b = int(off[e]), int(off[e + 1])
        sub = dict(layer)
        sub_off = np.zeros(spec.E + 1, np.int32)
        sub_off[e + 1:] = b - a
        rh, ry = O.expert_ffn(xp[a:b], sub_off, sub, spec.limit, spec.alpha)
        check_stored(f64(h[a:b]), rh, 2e-2, True)
        check_stored(f64(yp[a:b]), ry, 2e-2, True)


@pytest.mark.parametrize("spec", [W.TINY_FP32, RAGGED_BF16, WIDE_K], ids=lambda s: s.name)
def test_combine(api, spec):
    rng = np.random.default_rng(11)
    T, k, D = spec.T, spec.k, spec.D
    ids = np.stack([rng.permutation(spec.E)[:k] for _ in range(T)]).astype(np.int32)
    _, ros, _ = O.dispatch(ids, spec.E)
    w = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    yp = rng.standard_normal((T * k, D)).astype(np.float32)
    if spec.dtype == "bf16":
        yp_store = W.f32_to_bf16_bits(yp)
    else:
        yp_store = yp
    cfg = api.config_from_spec(spec)
    y = api.combine(cfg, api.to_torch(yp_store).cuda(), torch.from_numpy(ros).cuda(), torch.from_numpy(w).cuda())
    ref = O.combine(O.decode(yp_store), ros, w.astype(np.float64))
    assert rel_rms(f64(y), ref) <= (1e-2 if spec.dtype == "bf16" else 1e-6)


# --------------------------------------------------------------------------- #
# whole layer
# --------------------------------------------------------------------------- #
# the workloads the acceptance bound is stated for: the default form must meet it too
CONFIGURED = {W.TINY_FP32.name, W.GPTOSS20B_PREFILL.name, W.GPTOSS20B_MXFP4.name, W.GPTOSS120B_SKEWED.name,
              *(W.gptoss20b_decode(t).name for t in W.GPTOSS20B_DECODE_T)}


def _run_layer(api, spec, layer, split=True):
    """Layer calls on the same inputs: y in the layer dtype, y in fp32, and (bf16 layers with
    dense weights, when `split`) y in fp32 with h kept as two bf16 halves.
    Returns (y, y32, y32s or None, ids, w); ids and w must agree between the calls."""
    d = dev(layer, api)
    ew = api.expert_weights_from(d)
    modes = [(False, False), (True, False)]
    if split and spec.dtype == "bf16" and spec.wfmt == "dense":
        modes.append((True, True))
    out = []
    for y_f32, h_split in modes:
        cfg = api.config_from_spec(spec, y_f32=y_f32, h_split=h_split)
        ids = torch.empty((spec.T, spec.k), dtype=torch.int32, device="cuda")
        w = torch.empty((spec.T, spec.k), dtype=torch.float32, device="cuda")
        y = api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew, topk_ids=ids, topk_w=w)
        torch.cuda.synchronize()
        assert api.last_device_error() == 0
        out.append((y, ids, w))
    y, ids, w = out[0]
    for _, ids2, w2 in out[1:]:
        assert torch.equal(ids, ids2) and torch.equal(w, w2)
    y32 = out[1][0]
    assert y32.dtype == torch.float32
    y32s = out[2][0] if len(out) > 2 else None
    return y, y32, y32s, ids.cpu().numpy(), w


def _check_layer(y, y32, y32s, ref, spec, layer):
    """The acceptance bound on the most precise form; the default form against it (configured
    workloads) and within the bf16 rounding of h of the precise form; the dtype output is the
    rounding of the fp32 output."""
    tol = tol_for(spec)
    if y32s is not None:
        print("h in two bf16 halves:", end=" ")
        check_output(f64(y32s), ref["y"], tol)
        bound = h_rounding_bound(layer, ref["ids"], ref["w"], ref["h"])
        check_h_rounding(f64(y32), f64(y32s), bound, ref["y"])
        if spec.name in CONFIGURED:
            print("h in bf16:", end=" ")
            check_output(f64(y32), ref["y"], tol)
        else:
            rms = float(np.sqrt(np.mean(np.square(ref["y"]))))
            print(f"h in bf16: max err / RMS = {np.max(np.abs(f64(y32) - ref['y'])) / rms:.3e}")
    else:
        check_output(f64(y32), ref["y"], tol)
    check_rounding(y, y32, ref["y"])


@pytest.mark.parametrize("spec", SMALL_SPECS + DECODE_SPECS, ids=lambda s: s.name)
def test_layer_forward_all_tokens(api, spec):
    layer = layer_for(spec)
    y, y32, y32s, gid, _ = _run_layer(api, spec, layer)
    ref = O.layer_tokens(layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
    check_ids(gid, ref["ids"], ref["logits"])
    _check_layer(y, y32, y32s, ref, spec, layer)


@pytest.mark.parametrize("spec", MANY_EXPERTS, ids=lambda s: s.name)
def test_layer_forward_many_experts(api, spec):
    layer = layer_for(spec)
    y, y32, y32s, gid, _ = _run_layer(api, spec, layer)
    ref = O.layer_tokens(layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
    check_ids(gid, ref["ids"], ref["logits"])
    _check_layer(y, y32, y32s, ref, spec, layer)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_layer_forward_zero_tokens(api, dtype):
    """T = 0: MOE_OK, nothing launched, nothing written."""
    from mixture_experts_ffn_12_b200 import _lib
    spec = W.tiny_spec(T=0, D=64, E=4, k=2, F=32, dtype=dtype, cfg_id=209)
    layer = layer_for(spec)
    d = dev(layer, api)
    lib = _lib.load()
    before = lib.moe_launch_count()
    y = api.layer_forward(api.config_from_spec(spec), d["x"], d["w_router"], d["b_router"],
                          api.expert_weights_from(d))
    torch.cuda.synchronize()
    assert tuple(y.shape) == (0, spec.D)
    assert lib.moe_launch_count() == before
    assert api.last_device_error() == 0


@pytest.mark.parametrize("spec", [W.GPTOSS20B_PREFILL, W.GPTOSS20B_MXFP4, W.GPTOSS120B_SKEWED],
                         ids=lambda s: s.name)
def test_layer_forward_full_size_sampled(api, spec):
    _full_size_sampled(api, spec)


@pytest.mark.parametrize("spec", [W.GPTOSS20B_PREFILL, W.GPTOSS120B_SKEWED], ids=lambda s: s.name)
def test_layer_forward_full_size_sampled_wm_pair(api, spec):
    """The full-size bf16 layers through the CTA-pair kernels with the weights in M."""
    api.set_expert_gemm_variant(4)
    try:
        _full_size_sampled(api, spec, split=False)   # this kernel has no two-halves form
    finally:
        api.set_expert_gemm_variant(0)


def _full_size_sampled(api, spec, split=True):
    layer = layer_for(spec)
    y, y32, y32s, gid, _ = _run_layer(api, spec, layer, split)
    # routing: every token, bit-exact
    lg = O.router_logits(layer["x"], layer["w_router"], layer["b_router"])
    rid, _ = O.topk_softmax(lg, spec.k)
    check_ids(gid, rid, lg)
    off, _, sor = O.dispatch(rid, spec.E)
    # outputs: a sample that covers the first and last tokens and the busiest expert
    rng = np.random.default_rng(5)
    toks = np.unique(np.concatenate([[0, spec.T - 1], rng.choice(spec.T, 46, replace=False),
                                     sor[off[0]:off[1]][:16] // spec.k]))
    ref = O.layer_tokens(layer, toks, spec.k, spec.limit, spec.alpha)
    sel = torch.from_numpy(toks).cuda()
    # the RMS of the full output, estimated from the sample
    _check_layer(y[sel], y32[sel], None if y32s is None else y32s[sel], ref, spec, layer)


def test_layer_forward_repeatable(api):
    """Two calls on the same inputs give bit-identical outputs (no order-dependent atomics)."""
    spec = RAGGED_BF16
    layer = layer_for(spec)
    d = dev(layer, api)
    cfg = api.config_from_spec(spec)
    ew = api.expert_weights_from(d)
    y1 = api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew)
    y2 = api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("variant", [1, 2, 3, 4], ids=["single_cta", "cta_pair", "decode", "wm_pair"])
@pytest.mark.parametrize("spec", [RAGGED_BF16, PAIR_RAGGED, W.gptoss20b_decode(8)], ids=lambda s: s.name)
def test_layer_forward_each_gemm_variant(api, spec, variant):
    """Every bf16 expert-GEMM kernel on the same layer: single-CTA 128-row tiles, CTA pairs
    (256 rows), the weight-stationary decode kernel (token chunks of 32, so experts with
    more rows run several chunks), and CTA pairs with the weights in M (token tiles of up
    to 256 columns, ragged last tiles rounded to 16)."""
    layer = layer_for(spec)
    api.set_expert_gemm_variant(variant)
    try:
        y, y32, y32s, gid, _ = _run_layer(api, spec, layer, split=variant != 4)
    finally:
        api.set_expert_gemm_variant(0)
    ref = O.layer_tokens(layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
    check_ids(gid, ref["ids"], ref["logits"])
    _check_layer(y, y32, y32s, ref, spec, layer)


def test_cuda_graph_replay_matches_eager(api):
    """A captured forward replays the same kernels on new contents of the input buffer."""
    spec = W.gptoss20b_decode(8)
    layer = layer_for(spec)
    d = dev(layer, api)
    moe = api.MoELayer(api.config_from_spec(spec), d["w_router"], d["b_router"], api.expert_weights_from(d))
    x = d["x"].clone()
    replay, y_graph = moe.graphed(x)
    x2 = torch.roll(d["x"], shifts=3, dims=0).contiguous()
    x.copy_(x2)
    replay()
    y_eager = moe(x2)
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    assert torch.equal(y_graph, y_eager)


def test_run_host_batches_matches_layer_calls(api):
    """The pipelined host->device->host runner gives each batch the layer's own output."""
    spec = RAGGED_BF16
    layer = layer_for(spec)
    d = dev(layer, api)
    moe = api.MoELayer(api.config_from_spec(spec), d["w_router"], d["b_router"], api.expert_weights_from(d))
    xs = [torch.roll(d["x"], shifts=7 * i, dims=0).contiguous() for i in range(5)]
    want = [moe(x).cpu() for x in xs]
    xs_host = [x.cpu().pin_memory() for x in xs]
    ys_host = [torch.empty_like(w).pin_memory() for w in want]
    moe.run_host_batches(xs_host, ys_host)
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    for got, w in zip(ys_host, want):
        assert torch.equal(got, w)


def test_mxfp4_matches_bf16_path_on_dequantised_weights(api):
    """Every dequantised MXFP4 weight is a bf16 number, so the in-mainloop dequant must give the
    bf16 CTA-pair kernel's result on those weights, bit for bit (same tiles, same accumulation order)."""
    spec = MXFP4_SMALL
    layer = layer_for(spec)
    dense = dict(layer)
    for name in ("gate", "up", "down"):
        wq = O.mxfp4_dequant(layer[f"w_{name}"], layer[f"s_{name}"])
        dense[f"w_{name}"] = W.f32_to_bf16_bits(wq.astype(np.float32))
        dense.pop(f"s_{name}")
        assert np.array_equal(W.bf16_bits_to_f32(dense[f"w_{name}"]).astype(np.float64), wq)
    import dataclasses
    y_mx, y32_mx, _, ids_mx, _ = _run_layer(api, spec, layer)
    api.set_expert_gemm_variant(2)
    try:
        y_bf, y32_bf, _, ids_bf, _ = _run_layer(api, dataclasses.replace(spec, wfmt="dense"), dense, split=False)
    finally:
        api.set_expert_gemm_variant(0)
    assert np.array_equal(ids_mx, ids_bf)
    assert torch.equal(y_mx, y_bf)
    assert torch.equal(y32_mx, y32_bf)
