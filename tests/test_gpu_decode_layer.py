"""The two-kernel decode layer (router logits, then one persistent kernel for top-k,
dispatch, both expert projections and the combine) against the oracle (marked gpu).

It serves dense bf16 layers with at most 512 routed rows averaging at most 16 per
expert; expert-GEMM variant 5 takes it wherever it applies (the tests below, unless
they say otherwise), and by size (variant 0) moe_layer_forward takes it for 2 <= T with
T * k <= E.  Asserted, through the C ABI:
  * it is the path taken: two launches per call (variant 5; variant 0 by the rule);
  * expert ids bit-exact (as sets; order where the logits are separated); the fp32
    output within the acceptance bound (2e-2 of the RMS) of the oracle with h kept
    as two bf16 halves, and, for the default form, within the bf16 rounding of h of
    that; the bf16 output exactly the rounding of the fp32 output;
  * routing ids and weights bit-identical to the separate-kernel path (variant 3:
    router, dispatch, decode GEMMs, combine as separate launches), whose arithmetic
    the router and top-k share, and outputs within 1e-3 of the RMS of it;
  * bit-identical outputs over repeated calls (the split units are summed in a
    fixed order whichever CTA finishes last);
  * a wait that gives up is reported and leaves the context usable.
Shapes cover: fewer (unit, K block) steps than CTAs (empty ranges), ragged D and F
(partial K blocks and feature blocks), experts with several 32-row chunks (a Zipf
router bias), 256 experts with k = 8, k = 1, and the GPT-OSS-20B decode sizes.
"""
import numpy as np
import pytest

import workloads as W
from oracle import moe_oracle as O
from parity_util import check_ids, check_output, check_rounding, f64, layer_for, tol_for
from test_gpu_parity import _check_layer, _run_layer

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api(cuda_ok):
    from mixture_experts_ffn_12_b200 import api as A, build
    build.build()
    return A


@pytest.fixture(autouse=True)
def decode_layer_variant(api):
    """Variant 5 (the decode layer wherever it applies) around every test; back to 0 after."""
    api.set_expert_gemm_variant(5)
    yield
    api.set_expert_gemm_variant(0)


DL_TINY = W.tiny_spec(T=1, D=64, E=4, k=2, F=64, dtype="bf16", cfg_id=701)
DL_RAGGED = W.tiny_spec(T=20, D=208, E=8, k=2, F=176, dtype="bf16", cfg_id=702, router_w_std=0.2)
DL_SKEW = W.tiny_spec(T=128, D=256, E=32, k=4, F=192, dtype="bf16", cfg_id=703, router_b="zipf")
DL_MANY = W.tiny_spec(T=64, D=128, E=256, k=8, F=64, dtype="bf16", cfg_id=704, router_w_std=0.2)
DL_K1 = W.tiny_spec(T=50, D=128, E=8, k=1, F=128, dtype="bf16", cfg_id=705, router_w_std=0.2)
DL_SPECS = [DL_TINY, DL_RAGGED, DL_SKEW, DL_MANY, DL_K1]


def _launches_per_call(api, spec, layer):
    from mixture_experts_ffn_12_b200 import _lib
    lib = _lib.load()
    d = api.upload_layer(layer)
    cfg = api.config_from_spec(spec)
    ew = api.expert_weights_from(d)
    api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew)
    torch.cuda.synchronize()
    before = lib.moe_launch_count()
    api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew)
    torch.cuda.synchronize()
    return lib.moe_launch_count() - before


@pytest.mark.parametrize("spec", DL_SPECS, ids=lambda s: s.name)
def test_decode_layer_parity(api, spec):
    layer = layer_for(spec)
    assert _launches_per_call(api, spec, layer) == 2
    y, y32, y32s, gid, _ = _run_layer(api, spec, layer)
    ref = O.layer_tokens(layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
    check_ids(gid, ref["ids"], ref["logits"])
    _check_layer(y, y32, y32s, ref, spec, layer)
    if spec is DL_SKEW:
        counts = np.bincount(gid.ravel(), minlength=spec.E)
        assert counts.max() > 64, "the Zipf bias should give one expert several 32-row chunks"


def _layer_outputs(api, spec, layer, variant, y_f32=True, h_split=False):
    d = api.upload_layer(layer)
    cfg = api.config_from_spec(spec, y_f32=y_f32, h_split=h_split)
    ids = torch.empty((spec.T, spec.k), dtype=torch.int32, device="cuda")
    w = torch.empty((spec.T, spec.k), dtype=torch.float32, device="cuda")
    api.set_expert_gemm_variant(variant)
    try:
        y = api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], api.expert_weights_from(d), topk_ids=ids,
                              topk_w=w)
        torch.cuda.synchronize()
    finally:
        api.set_expert_gemm_variant(5)
    assert api.last_device_error() == 0
    return y, ids, w


@pytest.mark.parametrize("spec", [DL_RAGGED, DL_SKEW, W.gptoss20b_decode(8)], ids=lambda s: s.name)
def test_decode_layer_matches_separate_kernels(api, spec):
    layer = layer_for(spec)
    y, ids, w = _layer_outputs(api, spec, layer, 5)
    y3, ids3, w3 = _layer_outputs(api, spec, layer, 3)
    assert torch.equal(ids, ids3) and torch.equal(w, w3)
    a, b = f64(y), f64(y3)
    rms = float(np.sqrt(np.mean(np.square(b))))
    assert np.max(np.abs(a - b)) <= 1e-3 * rms


@pytest.mark.parametrize("h_split", [False, True])
@pytest.mark.parametrize("spec", [DL_TINY, DL_SKEW, W.gptoss20b_decode(1)], ids=lambda s: s.name)
def test_decode_layer_reproducible(api, spec, h_split):
    layer = layer_for(spec)
    outs = [_layer_outputs(api, spec, layer, 5, y_f32=True, h_split=h_split)[0] for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int32), outs[0].view(torch.int32))


@pytest.mark.parametrize("spec", [W.gptoss20b_decode(t) for t in (1, 64)], ids=lambda s: s.name)
def test_decode_layer_full_size_sampled(api, spec):
    """The GPT-OSS-20B layer at T = 1 and 64: every routing decision; outputs of sampled tokens."""
    layer = layer_for(spec)
    assert _launches_per_call(api, spec, layer) == 2
    y, ids, _ = _layer_outputs(api, spec, layer, 5, y_f32=True)
    toks = np.unique(np.linspace(0, spec.T - 1, min(spec.T, 9)).astype(np.int64))
    ref = O.layer_tokens(layer, toks, spec.k, spec.limit, spec.alpha)
    lg = O.router_logits(layer["x"], layer["w_router"], layer["b_router"])
    rid, _ = O.topk_softmax(lg, spec.k)
    check_ids(ids.cpu().numpy(), rid, lg)
    check_output(f64(y)[toks], ref["y"], tol_for(spec))


def test_decode_layer_timeout_reported_and_context_survives(api):
    from mixture_experts_ffn_12_b200 import _lib
    spec = DL_SKEW
    layer = layer_for(spec)
    d = api.upload_layer(layer)
    ew = api.expert_weights_from(d)
    assert api.last_device_error() == _lib.MOE_OK
    api.set_wait_limit_ns(1)
    try:
        api.layer_forward(api.config_from_spec(spec), d["x"], d["w_router"], d["b_router"], ew)
        torch.cuda.synchronize()
        status = api.last_device_error()
    finally:
        api.set_wait_limit_ns(0)
    assert status == _lib.MOE_ERR_TIMEOUT
    # the context is intact: the next calls are right
    ids = torch.empty((spec.T, spec.k), dtype=torch.int32, device="cuda")
    y32s = api.layer_forward(api.config_from_spec(spec, y_f32=True, h_split=True), d["x"], d["w_router"],
                             d["b_router"], ew, topk_ids=ids)
    y32 = api.layer_forward(api.config_from_spec(spec, y_f32=True), d["x"], d["w_router"], d["b_router"], ew)
    y = api.layer_forward(api.config_from_spec(spec), d["x"], d["w_router"], d["b_router"], ew)
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.MOE_OK
    ref = O.layer_tokens(layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
    check_ids(ids.cpu().numpy(), ref["ids"], ref["logits"])
    check_output(f64(y32s), ref["y"], tol_for(spec))
    check_rounding(y, y32, ref["y"])


@pytest.mark.parametrize("T,taken", [(1, False), (2, True), (8, True), (9, False)])
def test_decode_layer_selected_by_size(api, T, taken):
    """Variant 0: the decode layer from two tokens up to T * k <= E (here E = 16, k = 2)."""
    spec = W.tiny_spec(T=T, D=128, E=16, k=2, F=128, dtype="bf16", cfg_id=706, router_w_std=0.2)
    layer = layer_for(spec)
    api.set_expert_gemm_variant(0)
    n = _launches_per_call(api, spec, layer)
    assert (n == 2) == taken, n
    y, ids, _ = _layer_outputs(api, spec, layer, 0, y_f32=True, h_split=True)
    ref = O.layer_tokens(layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
    check_ids(ids.cpu().numpy(), ref["ids"], ref["logits"])
    check_output(f64(y), ref["y"], tol_for(spec))
