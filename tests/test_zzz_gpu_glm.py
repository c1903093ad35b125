"""The GLM4-MoE-Lite variant on the GPU against its CPU oracle, through the C ABI (marked gpu).

Source of the variant: "Ollama glm4_moe_lite.go" (MoEGate.Forward, SwitchMLP.Forward,
SharedExperts.Forward, MoE.Forward).  Bit-exact: the chosen expert sets (and their
order where the corrected scores are separated).  Routing weights within 2e-5 (they
include routed_scaling_factor).  Each layer runs with the output in the layer dtype
and in fp32 (y_f32), and (bf16) with h kept as two bf16 halves (h_split): that
form's fp32 output within 2e-2 of the output's RMS, the bound of the GPT-OSS layer
as written; the default form within the bf16 rounding of h of it; the dtype output
exactly the rounding of the fp32 output.
"""
import numpy as np
import pytest

import workloads as W
from oracle import glm_moe as G
from parity_util import (TOL_W, TOL_Y, check_h_rounding, check_ids, check_output, check_rounding, f64,
                         h_rounding_bound_glm)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api(cuda_ok):
    from mixture_experts_ffn_12_b200 import api as A, build
    build.build()
    return A


# T >= 256 with D = 256 (bf16): the tensor-core router with its K split; fewer tokens
# or fp32: the SIMT router.  <= 16 rows per expert on average: the decode kernels.
GLM_TC_ROUTER = W.glm_tiny_spec(T=300, D=256, E=8, k=2, F=144, F_shared=96, dtype="bf16", cfg_id=330)
GLM_F32 = W.glm_tiny_spec(T=77, D=96, E=5, k=3, F=48, F_shared=32, dtype="f32", cfg_id=331)
GLM_DECODE = W.glm_tiny_spec(T=40, D=64, E=16, k=4, F=64, F_shared=0, dtype="bf16", norm_topk_prob=False,
                             routed_scaling_factor=1.0, correction_b_std=None, cfg_id=332)
GLM_K1 = W.glm_tiny_spec(T=20, D=32, E=4, k=1, F=32, F_shared=32, dtype="bf16", cfg_id=333)
GLM_KE = W.glm_tiny_spec(T=30, D=32, E=4, k=4, F=32, F_shared=16, dtype="bf16", cfg_id=334)
GLM_MANY = W.glm_tiny_spec(T=300, D=256, E=64, k=6, F=64, F_shared=64, dtype="bf16", router_w_std=0.1, cfg_id=335)
SPECS = [GLM_TC_ROUTER, GLM_F32, GLM_DECODE, GLM_K1, GLM_KE, GLM_MANY]


def _scores_fn(spec):
    def f(layer):
        return G.route(G.gate_logits(layer["x"], layer["w_router"]), spec.k, layer.get("e_score_correction_bias"))[3]
    return f


def _layer(spec):
    return W.make_glm_layer(spec, seed=0, scores_fn=_scores_fn(spec))


def _run(api, spec, layer, split=True):
    """The layer with y in its dtype, with y in fp32, and (bf16, `split`) with y in fp32 and h
    in two bf16 halves: (y, y32, y32s or None, ids, w)."""
    d = api.upload_layer(layer)
    params = api.glm_params_from(spec, d)
    out = []
    modes = [(False, False), (True, False)] + ([(True, True)] if split and spec.dtype == "bf16" else [])
    for y_f32, h_split in modes:
        cfg = api.glm_config_from_spec(spec, y_f32=y_f32, h_split=h_split)
        ids = torch.empty((spec.T, spec.k), dtype=torch.int32, device="cuda")
        w = torch.empty((spec.T, spec.k), dtype=torch.float32, device="cuda")
        y = api.glm_layer_forward(cfg, params, d["x"], d["w_router"], api.glm_expert_weights_from(d),
                                  topk_ids=ids, topk_w=w)
        torch.cuda.synchronize()
        assert api.last_device_error() == 0
        out.append((y, ids, w))
    y, ids, w = out[0]
    for _, ids2, w2 in out[1:]:
        assert torch.equal(ids, ids2) and torch.equal(w, w2)
    y32s = out[2][0] if len(out) > 2 else None
    return y, out[1][0], y32s, ids.cpu().numpy(), w.cpu().numpy().astype(np.float64)


def _check_layer(y, y32, y32s, ref, tol, layer):
    if y32s is not None:
        print("h in two bf16 halves:", end=" ")
        check_output(f64(y32s), ref["y"], tol)
        check_h_rounding(f64(y32), f64(y32s), h_rounding_bound_glm(layer, ref), ref["y"])
        rms = float(np.sqrt(np.mean(np.square(ref["y"]))))
        print(f"h in bf16: max err / RMS = {np.max(np.abs(f64(y32) - ref['y'])) / rms:.3e}")
    else:
        check_output(f64(y32), ref["y"], tol)
    check_rounding(y, y32, ref["y"])


def _check_weights(gid, gw, rid, rw):
    got = np.take_along_axis(gw, np.argsort(gid, axis=1), axis=1)
    ref = np.take_along_axis(rw, np.argsort(rid, axis=1), axis=1)
    assert np.max(np.abs(got - ref)) <= TOL_W


@pytest.mark.parametrize("spec", SPECS, ids=lambda s: s.name)
def test_glm_layer_forward(api, spec):
    layer = _layer(spec)
    y, y32, y32s, gid, gw = _run(api, spec, layer)
    ref = G.layer_forward(layer, spec.k, spec.norm_topk_prob, spec.routed_scaling_factor)
    check_ids(gid, ref["ids"], ref["chosen_by"])
    _check_weights(gid, gw, ref["ids"], ref["w"])
    _check_layer(y, y32, y32s, ref, TOL_Y[spec.dtype], layer)


@pytest.mark.parametrize("spec", [GLM_TC_ROUTER, GLM_F32, GLM_K1, GLM_MANY], ids=lambda s: s.name)
def test_glm_router_topk(api, spec):
    layer = _layer(spec)
    d = api.upload_layer({k: layer[k] for k in layer if k in ("x", "w_router", "e_score_correction_bias")})
    ids, w = api.glm_router_topk(api.glm_config_from_spec(spec), api.glm_params_from(spec, d), d["x"], d["w_router"])
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    rid, rw, _, chosen_by = G.route(G.gate_logits(layer["x"], layer["w_router"]), spec.k,
                                    layer.get("e_score_correction_bias"), spec.norm_topk_prob,
                                    spec.routed_scaling_factor)
    gid = ids.cpu().numpy()
    check_ids(gid, rid, chosen_by)
    _check_weights(gid, w.cpu().numpy().astype(np.float64), rid, rw)
    if spec.k > 1 and spec.norm_topk_prob:
        np.testing.assert_allclose(w.sum(dim=1).cpu().numpy(), spec.routed_scaling_factor, rtol=1e-6)


@pytest.mark.parametrize("variant", [1, 2, 3, 4], ids=["single_cta", "cta_pair", "decode", "wm_pair"])
def test_glm_each_gemm_variant(api, variant):
    """SiLU(g) * u through every bf16 expert-GEMM kernel (routed and shared experts)."""
    spec = GLM_TC_ROUTER
    layer = _layer(spec)
    api.set_expert_gemm_variant(variant)
    try:
        y, y32, y32s, gid, _ = _run(api, spec, layer, split=variant != 4)
    finally:
        api.set_expert_gemm_variant(0)
    ref = G.layer_forward(layer, spec.k, spec.norm_topk_prob, spec.routed_scaling_factor)
    check_ids(gid, ref["ids"], ref["chosen_by"])
    _check_layer(y, y32, y32s, ref, TOL_Y["bf16"], layer)


def test_glm_zero_tokens(api):
    from mixture_experts_ffn_12_b200 import _lib
    spec = W.glm_tiny_spec(T=0, D=32, E=4, k=2, F=32, F_shared=16, dtype="bf16", cfg_id=336)
    d = api.upload_layer(W.make_glm_layer(spec))
    lib = _lib.load()
    before = lib.moe_launch_count()
    y = api.glm_layer_forward(api.glm_config_from_spec(spec), api.glm_params_from(spec, d), d["x"], d["w_router"],
                              api.glm_expert_weights_from(d))
    torch.cuda.synchronize()
    assert tuple(y.shape) == (0, spec.D)
    assert lib.moe_launch_count() == before
