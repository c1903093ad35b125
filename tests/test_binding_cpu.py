"""The Python binding's argument checks, on CPU tensors (no device, no library call).

The C ABI receives bare pointers, so the binding checks every tensor's shape,
dtype, contiguity and device against the layouts the header documents before it
passes a pointer on.  These tests run the arrays the seeded workloads produce
(the same arrays the GPU tests upload) through those checks, and check that each
kind of mismatch is refused.
"""
import dataclasses

import numpy as np
import pytest

import workloads as W
from oracle import moe_oracle as O

torch = pytest.importorskip("torch")

from mixture_experts_ffn_12_b200 import api  # noqa: E402

SPECS = [W.TINY_FP32,
         W.tiny_spec(T=300, D=128, E=7, k=2, F=272, dtype="bf16", cfg_id=201),
         W.tiny_spec(T=77, D=96, E=5, k=3, F=144, dtype="f32", cfg_id=202),
         W.tiny_spec(T=40, D=32, E=1, k=1, F=32, dtype="bf16", cfg_id=204),
         W.tiny_spec(T=280, D=128, E=6, k=2, F=160, dtype="bf16", wfmt="mxfp4", cfg_id=205),
         W.tiny_spec(T=0, D=64, E=4, k=2, F=32, dtype="bf16", cfg_id=209)]


def _host(spec):
    layer = W.make_layer(spec, seed=0)
    return layer, {k: api.to_torch(v) for k, v in layer.items()}


@pytest.mark.parametrize("spec", SPECS, ids=lambda s: s.name)
def test_workload_arrays_pass_every_check(spec):
    layer, d = _host(spec)
    cfg = api.config_from_spec(spec)
    ew = api.expert_weights_from(d)
    T, k = spec.T, spec.k
    ids = torch.empty((T, k), dtype=torch.int32)
    w = torch.empty((T, k), dtype=torch.float32)
    assert api.check_router_args(cfg, d["x"], d["w_router"], d["b_router"], ids, w) == T
    assert api.check_layer_args(cfg, d["x"], d["w_router"], d["b_router"], ew, torch.empty_like(d["x"]),
                                ids, w) == T
    api.check_expert_weights(cfg, ew)
    # the dispatch and expert arrays as the oracle lays them out
    rid = np.zeros((T, k), np.int32) if T == 0 else \
        O.topk_softmax(O.router_logits(layer["x"], layer["w_router"], layer["b_router"]), k)[0].astype(np.int32)
    off, ros, sor = O.dispatch(rid, spec.E)
    assert api.check_permute_args(cfg, torch.from_numpy(rid), d["x"]) == T
    assert api.check_permute_args(cfg, torch.from_numpy(rid)) == T
    x_perm = api.to_torch(O.permute_rows(layer["x"], sor, k) if T else layer["x"][:0])
    x_perm = x_perm.reshape(T * k, spec.D)
    assert api.check_expert_ffn_args(cfg, x_perm, torch.from_numpy(off), ew) == T
    y_perm = torch.empty((T * k, spec.D), dtype=api.torch_dtype(cfg))
    assert api.check_combine_args(cfg, y_perm, torch.from_numpy(ros), w) == T


def _expect_refused(fn, *args, match):
    with pytest.raises(ValueError, match=match):
        fn(*args)


def test_mismatches_are_refused():
    spec = SPECS[1]                                   # bf16 dense
    _, d = _host(spec)
    cfg = api.config_from_spec(spec)
    x, wr, br = d["x"], d["w_router"], d["b_router"]
    T, D, E, k = spec.T, spec.D, spec.E, spec.k
    # dtype: an fp32 x where the layer is bf16 (would be read as 2T rows of bf16)
    _expect_refused(api.check_router_args, cfg, x.float(), wr, br, match="dtype")
    # shape: x with the wrong width, a router with the wrong expert count
    _expect_refused(api.check_router_args, cfg, x[:, :-16].contiguous(), wr, br, match="shape")
    _expect_refused(api.check_router_args, cfg, x, wr[:-1].contiguous(), br, match="shape")
    # a strided view
    wide = torch.empty((T, 2 * D), dtype=x.dtype)
    _expect_refused(api.check_router_args, cfg, wide[:, :D], wr, br, match="contiguous")
    # outputs of the wrong dtype / shape
    _expect_refused(api.check_router_args, cfg, x, wr, br, torch.empty((T, k), dtype=torch.int64),
                    match="dtype")
    _expect_refused(api.check_router_args, cfg, x, wr, br, None, torch.empty((T, k + 1)), match="shape")
    # a tensor on another device
    _expect_refused(api.check_router_args, cfg, x, wr.to("meta"), br, match="expected cpu")
    # a missing argument
    _expect_refused(api.check_router_args, cfg, None, wr, br, match="required")
    # permute: int64 ids
    _expect_refused(api.check_permute_args, cfg, torch.zeros((T, k), dtype=torch.int64), match="dtype")
    # expert_ffn: row count not a multiple of k, int64 offsets
    ew = api.expert_weights_from(d)
    xp = torch.empty((T * k + 1, D), dtype=x.dtype)
    _expect_refused(api.check_expert_ffn_args, cfg, xp, torch.zeros(E + 1, dtype=torch.int32), ew,
                    match="multiple of k")
    xp = torch.empty((T * k, D), dtype=x.dtype)
    _expect_refused(api.check_expert_ffn_args, cfg, xp, torch.zeros(E + 1, dtype=torch.int64), ew, match="dtype")
    # weights: transposed down projection, missing bias
    bad = dataclasses.replace(ew, w_down=ew.w_down.transpose(1, 2).contiguous())
    _expect_refused(api.check_expert_weights, cfg, bad, match="w_down: shape")
    _expect_refused(api.check_expert_weights, cfg, dataclasses.replace(ew, b_down=None), match="b_down is required")
    # combine: y_perm rows must be T*k
    _expect_refused(api.check_combine_args, cfg, torch.empty((T, D), dtype=x.dtype),
                    torch.zeros((T, k), dtype=torch.int32), torch.zeros((T, k)), match="y_perm: shape")


def test_mxfp4_weights_need_codes_and_scales():
    spec = SPECS[4]
    _, d = _host(spec)
    cfg = api.config_from_spec(spec)
    ew = api.expert_weights_from(d)
    api.check_expert_weights(cfg, ew)
    _expect_refused(api.check_expert_weights, cfg, dataclasses.replace(ew, s_gate=None), match="s_gate is required")
    # dense bf16 weights under an MXFP4 config
    E, F, D = spec.E, spec.F, spec.D
    dense = dataclasses.replace(ew, w_gate=torch.empty((E, F, D), dtype=torch.bfloat16))
    _expect_refused(api.check_expert_weights, cfg, dense, match="w_gate")
    # scales with one byte per 16 elements instead of 32
    _expect_refused(api.check_expert_weights, cfg,
                    dataclasses.replace(ew, s_up=torch.empty((E, F, D // 16), dtype=torch.uint8)),
                    match="s_up: shape")


GLM_SPECS = [W.glm_tiny_spec(T=7, D=16, E=6, k=2, F=16, F_shared=32, dtype="f32"),
             W.glm_tiny_spec(T=5, D=32, E=4, k=3, F=16, F_shared=0, dtype="bf16", correction_b_std=None, cfg_id=311)]


@pytest.mark.parametrize("spec", GLM_SPECS, ids=lambda s: s.name)
def test_glm_arrays_pass_the_variant_checks(spec):
    d = {k: api.to_torch(v) for k, v in W.make_glm_layer(spec).items()}
    cfg = api.glm_config_from_spec(spec)
    params = api.glm_params_from(spec, d)
    assert params.shared_intermediate_size == spec.F_shared
    T, k = spec.T, spec.k
    assert api.check_glm_args(cfg, params, d["x"], d["w_router"], api.glm_expert_weights_from(d),
                              torch.empty_like(d["x"]), torch.empty((T, k), dtype=torch.int32),
                              torch.empty((T, k))) == T
    c = params.c_struct()
    assert c.shared_intermediate_size == spec.F_shared and c.norm_topk_prob == int(spec.norm_topk_prob)


def test_glm_mismatches_are_refused():
    spec = GLM_SPECS[0]
    d = {k: api.to_torch(v) for k, v in W.make_glm_layer(spec).items()}
    cfg = api.glm_config_from_spec(spec)
    params = api.glm_params_from(spec, d)
    x, wr = d["x"], d["w_router"]
    _expect_refused(api.check_glm_args, cfg, dataclasses.replace(params, ws_up=None), x, wr, match="ws_up is required")
    _expect_refused(api.check_glm_args, cfg,
                    dataclasses.replace(params, ws_down=params.ws_down.t().contiguous()), x, wr, match="ws_down: shape")
    _expect_refused(api.check_glm_args, cfg,
                    dataclasses.replace(params, e_score_correction_bias=torch.zeros(spec.E + 1)), x, wr,
                    match="e_score_correction_bias: shape")
    mx = api.make_config(spec.D, spec.F, spec.E, spec.k, dtype="bf16", wfmt="mxfp4")
    _expect_refused(api.check_glm_args, mx, params, x, wr, match="dense expert weights")
