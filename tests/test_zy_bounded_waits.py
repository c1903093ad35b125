"""Bounded waits: a kernel whose pipeline waits give up reports it and leaves the GPU usable.

Every wait inside the tcgen05 kernels is bounded (mbarrier polls against a global
timer).  With the limit set to 1 ns, any wait that is not satisfied on its first
polls gives up: the CTA raises its abort flag, lets the TMA loads and MMAs it
already issued land, frees TMEM and exits, and the device error word says
MOE_ERR_TIMEOUT.  Nothing traps, and the next normal call is correct.
"""
import numpy as np
import pytest

import workloads as W
from oracle import moe_oracle as O
from parity_util import check_ids, check_output, check_rounding, f64, layer_for, tol_for

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def test_timeout_is_reported_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixture_experts_ffn_12_b200 import _lib, api, build
    build.build()
    spec = W.tiny_spec(T=300, D=128, E=7, k=2, F=272, dtype="bf16", cfg_id=401)
    layer = layer_for(spec)
    d = api.upload_layer(layer)
    cfg = api.config_from_spec(spec)
    ew = api.expert_weights_from(d)
    assert api.last_device_error() == _lib.MOE_OK
    api.set_expert_gemm_variant(1)          # tcgen05 single-CTA kernels (router and experts)
    api.set_wait_limit_ns(1)
    try:
        api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew)
        torch.cuda.synchronize()
        status = api.last_device_error()
    finally:
        api.set_wait_limit_ns(0)
        api.set_expert_gemm_variant(0)
    assert status == _lib.MOE_ERR_TIMEOUT
    # the context is intact: a normal call is right (fp32 output within the bound, and the
    # bf16 output of a second call its rounding)
    ids = torch.empty((spec.T, spec.k), dtype=torch.int32, device="cuda")
    y32 = api.layer_forward(api.config_from_spec(spec, y_f32=True), d["x"], d["w_router"], d["b_router"], ew,
                            topk_ids=ids)
    y = api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew)
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.MOE_OK
    ref = O.layer_tokens(layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
    check_ids(ids.cpu().numpy(), ref["ids"], ref["logits"])
    check_output(f64(y32), ref["y"], tol_for(spec))
    check_rounding(y, y32, ref["y"])
