"""The gate/up A rows gathered from x by TMA gather4 (marked gpu).

With expert-GEMM variant 6, moe_layer_forward's single-CTA gate/up kernel loads the rows of
each expert's tile straight from x (row slot_of_row[r] / k for permuted row r), four rows per
`tile::gather4`, so the dispatch writes no x_perm; by default (variant 0) it reads them from
the dispatched x_perm.  Asserted, through the C ABI: the two give the same output bit
for bit (y in fp32 and in the layer dtype, h in one value and in two halves), the gathered
form launches one kernel fewer (no row copy), and the output meets the bound against the
oracle.  Shapes: ragged experts and feature blocks, an expert with no rows, D not a multiple
of 64 (a partial last K block), k = 8, and the GPT-OSS-20B prefill layer.
"""
import numpy as np
import pytest

import workloads as W
from oracle import moe_oracle as O
from parity_util import check_ids, check_output, f64, layer_for, tol_for

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api(cuda_ok):
    from mixture_experts_ffn_12_b200 import api as A, build
    build.build()
    return A


SPECS = [
    W.tiny_spec(T=300, D=128, E=7, k=2, F=272, dtype="bf16", cfg_id=801),
    W.tiny_spec(T=900, D=256, E=5, k=2, F=272, dtype="bf16", cfg_id=802, dead_experts=(3,), router_w_std=0.2),
    W.tiny_spec(T=400, D=208, E=6, k=3, F=176, dtype="bf16", cfg_id=803, router_w_std=0.2),
    W.tiny_spec(T=520, D=128, E=16, k=8, F=64, dtype="bf16", cfg_id=804, router_w_std=0.2),
]


def _forward(api, spec, d, ew, variant, y_f32, h_split):
    from mixture_experts_ffn_12_b200 import _lib
    lib = _lib.load()
    cfg = api.config_from_spec(spec, y_f32=y_f32, h_split=h_split)
    api.set_expert_gemm_variant(variant)
    try:
        n0 = lib.moe_launch_count()
        y = api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew)
        n = lib.moe_launch_count() - n0
        torch.cuda.synchronize()
    finally:
        api.set_expert_gemm_variant(0)
    assert api.last_device_error() == 0
    return y, n


@pytest.mark.parametrize("spec", SPECS + [W.GPTOSS20B_PREFILL], ids=lambda s: s.name)
def test_gathered_rows_match_x_perm(api, spec):
    layer = layer_for(spec)
    d = api.upload_layer(layer)
    ew = api.expert_weights_from(d)
    for y_f32, h_split in ((True, False), (False, False), (True, True)):
        yg, ng = _forward(api, spec, d, ew, 6, y_f32, h_split)
        yp, np_ = _forward(api, spec, d, ew, 0, y_f32, h_split)
        assert torch.equal(yg.view(torch.int16) if yg.dtype == torch.bfloat16 else yg.view(torch.int32),
                           yp.view(torch.int16) if yp.dtype == torch.bfloat16 else yp.view(torch.int32))
        assert ng == np_ - 1, (ng, np_)
    if spec.T <= 1000:
        ids = torch.empty((spec.T, spec.k), dtype=torch.int32, device="cuda")
        cfg = api.config_from_spec(spec, y_f32=True, h_split=True)
        api.set_expert_gemm_variant(6)
        try:
            y = api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew, topk_ids=ids)
            torch.cuda.synchronize()
        finally:
            api.set_expert_gemm_variant(0)
        ref = O.layer_tokens(layer, np.arange(spec.T), spec.k, spec.limit, spec.alpha)
        check_ids(ids.cpu().numpy(), ref["ids"], ref["logits"])
        check_output(f64(y), ref["y"], tol_for(spec))
