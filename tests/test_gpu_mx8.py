"""MXFP4 weights with MXFP8 activations on the block-scaled tensor cores (marked gpu).

The layer's block-scaled numerics variant (MOE_W_MXFP4_A8) against its own oracle
(``oracle.mx_act``: the activations of both expert projections quantized to MXFP8,
everything else the plain layer in fp64), through the C ABI:
  * the quantizer itself (moe_quantize_mxfp8) is bit-exact: every E4M3 code and
    every scale byte equals the oracle's;
  * expert ids are bit-exact, and the layer's fp32 output is within 5e-2 of the
    output's RMS (the MXFP4 bound) of the variant's oracle; the bf16 output is
    exactly its rounding.  The variant's distance from the plain layer (what the
    8-bit activations cost) is printed.
"""
import numpy as np
import pytest

import workloads as W
from oracle import moe_oracle as O
from oracle import mx_act as M
from parity_util import TOL_Y, check_ids, check_output, check_rounding, f64, layer_for

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api(cuda_ok):
    from mixture_experts_ffn_12_b200 import api as A, build
    build.build()
    return A


def _bf16_rows(rng, rows, K):
    a = rng.normal(0, 1, (rows, K)) * np.exp(rng.normal(0, 3, (rows, 1)))
    a[0, :32] = 0.0                                   # an all-zero block
    a[1, :32] = 448.0 * 2.0 ** -5                     # largest magnitude exactly 448 * 2^X
    if K >= 64:
        a[1, 32:64] = 1.75 * 2.0 ** np.arange(-16, 16)    # one block spanning many binades
    a[2, :32] = 1e-30                                 # bf16 values far below the E4M3 range of 2^0
    return W.f32_to_bf16_bits(a.astype(np.float32))


@pytest.mark.parametrize("rows,K", [(1, 32), (37, 96), (300, 2880)])
def test_quantize_mxfp8_bit_exact(api, rows, K):
    rng = np.random.default_rng(rows + K)
    xb = _bf16_rows(rng, max(rows, 3), K)[:rows]
    xq, sf = api.quantize_mxfp8(api.to_torch(xb).cuda())
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    q, X = M.quantize(O.decode(xb))
    nb = K // 32
    sfn = sf.cpu().numpy()
    assert np.array_equal(sfn[:, :nb].astype(np.int64), X + 127)
    assert np.all(sfn[:, nb:] == 127)
    got = M.e4m3_value(xq.cpu().numpy()) * np.repeat(np.ldexp(1.0, sfn[:, :nb].astype(np.int64) - 127), 32, axis=1)
    assert np.array_equal(got, q)


MX8_SMALL = W.tiny_spec(T=300, D=128, E=6, k=2, F=192, dtype="bf16", wfmt="mxfp4", cfg_id=601)
# several row blocks per expert, a ragged last gate/up tile (F = 320 = 3 x 96 + 32), a down tile
# wider than D (192 < 240) and an expert with no rows
MX8_RAGGED = W.tiny_spec(T=700, D=192, E=5, k=2, F=320, dtype="bf16", wfmt="mxfp4", cfg_id=602, dead_experts=(2,),
                         router_w_std=0.2)
# many experts with a few rows each
MX8_MANY = W.tiny_spec(T=260, D=64, E=64, k=4, F=64, dtype="bf16", wfmt="mxfp4", cfg_id=603, router_w_std=0.2)


def _run_a8(api, spec, layer):
    d = api.upload_layer(layer)
    ew = api.expert_weights_from(d)
    out = []
    for y_f32 in (False, True):
        cfg = api.config_from_spec(spec, y_f32=y_f32, wfmt="mxfp4_a8")
        ids = torch.empty((spec.T, spec.k), dtype=torch.int32, device="cuda")
        y = api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew, topk_ids=ids)
        torch.cuda.synchronize()
        assert api.last_device_error() == 0
        out.append((y, ids))
    assert torch.equal(out[0][1], out[1][1])
    return out[0][0], out[1][0], out[0][1].cpu().numpy()


def _check(api, spec, layer, toks):
    y, y32, gid = _run_a8(api, spec, layer)
    lg = O.router_logits(layer["x"], layer["w_router"], layer["b_router"])
    rid, _ = O.topk_softmax(lg, spec.k)
    check_ids(gid, rid, lg)
    ref = M.layer_tokens(layer, toks, spec.k, spec.limit, spec.alpha)
    sel = torch.from_numpy(toks).cuda()
    check_output(f64(y32[sel]), ref["y"], TOL_Y["mxfp4"])
    check_rounding(y[sel], y32[sel], ref["y"])
    plain = O.layer_tokens(layer, toks, spec.k, spec.limit, spec.alpha)["y"]
    rms = float(np.sqrt(np.mean(np.square(plain))))
    print(f"variant oracle vs plain layer: max |dy| / RMS = {np.max(np.abs(ref['y'] - plain)) / rms:.3e}")


@pytest.mark.parametrize("spec", [MX8_SMALL, MX8_RAGGED, MX8_MANY], ids=lambda s: s.name)
def test_layer_a8_all_tokens(api, spec):
    _check(api, spec, layer_for(spec), np.arange(spec.T))


def test_layer_a8_full_size_sampled(api):
    """The GPT-OSS-20B-shaped MXFP4 layer (T = 8192): every routing decision, sampled outputs."""
    spec = W.GPTOSS20B_MXFP4
    layer = layer_for(spec)
    lg = O.router_logits(layer["x"], layer["w_router"], layer["b_router"])
    rid, _ = O.topk_softmax(lg, spec.k)
    off, _, sor = O.dispatch(rid, spec.E)
    rng = np.random.default_rng(5)
    toks = np.unique(np.concatenate([[0, spec.T - 1], rng.choice(spec.T, 46, replace=False),
                                     sor[off[0]:off[1]][:16] // spec.k]))
    _check(api, spec, layer, toks)


@pytest.mark.parametrize("spec", [MX8_SMALL, MX8_RAGGED, MX8_MANY, W.GPTOSS20B_MXFP4], ids=lambda s: s.name)
def test_layer_a8_unpacked_weights_match_widened(api, spec):
    """Whole 128-code K blocks of the E2M1 weights through TMA's 4-bit unpacking type (the
    default) against every stage widened by the converter warps (expert-GEMM variant 7): the
    same tiles reach the tensor core, so the outputs agree bit for bit.  K = 128 (all blocks
    unpacked), 192 and 320 (a 64-code tail widened), 64 (no whole block) and 2880."""
    layer = layer_for(spec)
    d = api.upload_layer(layer)
    ew = api.expert_weights_from(d)
    cfg = api.config_from_spec(spec, y_f32=True, wfmt="mxfp4_a8")
    outs = []
    for variant in (0, 7):
        api.set_expert_gemm_variant(variant)
        try:
            outs.append(api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], ew))
            torch.cuda.synchronize()
        finally:
            api.set_expert_gemm_variant(0)
        assert api.last_device_error() == 0
    assert torch.equal(outs[0].view(torch.int32), outs[1].view(torch.int32))


def test_layer_a8_weights_off_32_byte_alignment(api):
    """E2M1 weights 16 bytes past a 32-byte boundary cannot be described to TMA's 4-bit
    unpacking type (it wants 32-byte aligned bases): every stage is then widened by the
    converter warps, and the output is the same bit for bit as with aligned weights."""
    spec = MX8_RAGGED
    layer = layer_for(spec)
    d = api.upload_layer(layer)
    ew = api.expert_weights_from(d)
    cfg = api.config_from_spec(spec, y_f32=True, wfmt="mxfp4_a8")

    def shifted(t):
        buf = torch.empty(t.numel() + 16, dtype=t.dtype, device=t.device)
        v = buf[16:].view(t.shape)
        v.copy_(t)
        assert v.data_ptr() % 32 == 16
        return v

    ew_off = api.ExpertWeights(shifted(ew.w_gate), shifted(ew.w_up), shifted(ew.w_down), ew.b_gate, ew.b_up,
                               ew.b_down, ew.s_gate, ew.s_up, ew.s_down)
    outs = []
    for w in (ew, ew_off):
        outs.append(api.layer_forward(cfg, d["x"], d["w_router"], d["b_router"], w))
        torch.cuda.synchronize()
        assert api.last_device_error() == 0
    assert torch.equal(outs[0].view(torch.int32), outs[1].view(torch.int32))
