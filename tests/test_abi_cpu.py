"""The C-ABI library loads and exports every symbol include/moe.h declares, and
its host-side validation rejects bad arguments before touching the GPU.
No compute call is made here (these run without a GPU)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

from mixture_experts_ffn_12_b200 import _lib, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src, flags=re.M)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding signatures must cover exactly the header"


def test_struct_layout_matches_header():
    assert ctypes.sizeof(_lib.MoeConfig) == 40
    assert _lib.MoeConfig.y_f32.offset == 32
    assert _lib.MoeConfig.h_split.offset == 36
    assert ctypes.sizeof(_lib.MoeExpertWeights) == 9 * ctypes.sizeof(ctypes.c_void_p)
    # int32, float, four pointers, int32 (+ tail padding to pointer alignment)
    assert ctypes.sizeof(_lib.MoeGlmParams) == 48
    assert _lib.MoeGlmParams.e_score_correction_bias.offset == 8
    assert _lib.MoeGlmParams.shared_intermediate_size.offset == 40


def cfg(**kw):
    base = dict(hidden_size=2880, intermediate_size=2880, num_local_experts=32, num_experts_per_tok=4,
                swiglu_limit=7.0, swiglu_alpha=1.702, dtype=_lib.MOE_BF16, wfmt=_lib.MOE_W_DENSE)
    base.update(kw)
    return _lib.MoeConfig(**base)


def test_version_and_status_strings(lib):
    assert lib.moe_abi_version() == 2 == _lib.ABI_VERSION
    for code in range(7):
        assert lib.moe_status_string(code).startswith(b"MOE_")
    assert b"unknown" in lib.moe_status_string(99)


@pytest.mark.parametrize("kw,want", [
    ({}, _lib.MOE_OK),
    (dict(dtype=_lib.MOE_F32, hidden_size=256, intermediate_size=512, num_local_experts=8, num_experts_per_tok=2),
     _lib.MOE_OK),
    (dict(wfmt=_lib.MOE_W_MXFP4), _lib.MOE_OK),
    (dict(wfmt=_lib.MOE_W_MXFP4, dtype=_lib.MOE_F32), _lib.MOE_ERR_UNSUPPORTED),
    (dict(num_experts_per_tok=0), _lib.MOE_ERR_INVALID_ARG),
    (dict(num_experts_per_tok=9, num_local_experts=16), _lib.MOE_ERR_INVALID_ARG),
    (dict(num_experts_per_tok=5, num_local_experts=4), _lib.MOE_ERR_INVALID_ARG),
    (dict(num_local_experts=257), _lib.MOE_ERR_INVALID_ARG),
    (dict(hidden_size=2888), _lib.MOE_ERR_INVALID_ARG),                 # not a multiple of 16
    (dict(wfmt=_lib.MOE_W_MXFP4, intermediate_size=2896), _lib.MOE_ERR_INVALID_ARG),  # not a multiple of 32
    (dict(hidden_size=0), _lib.MOE_ERR_INVALID_ARG),
    (dict(swiglu_limit=0.0), _lib.MOE_ERR_INVALID_ARG),
    (dict(swiglu_limit=float("inf")), _lib.MOE_ERR_INVALID_ARG),
    (dict(swiglu_limit=float("nan")), _lib.MOE_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.MOE_ERR_INVALID_ARG),
    (dict(wfmt=3), _lib.MOE_ERR_INVALID_ARG),
    (dict(y_f32=1), _lib.MOE_OK),
    (dict(y_f32=1, dtype=_lib.MOE_F32), _lib.MOE_OK),
    (dict(y_f32=2), _lib.MOE_ERR_INVALID_ARG),
    (dict(y_f32=-1), _lib.MOE_ERR_INVALID_ARG),
    (dict(h_split=1), _lib.MOE_OK),
    (dict(h_split=1, dtype=_lib.MOE_F32), _lib.MOE_OK),          # fp32 layers keep h in fp32 anyway
    (dict(h_split=1, wfmt=_lib.MOE_W_MXFP4), _lib.MOE_ERR_UNSUPPORTED),
    (dict(h_split=3), _lib.MOE_ERR_INVALID_ARG),
])
def test_config_check(lib, kw, want):
    assert lib.moe_config_check(ctypes.byref(cfg(**kw))) == want


def test_null_config(lib):
    assert lib.moe_config_check(None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_workspace_size(None, 4) == _lib.SIZE_INVALID


def test_workspace_sizes(lib):
    c = cfg()
    assert lib.moe_permute_workspace_size(ctypes.byref(c), 0) == 0
    assert lib.moe_expert_ffn_workspace_size(ctypes.byref(c), 4096) == 0
    T, k, D, F = 4096, 4, 2880, 2880
    ws = lib.moe_workspace_size(ctypes.byref(c), T)
    R = T * k
    # x_perm's region holds the fp32 weighted outputs later (R*D*4), then h, plus maps
    assert ws >= R * D * 4 + R * F * 2 + 4 * R * 4
    assert ws < R * D * 4 + R * F * 2 + 4 * R * 4 + 64 * 1024 * 1024
    assert lib.moe_workspace_size(ctypes.byref(c), -1) == _lib.SIZE_INVALID
    assert lib.moe_workspace_size(ctypes.byref(c), 1 << 30) == _lib.SIZE_INVALID   # T*k >= 2^31
    mx = cfg(wfmt=_lib.MOE_W_MXFP4)
    # MXFP4: the three scale tensors relaid as [E][ceil(K/64)][N][2], 256-byte aligned regions
    E = 32
    gu = -(-(E * (D // 64) * F * 2) // 256) * 256
    dn = -(-(E * (F // 64) * D * 2) // 256) * 256
    assert lib.moe_expert_ffn_workspace_size(ctypes.byref(mx), 8) == 2 * gu + dn
    assert lib.moe_expert_ffn_workspace_size(ctypes.byref(mx), 4096) == 2 * gu + dn


def test_rejections_launch_nothing(lib):
    """Every one of these returns before any CUDA call (no GPU here)."""
    c = cfg()
    p = ctypes.c_void_p(0x10000)        # aligned, never dereferenced
    bad = ctypes.c_void_p(0x10008)      # misaligned
    assert lib.moe_router_topk(ctypes.byref(c), 0, None, None, None, None, None, None) == _lib.MOE_OK
    assert lib.moe_router_topk(ctypes.byref(c), 8, None, p, p, p, p, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_router_topk(ctypes.byref(c), 8, bad, p, p, p, p, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_router_topk(ctypes.byref(c), -1, p, p, p, p, p, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_router_topk(None, 8, p, p, p, p, p, None) == _lib.MOE_ERR_INVALID_ARG
    # permute: workspace too small, x without x_perm
    assert lib.moe_permute(ctypes.byref(c), 8, p, p, p, p, p, p, p, 0, None) == _lib.MOE_ERR_WORKSPACE
    assert lib.moe_permute(ctypes.byref(c), 8, p, p, p, p, p, None, p, 1 << 20, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(ctypes.byref(c), 8, p, p, None, p, p, p, p, 1 << 20, None) == _lib.MOE_ERR_INVALID_ARG
    w = _lib.MoeExpertWeights(*([0x10000] * 3 + [None] * 3 + [0x10000] * 3))
    assert lib.moe_expert_ffn(ctypes.byref(c), 8, p, p, None, p, p, None, 0, None) == _lib.MOE_ERR_INVALID_ARG
    # MXFP4 needs its scale tensors
    mx = cfg(wfmt=_lib.MOE_W_MXFP4)
    assert lib.moe_expert_ffn(ctypes.byref(mx), 8, p, p, ctypes.byref(w), p, p, None, 0, None) == \
        _lib.MOE_ERR_INVALID_ARG
    wmx = _lib.MoeExpertWeights(*([0x10000] * 5 + [0x10008] + [0x10000] * 3))   # misaligned s_down
    assert lib.moe_expert_ffn(ctypes.byref(mx), 8, p, p, ctypes.byref(wmx), p, p, None, 0, None) == \
        _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(ctypes.byref(c), 8, p, None, p, p, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_forward(ctypes.byref(c), 8, p, p, p, ctypes.byref(w), p, None, None, p, 10, None) == \
        _lib.MOE_ERR_WORKSPACE
    assert lib.moe_layer_forward(ctypes.byref(c), 8, p, p, p, None, p, None, None, p, 1 << 40, None) == \
        _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_forward(ctypes.byref(c), 0, None, None, None, None, None, None, None, None, 0, None) == \
        _lib.MOE_OK


def test_h_split_workspace_and_variant_check(lib):
    """h in two bf16 halves doubles the h region of the workspace; the weights-in-M pair
    kernels have no such form, and the call says so before launching anything."""
    T, k, F = 4096, 4, 2880
    c, cs = cfg(), cfg(h_split=1)
    assert lib.moe_workspace_size(ctypes.byref(cs), T) - lib.moe_workspace_size(ctypes.byref(c), T) == T * k * F * 2
    c32, c32s = cfg(dtype=_lib.MOE_F32), cfg(dtype=_lib.MOE_F32, h_split=1)
    assert lib.moe_workspace_size(ctypes.byref(c32), T) == lib.moe_workspace_size(ctypes.byref(c32s), T)
    p = ctypes.c_void_p(0x10000)
    w = _lib.MoeExpertWeights(*([0x10000] * 3 + [None] * 3 + [0x10000] * 3))
    assert lib.moe_set_expert_gemm_variant(4) == _lib.MOE_OK
    try:
        assert lib.moe_layer_forward(ctypes.byref(cs), 8, p, p, p, ctypes.byref(w), p, None, None, p, 1 << 40,
                                     None) == _lib.MOE_ERR_UNSUPPORTED
        assert lib.moe_expert_ffn(ctypes.byref(cs), 8, p, p, ctypes.byref(w), p, p, None, 0, None) == \
            _lib.MOE_ERR_UNSUPPORTED
    finally:
        assert lib.moe_set_expert_gemm_variant(0) == _lib.MOE_OK


def test_block_scaled_variant_checks(lib):
    """MXFP4 weights with MXFP8 activations: bf16 layers, D and F multiples of 32, no h_split,
    moe_layer_forward only; the quantizer's argument checks; all before any launch."""
    a8 = _lib.MOE_W_MXFP4_A8
    assert lib.moe_config_check(ctypes.byref(cfg(wfmt=a8))) == _lib.MOE_OK
    assert lib.moe_config_check(ctypes.byref(cfg(wfmt=a8, hidden_size=2880 - 32))) == _lib.MOE_OK
    assert lib.moe_config_check(ctypes.byref(cfg(wfmt=a8, hidden_size=2880 - 16))) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_config_check(ctypes.byref(cfg(wfmt=a8, dtype=_lib.MOE_F32))) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_config_check(ctypes.byref(cfg(wfmt=a8, h_split=1))) == _lib.MOE_ERR_UNSUPPORTED
    p = ctypes.c_void_p(0x10000)
    w = _lib.MoeExpertWeights(*([0x10000] * 9))
    assert lib.moe_expert_ffn(ctypes.byref(cfg(wfmt=a8)), 8, p, p, ctypes.byref(w), p, p, None, 0, None) == \
        _lib.MOE_ERR_UNSUPPORTED
    w8 = _lib.MoeExpertWeights(*([0x10008] + [0x10000] * 8))       # codes not 16-byte aligned
    assert lib.moe_layer_forward(ctypes.byref(cfg(wfmt=a8)), 8, p, p, p, ctypes.byref(w8), p, None, None, p,
                                 1 << 40, None) == _lib.MOE_ERR_INVALID_ARG
    c, big = cfg(wfmt=a8), 1 << 40
    assert lib.moe_workspace_size(ctypes.byref(c), 8192) != _lib.SIZE_INVALID
    assert lib.moe_mxfp8_scale_stride(2880) == 96 and lib.moe_mxfp8_scale_stride(32) == 16
    assert lib.moe_quantize_mxfp8(0, 2880, None, None, None, None) == _lib.MOE_OK
    assert lib.moe_quantize_mxfp8(4, 2880 + 16, p, p, p, None) == _lib.MOE_ERR_INVALID_ARG   # K % 32
    assert lib.moe_quantize_mxfp8(4, 2880, p, None, p, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_quantize_mxfp8(-1, 2880, p, p, p, None) == _lib.MOE_ERR_INVALID_ARG
    assert big > 0


def glm_params(**kw):
    base = dict(norm_topk_prob=1, routed_scaling_factor=2.5, e_score_correction_bias=None, ws_gate=None,
                ws_up=None, ws_down=None, shared_intermediate_size=0)
    base.update(kw)
    return _lib.MoeGlmParams(**base)


def test_glm_workspace_sizes(lib):
    c = cfg()
    T, k, D, F, E = 4096, 4, 2880, 2880, 32
    R = T * k
    assert lib.moe_glm_router_workspace_size(ctypes.byref(c), T) == 4 * T * E * 4
    base = lib.moe_glm_workspace_size(ctypes.byref(c), ctypes.byref(glm_params()), T)
    # as the GPT-OSS layer (maps, x_perm / fp32 rows, h) plus E * max(F, D) zero biases
    assert base >= R * D * 4 + R * F * 2 + 4 * R * 4 + E * F * 2
    assert base < R * D * 4 + R * F * 2 + 4 * R * 4 + E * F * 2 + 64 * 1024 * 1024
    p = ctypes.c_void_p(0x10000).value
    shared = glm_params(ws_gate=p, ws_up=p, ws_down=p, shared_intermediate_size=1408)
    # a shared expert adds its offsets, identity slots and unit weights [T], [T, Fs] in bf16
    # and its fp32 output rows [T, D]
    extra = lib.moe_glm_workspace_size(ctypes.byref(c), ctypes.byref(shared), T) - base
    want = T * 4 * 2 + T * 1408 * 2 + T * D * 4
    assert want <= extra <= want + 6 * 256
    assert lib.moe_glm_workspace_size(ctypes.byref(c), None, T) == _lib.SIZE_INVALID
    assert lib.moe_glm_workspace_size(ctypes.byref(c), ctypes.byref(glm_params(shared_intermediate_size=24)), T) \
        == _lib.SIZE_INVALID
    assert lib.moe_glm_workspace_size(ctypes.byref(cfg(wfmt=_lib.MOE_W_MXFP4)), ctypes.byref(glm_params()), T) \
        == _lib.SIZE_INVALID


def test_glm_rejections_launch_nothing(lib):
    """The variant's calls return before any CUDA call on bad arguments (no GPU here)."""
    c = cfg()
    gp = glm_params()
    p = ctypes.c_void_p(0x10000)
    bad = ctypes.c_void_p(0x10008)
    w = _lib.MoeExpertWeights(*([0x10000] * 3 + [None] * 6))       # the variant's experts have no biases
    big = 1 << 40
    fwd = lib.moe_glm_layer_forward
    assert fwd(ctypes.byref(c), ctypes.byref(gp), 0, None, None, None, None, None, None, None, 0, None) == _lib.MOE_OK
    assert fwd(ctypes.byref(c), None, 8, p, p, ctypes.byref(w), p, None, None, p, big, None) == \
        _lib.MOE_ERR_INVALID_ARG
    assert fwd(ctypes.byref(cfg(wfmt=_lib.MOE_W_MXFP4)), ctypes.byref(gp), 8, p, p, ctypes.byref(w), p, None, None,
               p, big, None) == _lib.MOE_ERR_UNSUPPORTED
    assert fwd(ctypes.byref(c), ctypes.byref(glm_params(routed_scaling_factor=float("nan"))), 8, p, p,
               ctypes.byref(w), p, None, None, p, big, None) == _lib.MOE_ERR_INVALID_ARG
    assert fwd(ctypes.byref(c), ctypes.byref(gp), 8, bad, p, ctypes.byref(w), p, None, None, p, big, None) == \
        _lib.MOE_ERR_INVALID_ARG
    assert fwd(ctypes.byref(c), ctypes.byref(gp), 8, p, p, None, p, None, None, p, big, None) == \
        _lib.MOE_ERR_INVALID_ARG
    # a shared expert needs its three matrices
    sh = glm_params(ws_gate=0x10000, ws_up=None, ws_down=0x10000, shared_intermediate_size=64)
    assert fwd(ctypes.byref(c), ctypes.byref(sh), 8, p, p, ctypes.byref(w), p, None, None, p, big, None) == \
        _lib.MOE_ERR_INVALID_ARG
    # misaligned correction bias
    cb = glm_params(e_score_correction_bias=0x10004)
    assert fwd(ctypes.byref(c), ctypes.byref(cb), 8, p, p, ctypes.byref(w), p, None, None, p, big, None) == \
        _lib.MOE_ERR_INVALID_ARG
    assert fwd(ctypes.byref(c), ctypes.byref(gp), 8, p, p, ctypes.byref(w), p, None, None, p, 10, None) == \
        _lib.MOE_ERR_WORKSPACE
    rt = lib.moe_glm_router_topk
    assert rt(ctypes.byref(c), ctypes.byref(gp), 0, None, None, None, None, None, 0, None) == _lib.MOE_OK
    assert rt(ctypes.byref(c), ctypes.byref(gp), 8, p, p, p, p, p, 16, None) == _lib.MOE_ERR_WORKSPACE
    assert rt(ctypes.byref(c), ctypes.byref(gp), 8, p, None, p, p, p, big, None) == _lib.MOE_ERR_INVALID_ARG
