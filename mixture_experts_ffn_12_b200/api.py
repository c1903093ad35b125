"""Python binding of libmoe: argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module turns
torch CUDA tensors into the pointers and sizes of the C ABI (include/moe.h),
allocates outputs and workspaces with torch, and passes torch's current
stream.  There is no fallback: without the library or a CUDA device the calls
raise.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Dict, Optional, Tuple

import numpy as np
import torch

from . import _lib
from ._lib import MoeConfig, MoeExpertWeights


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {_lib.status_string(code)}" if what else _lib.status_string(code))


def _check(code: int, what: str) -> None:
    if code != _lib.MOE_OK:
        raise MoeError(code, what)


_DT = {"bf16": (_lib.MOE_BF16, torch.bfloat16), "f32": (_lib.MOE_F32, torch.float32)}
# expert-weight formats: dense, MXFP4 (decoded to bf16 in the GEMM mainloop), MXFP4 with MXFP8
# activations on the block-scaled tensor cores
_WF = {"dense": _lib.MOE_W_DENSE, "mxfp4": _lib.MOE_W_MXFP4, "mxfp4_a8": _lib.MOE_W_MXFP4_A8}


def make_config(hidden_size: int, intermediate_size: int, num_local_experts: int, num_experts_per_tok: int,
                swiglu_limit: float = 7.0, swiglu_alpha: float = 1.702, dtype: str = "bf16",
                wfmt: str = "dense", y_f32: bool = False, h_split: bool = False) -> MoeConfig:
    """y_f32: the layer output y is stored in fp32 (the sums before their rounding to dtype).
    h_split: the SwiGLU output is kept as two bf16 halves (hi + lo) between the expert GEMMs."""
    return MoeConfig(hidden_size, intermediate_size, num_local_experts, num_experts_per_tok, swiglu_limit,
                     swiglu_alpha, _DT[dtype][0], _WF[wfmt], 1 if y_f32 else 0, 1 if h_split else 0)


def config_from_spec(spec, y_f32: bool = False, h_split: bool = False, wfmt: Optional[str] = None) -> MoeConfig:
    """Config of a ``workloads.LayerSpec``; `wfmt` overrides the spec's weight format (the MXFP4
    weights of a spec also run as "mxfp4_a8")."""
    return make_config(spec.D, spec.F, spec.E, spec.k, spec.limit, spec.alpha, spec.dtype, wfmt or spec.wfmt,
                       y_f32, h_split)


def torch_dtype(cfg: MoeConfig) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == _lib.MOE_BF16 else torch.float32


def out_dtype(cfg: MoeConfig) -> torch.dtype:
    """dtype of the layer output y: fp32 when cfg.y_f32 is set, else the layer dtype."""
    return torch.float32 if cfg.y_f32 else torch_dtype(cfg)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmoe takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


# --------------------------------------------------------------------------- #
# argument checks: the C ABI sees pointers only, so shapes and dtypes are checked
# here, against the layouts include/moe.h documents, before any pointer is passed
# (a bf16 buffer passed where fp32 is declared would be read past its end).
# These checks touch no device and run on CPU tensors too.
# --------------------------------------------------------------------------- #
def _want(name: str, t: Optional[torch.Tensor], shape, dtype: torch.dtype,
          device: Optional[torch.device] = None) -> None:
    if t is None:
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _rows(name: str, t: Optional[torch.Tensor]) -> int:
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dim() == 0:
        raise ValueError(f"{name} must have a leading token dimension")
    return int(t.shape[0])


def check_expert_weights(cfg: MoeConfig, w: "ExpertWeights", device: Optional[torch.device] = None) -> None:
    """Dense: W_g, W_u [E, F, D], W_d [E, D, F] in the layer dtype.  MXFP4: packed E2M1
    codes [E, F, D/2], [E, F, D/2], [E, D, F/2] and E8M0 scales [E, F, D/32], [E, F, D/32],
    [E, D, F/32], all uint8.  Biases [E, F], [E, F], [E, D] in the layer dtype."""
    D, F, E = cfg.hidden_size, cfg.intermediate_size, cfg.num_local_experts
    dt = torch_dtype(cfg)
    if cfg.wfmt in (_lib.MOE_W_MXFP4, _lib.MOE_W_MXFP4_A8):
        if D % 32 or F % 32:
            raise ValueError(f"MXFP4 weights need D and F divisible by 32 (D={D}, F={F})")
        _want("w_gate", w.w_gate, (E, F, D // 2), torch.uint8, device)
        _want("w_up", w.w_up, (E, F, D // 2), torch.uint8, device)
        _want("w_down", w.w_down, (E, D, F // 2), torch.uint8, device)
        _want("s_gate", w.s_gate, (E, F, D // 32), torch.uint8, device)
        _want("s_up", w.s_up, (E, F, D // 32), torch.uint8, device)
        _want("s_down", w.s_down, (E, D, F // 32), torch.uint8, device)
    else:
        _want("w_gate", w.w_gate, (E, F, D), dt, device)
        _want("w_up", w.w_up, (E, F, D), dt, device)
        _want("w_down", w.w_down, (E, D, F), dt, device)
    _want("b_gate", w.b_gate, (E, F), dt, device)
    _want("b_up", w.b_up, (E, F), dt, device)
    _want("b_down", w.b_down, (E, D), dt, device)


def check_router_args(cfg: MoeConfig, x, w_router, b_router, topk_ids=None, topk_w=None) -> int:
    """x [T, D], W_r [E, D], b_r [E] in the layer dtype; topk_ids [T, k] int32 and
    topk_w [T, k] fp32 when given.  Returns T."""
    D, E, k = cfg.hidden_size, cfg.num_local_experts, cfg.num_experts_per_tok
    dt = torch_dtype(cfg)
    T = _rows("x", x)
    _want("x", x, (T, D), dt)
    _want("w_router", w_router, (E, D), dt, x.device)
    _want("b_router", b_router, (E,), dt, x.device)
    if topk_ids is not None:
        _want("topk_ids", topk_ids, (T, k), torch.int32, x.device)
    if topk_w is not None:
        _want("topk_w", topk_w, (T, k), torch.float32, x.device)
    return T


def check_permute_args(cfg: MoeConfig, topk_ids, x=None) -> int:
    """topk_ids [T, k] int32; x [T, D] in the layer dtype when given.  Returns T."""
    T = _rows("topk_ids", topk_ids)
    _want("topk_ids", topk_ids, (T, cfg.num_experts_per_tok), torch.int32)
    if x is not None:
        _want("x", x, (T, cfg.hidden_size), torch_dtype(cfg), topk_ids.device)
    return T


def check_expert_ffn_args(cfg: MoeConfig, x_perm, expert_off, weights: "ExpertWeights") -> int:
    """x_perm [R, D] in the layer dtype with R = T·k; expert_off [E+1] int32.  Returns T."""
    R, k = _rows("x_perm", x_perm), cfg.num_experts_per_tok
    if R % k:
        raise ValueError(f"x_perm has {R} rows, not a multiple of k = {k}")
    _want("x_perm", x_perm, (R, cfg.hidden_size), torch_dtype(cfg))
    _want("expert_off", expert_off, (cfg.num_local_experts + 1,), torch.int32, x_perm.device)
    check_expert_weights(cfg, weights, x_perm.device)
    return R // k


def check_combine_args(cfg: MoeConfig, y_perm, row_of_slot, topk_w) -> int:
    """y_perm [T·k, D] in the layer dtype; row_of_slot [T, k] int32; topk_w [T, k] fp32.  Returns T."""
    k = cfg.num_experts_per_tok
    T = _rows("row_of_slot", row_of_slot)
    _want("row_of_slot", row_of_slot, (T, k), torch.int32)
    _want("y_perm", y_perm, (T * k, cfg.hidden_size), torch_dtype(cfg), row_of_slot.device)
    _want("topk_w", topk_w, (T, k), torch.float32, row_of_slot.device)
    return T


def check_layer_args(cfg: MoeConfig, x, w_router, b_router, weights: Optional["ExpertWeights"], y=None,
                     topk_ids=None, topk_w=None) -> int:
    """The router's arguments, the expert weights (skipped when None: already checked)
    and y [T, D] in the output dtype (``out_dtype``) when given.  Returns T."""
    T = check_router_args(cfg, x, w_router, b_router, topk_ids, topk_w)
    if weights is not None:
        check_expert_weights(cfg, weights, x.device)
    if y is not None:
        _want("y", y, (T, cfg.hidden_size), out_dtype(cfg), x.device)
    return T


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


@dataclasses.dataclass
class ExpertWeights:
    """Device expert parameters: dense (dtype) or MXFP4 (uint8 codes + E8M0 scales)."""
    w_gate: torch.Tensor
    w_up: torch.Tensor
    w_down: torch.Tensor
    b_gate: torch.Tensor
    b_up: torch.Tensor
    b_down: torch.Tensor
    s_gate: Optional[torch.Tensor] = None
    s_up: Optional[torch.Tensor] = None
    s_down: Optional[torch.Tensor] = None

    def c_struct(self) -> MoeExpertWeights:
        return MoeExpertWeights(*(None if t is None else t.data_ptr() for t in (
            self.w_gate, self.w_up, self.w_down, self.s_gate, self.s_up, self.s_down,
            self.b_gate, self.b_up, self.b_down)))


def to_torch(a: np.ndarray) -> torch.Tensor:
    """Host array from ``workloads`` -> torch CPU tensor (uint16 bits -> bfloat16)."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a))


def upload_layer(layer: Dict[str, np.ndarray], device="cuda") -> Dict[str, torch.Tensor]:
    return {k: to_torch(v).to(device) for k, v in layer.items()}


def expert_weights_from(d: Dict[str, torch.Tensor]) -> ExpertWeights:
    return ExpertWeights(d["w_gate"], d["w_up"], d["w_down"], d["b_gate"], d["b_up"], d["b_down"],
                         d.get("s_gate"), d.get("s_up"), d.get("s_down"))


# --------------------------------------------------------------------------- #
# the five calls (each on torch's current stream of the tensors' device)
# --------------------------------------------------------------------------- #
def _size(n: int, what: str) -> int:
    if n == _lib.SIZE_INVALID:
        raise MoeError(_lib.MOE_ERR_INVALID_ARG, what)
    return n


def router_topk(cfg: MoeConfig, x: torch.Tensor, w_router: torch.Tensor, b_router: torch.Tensor,
                topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None
                ) -> Tuple[torch.Tensor, torch.Tensor]:
    T = check_router_args(cfg, x, w_router, b_router, topk_ids, topk_w)
    k = cfg.num_experts_per_tok
    if topk_ids is None:
        topk_ids = torch.empty((T, k), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        _check(_lib.load().moe_router_topk(ctypes.byref(cfg), T, _p(x), _p(w_router), _p(b_router), _p(topk_ids),
                                           _p(topk_w), _stream(x.device)), "moe_router_topk")
    return topk_ids, topk_w


def permute(cfg: MoeConfig, topk_ids: torch.Tensor, x: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    T = check_permute_args(cfg, topk_ids, x)
    L = _lib.load()
    k, dev = cfg.num_experts_per_tok, topk_ids.device
    R = T * k
    out = dict(
        expert_off=torch.empty(cfg.num_local_experts + 1, dtype=torch.int32, device=dev),
        row_of_slot=torch.empty((T, k), dtype=torch.int32, device=dev),
        slot_of_row=torch.empty(R, dtype=torch.int32, device=dev),
    )
    out["x_perm"] = None if x is None else torch.empty((R, cfg.hidden_size), dtype=x.dtype, device=dev)
    nws = _size(L.moe_permute_workspace_size(ctypes.byref(cfg), T), "moe_permute_workspace_size")
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(L.moe_permute(ctypes.byref(cfg), T, _p(topk_ids), _p(x), _p(out["expert_off"]),
                             _p(out["row_of_slot"]), _p(out["slot_of_row"]), _p(out["x_perm"]), _p(ws), ws.numel(),
                             _stream(dev)), "moe_permute")
    return out


def expert_ffn(cfg: MoeConfig, x_perm: torch.Tensor, expert_off: torch.Tensor, weights: ExpertWeights
               ) -> Tuple[torch.Tensor, torch.Tensor]:
    T = check_expert_ffn_args(cfg, x_perm, expert_off, weights)
    L = _lib.load()
    R, dev = x_perm.shape[0], x_perm.device
    dt = torch_dtype(cfg)
    # with h_split (bf16) each row of h holds the bf16 halves hi and lo: [R, 2, F]
    halves = 2 if (cfg.h_split and cfg.dtype == _lib.MOE_BF16) else 1
    h = torch.empty((R, halves * cfg.intermediate_size), dtype=dt, device=dev)
    y_perm = torch.empty((R, cfg.hidden_size), dtype=dt, device=dev)
    nws = _size(L.moe_expert_ffn_workspace_size(ctypes.byref(cfg), T), "moe_expert_ffn_workspace_size")
    ws = torch.empty(nws, dtype=torch.uint8, device=dev) if nws else None
    ws_struct = weights.c_struct()
    with torch.cuda.device(dev):
        _check(L.moe_expert_ffn(ctypes.byref(cfg), T, _p(x_perm), _p(expert_off), ctypes.byref(ws_struct), _p(h),
                                _p(y_perm), _p(ws), nws, _stream(dev)), "moe_expert_ffn")
    return h, y_perm


def combine(cfg: MoeConfig, y_perm: torch.Tensor, row_of_slot: torch.Tensor, topk_w: torch.Tensor) -> torch.Tensor:
    T = check_combine_args(cfg, y_perm, row_of_slot, topk_w)
    dev = y_perm.device
    y = torch.empty((T, cfg.hidden_size), dtype=out_dtype(cfg), device=dev)
    with torch.cuda.device(dev):
        _check(_lib.load().moe_combine(ctypes.byref(cfg), T, _p(y_perm), _p(row_of_slot), _p(topk_w), _p(y),
                                       _stream(dev)), "moe_combine")
    return y


def workspace_size(cfg: MoeConfig, T: int) -> int:
    return _size(_lib.load().moe_workspace_size(ctypes.byref(cfg), T), "moe_workspace_size")


def layer_forward(cfg: MoeConfig, x: torch.Tensor, w_router: torch.Tensor, b_router: torch.Tensor,
                  weights: ExpertWeights, y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                  topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                  _weights_checked: bool = False) -> torch.Tensor:
    T = check_layer_args(cfg, x, w_router, b_router, None if _weights_checked else weights, y, topk_ids, topk_w)
    dev = x.device
    if y is None:
        y = torch.empty((T, cfg.hidden_size), dtype=out_dtype(cfg), device=dev)
    if ws is None:
        ws = torch.empty(max(workspace_size(cfg, T), 16), dtype=torch.uint8, device=dev)
    elif ws.device != dev:
        raise ValueError(f"ws is on {ws.device}, expected {dev}")
    wst = weights.c_struct()
    with torch.cuda.device(dev):
        _check(_lib.load().moe_layer_forward(ctypes.byref(cfg), T, _p(x), _p(w_router), _p(b_router),
                                             ctypes.byref(wst), _p(y), _p(topk_ids), _p(topk_w), _p(ws),
                                             ws.numel() * ws.element_size(), _stream(dev)), "moe_layer_forward")
    return y


# --------------------------------------------------------------------------- #
# the GLM4-MoE-Lite variant (moe_glm_*)
# --------------------------------------------------------------------------- #
@dataclasses.dataclass
class GlmParams:
    """Router and shared-expert parameters of the GLM4-MoE-Lite variant (moe_glm_params_t):
    e_score_correction_bias [E] and the shared expert ws_gate / ws_up [Fs, D], ws_down [D, Fs],
    all in the layer dtype and optional."""
    norm_topk_prob: bool = True
    routed_scaling_factor: float = 1.0
    e_score_correction_bias: Optional[torch.Tensor] = None
    ws_gate: Optional[torch.Tensor] = None
    ws_up: Optional[torch.Tensor] = None
    ws_down: Optional[torch.Tensor] = None

    @property
    def shared_intermediate_size(self) -> int:
        return 0 if self.ws_gate is None else int(self.ws_gate.shape[0])

    def c_struct(self) -> _lib.MoeGlmParams:
        ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        return _lib.MoeGlmParams(1 if self.norm_topk_prob else 0, float(self.routed_scaling_factor),
                                 ptr(self.e_score_correction_bias), ptr(self.ws_gate), ptr(self.ws_up),
                                 ptr(self.ws_down), self.shared_intermediate_size)


def glm_params_from(spec, d: Dict[str, torch.Tensor]) -> GlmParams:
    """Parameters of a ``workloads.GlmLayerSpec`` layer uploaded with ``upload_layer``."""
    return GlmParams(spec.norm_topk_prob, spec.routed_scaling_factor, d.get("e_score_correction_bias"),
                     d.get("ws_gate"), d.get("ws_up"), d.get("ws_down"))


def glm_expert_weights_from(d: Dict[str, torch.Tensor]) -> ExpertWeights:
    """The variant's expert weights (no biases)."""
    return ExpertWeights(d["w_gate"], d["w_up"], d["w_down"], None, None, None)


def glm_config_from_spec(spec, y_f32: bool = False, h_split: bool = False) -> MoeConfig:
    """Config of a ``workloads.GlmLayerSpec`` (the SwiGLU limit and alpha are not used by the variant)."""
    return make_config(spec.D, spec.F, spec.E, spec.k, dtype=spec.dtype, y_f32=y_f32, h_split=h_split)


def check_glm_args(cfg: MoeConfig, params: GlmParams, x, w_router, weights: Optional[ExpertWeights] = None,
                   y=None, topk_ids=None, topk_w=None) -> int:
    """x [T, D], W_r [E, D], e_score_correction_bias [E], the shared expert (all three or none:
    [Fs, D], [Fs, D], [D, Fs]) and, when given, the expert weights (dense, no biases) and
    y [T, D], in the layer dtype; topk_ids [T, k] int32 and topk_w [T, k] fp32.  Returns T."""
    D, F, E, k = cfg.hidden_size, cfg.intermediate_size, cfg.num_local_experts, cfg.num_experts_per_tok
    dt = torch_dtype(cfg)
    if cfg.wfmt != _lib.MOE_W_DENSE:
        raise ValueError("the GLM4-MoE-Lite variant takes dense expert weights")
    T = _rows("x", x)
    dev = x.device
    _want("x", x, (T, D), dt)
    _want("w_router", w_router, (E, D), dt, dev)
    if params.e_score_correction_bias is not None:
        _want("e_score_correction_bias", params.e_score_correction_bias, (E,), dt, dev)
    shared = [params.ws_gate, params.ws_up, params.ws_down]
    if any(t is not None for t in shared):
        Fs = _rows("ws_gate", params.ws_gate)
        _want("ws_gate", params.ws_gate, (Fs, D), dt, dev)
        _want("ws_up", params.ws_up, (Fs, D), dt, dev)
        _want("ws_down", params.ws_down, (D, Fs), dt, dev)
    if weights is not None:
        _want("w_gate", weights.w_gate, (E, F, D), dt, dev)
        _want("w_up", weights.w_up, (E, F, D), dt, dev)
        _want("w_down", weights.w_down, (E, D, F), dt, dev)
    if y is not None:
        _want("y", y, (T, D), out_dtype(cfg), dev)
    if topk_ids is not None:
        _want("topk_ids", topk_ids, (T, k), torch.int32, dev)
    if topk_w is not None:
        _want("topk_w", topk_w, (T, k), torch.float32, dev)
    return T


def glm_router_topk(cfg: MoeConfig, params: GlmParams, x: torch.Tensor, w_router: torch.Tensor,
                    topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None
                    ) -> Tuple[torch.Tensor, torch.Tensor]:
    T = check_glm_args(cfg, params, x, w_router, topk_ids=topk_ids, topk_w=topk_w)
    L = _lib.load()
    k, dev = cfg.num_experts_per_tok, x.device
    if topk_ids is None:
        topk_ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    nws = _size(L.moe_glm_router_workspace_size(ctypes.byref(cfg), T), "moe_glm_router_workspace_size")
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    gp = params.c_struct()
    with torch.cuda.device(dev):
        _check(L.moe_glm_router_topk(ctypes.byref(cfg), ctypes.byref(gp), T, _p(x), _p(w_router), _p(topk_ids),
                                     _p(topk_w), _p(ws), ws.numel(), _stream(dev)), "moe_glm_router_topk")
    return topk_ids, topk_w


def glm_workspace_size(cfg: MoeConfig, params: GlmParams, T: int) -> int:
    gp = params.c_struct()
    return _size(_lib.load().moe_glm_workspace_size(ctypes.byref(cfg), ctypes.byref(gp), T), "moe_glm_workspace_size")


def glm_layer_forward(cfg: MoeConfig, params: GlmParams, x: torch.Tensor, w_router: torch.Tensor,
                      weights: ExpertWeights, y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                      topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None
                      ) -> torch.Tensor:
    T = check_glm_args(cfg, params, x, w_router, weights, y, topk_ids, topk_w)
    dev = x.device
    if y is None:
        y = torch.empty((T, cfg.hidden_size), dtype=out_dtype(cfg), device=dev)
    if ws is None:
        ws = torch.empty(max(glm_workspace_size(cfg, params, T), 16), dtype=torch.uint8, device=dev)
    elif ws.device != dev:
        raise ValueError(f"ws is on {ws.device}, expected {dev}")
    wst = weights.c_struct()
    gp = params.c_struct()
    with torch.cuda.device(dev):
        _check(_lib.load().moe_glm_layer_forward(ctypes.byref(cfg), ctypes.byref(gp), T, _p(x), _p(w_router),
                                                 ctypes.byref(wst), _p(y), _p(topk_ids), _p(topk_w), _p(ws),
                                                 ws.numel() * ws.element_size(), _stream(dev)),
               "moe_glm_layer_forward")
    return y


def quantize_mxfp8(x: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """x [rows, K] bf16 -> (E4M3 codes [rows, K] uint8, E8M0 scale rows [rows, stride] uint8)."""
    if x.dim() != 2 or x.dtype != torch.bfloat16:
        raise ValueError("quantize_mxfp8 takes a 2-D bf16 tensor")
    L = _lib.load()
    rows, K = x.shape
    stride = L.moe_mxfp8_scale_stride(K)
    xq = torch.empty((rows, K), dtype=torch.uint8, device=x.device)
    sf = torch.empty((rows, max(stride, 1)), dtype=torch.uint8, device=x.device)
    with torch.cuda.device(x.device):
        _check(L.moe_quantize_mxfp8(rows, K, _p(x), _p(xq), _p(sf), _stream(x.device)), "moe_quantize_mxfp8")
    return xq, sf


def last_device_error() -> int:
    """Reads and clears the device error word (synchronises); returns a status code."""
    return _lib.load().moe_last_device_error()


def set_expert_gemm_variant(variant: int) -> None:
    """Expert-GEMM kernel choice for bf16 dense weights: 0 = by size (the default), 1 = single-CTA
    128-row tiles, 2 = CTA-pair 256-row tiles, 3 = the weight-stationary decode kernel,
    4 = CTA pairs with the weights in M, 5 = layer_forward as the two-kernel decode layer
    wherever it applies, 6 = by size with the layer's gate/up rows gathered from x (TMA gather4)
    rather than read from x_perm, 7 = by size, with the MXFP4 x MXFP8 GEMMs widening every E2M1
    stage in their converter warps (no TMA 4-bit unpacking).  Process-wide; other MXFP4 layers
    ignore it."""
    _check(_lib.load().moe_set_expert_gemm_variant(variant), "moe_set_expert_gemm_variant")


def set_wait_limit_ns(ns: int) -> None:
    _lib.load().moe_set_wait_limit_ns(ns)


class MoELayer:
    """A GPT-OSS MoE FFN layer resident on one GPU: weights, config and a reusable workspace."""

    def __init__(self, cfg: MoeConfig, w_router: torch.Tensor, b_router: torch.Tensor, experts: ExpertWeights):
        _check(_lib.load().moe_config_check(ctypes.byref(cfg)), "moe_config_check")
        check_expert_weights(cfg, experts, w_router.device)
        self.cfg, self.w_router, self.b_router, self.experts = cfg, w_router, b_router, experts
        self._ws: Optional[torch.Tensor] = None

    def workspace(self, T: int) -> torch.Tensor:
        n = max(workspace_size(self.cfg, T), 16)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, dtype=torch.uint8, device=self.w_router.device)
        return self._ws

    def __call__(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, topk_ids=None, topk_w=None) -> torch.Tensor:
        return layer_forward(self.cfg, x, self.w_router, self.b_router, self.experts, y=y,
                             ws=self.workspace(_rows("x", x)), topk_ids=topk_ids, topk_w=topk_w,
                             _weights_checked=True)

    def graphed(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, topk_ids=None, topk_w=None):
        """Capture one forward on these fixed buffers into a CUDA graph; returns (replay, y).

        The library makes no host synchronisation and allocates nothing, so its
        launches are captured as they are; ``replay()`` re-runs them on whatever
        ``x`` holds at that time.  Removes host launch overhead (decode sizes).
        """
        if y is None:
            y = torch.empty((x.shape[0], self.cfg.hidden_size), dtype=out_dtype(self.cfg), device=x.device)
        ws = self.workspace(x.shape[0])
        self(x, y=y, topk_ids=topk_ids, topk_w=topk_w)          # warm: per-device set-up outside capture
        torch.cuda.synchronize(x.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer_forward(self.cfg, x, self.w_router, self.b_router, self.experts, y=y, ws=ws,
                          topk_ids=topk_ids, topk_w=topk_w, _weights_checked=True)
        return g.replay, y

    def run_host_batches(self, xs_host, ys_host) -> None:
        """Run the layer on a sequence of pinned host batches, results into pinned host buffers.

        Batch i's host->device copy, forward and device->host copy go on three
        streams with two device buffers each way, so the copies of neighbouring
        batches overlap this batch's forward (PCIe is full duplex).  Ordering:
        copy-in(i) after forward(i-2) released its input buffer; forward(i) after
        copy-in(i) and after copy-out(i-2) released its output buffer; copy-out(i)
        after forward(i).  Returns when everything has been queued; the caller
        synchronises.  All batches must have the same shape.
        """
        if len(xs_host) == 0:
            return
        dev = self.w_router.device
        T, D = xs_host[0].shape
        xd = [torch.empty((T, D), dtype=xs_host[0].dtype, device=dev) for _ in range(2)]
        yd = [torch.empty((T, self.cfg.hidden_size), dtype=out_dtype(self.cfg), device=dev) for _ in range(2)]
        s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        cur = torch.cuda.current_stream(dev)
        for st in (s_in, s_run, s_out):
            st.wait_stream(cur)
        copied = [torch.cuda.Event() for _ in range(2)]
        ran = [torch.cuda.Event() for _ in range(2)]
        drained = [torch.cuda.Event() for _ in range(2)]
        self.workspace(T)
        for i, (xh, yh) in enumerate(zip(xs_host, ys_host)):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ran[b])
                xd[b].copy_(xh, non_blocking=True)
                copied[b].record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(copied[b])
                if i >= 2:
                    s_run.wait_event(drained[b])
                self(xd[b], y=yd[b])
                ran[b].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ran[b])
                yh.copy_(yd[b], non_blocking=True)
                drained[b].record(s_out)
        for st in (s_in, s_run, s_out):
            cur.wait_stream(st)
        for t in xd + yd:
            t.record_stream(s_in)
            t.record_stream(s_run)
            t.record_stream(s_out)
