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


def make_config(hidden_size: int, intermediate_size: int, num_local_experts: int, num_experts_per_tok: int,
                swiglu_limit: float = 7.0, swiglu_alpha: float = 1.702, dtype: str = "bf16",
                wfmt: str = "dense") -> MoeConfig:
    return MoeConfig(hidden_size, intermediate_size, num_local_experts, num_experts_per_tok, swiglu_limit,
                     swiglu_alpha, _DT[dtype][0], _lib.MOE_W_MXFP4 if wfmt == "mxfp4" else _lib.MOE_W_DENSE)


def config_from_spec(spec) -> MoeConfig:
    """Config of a ``workloads.LayerSpec``."""
    return make_config(spec.D, spec.F, spec.E, spec.k, spec.limit, spec.alpha, spec.dtype, spec.wfmt)


def torch_dtype(cfg: MoeConfig) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == _lib.MOE_BF16 else torch.float32


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmoe takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


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
# the five calls
# --------------------------------------------------------------------------- #
def router_topk(cfg: MoeConfig, x: torch.Tensor, w_router: torch.Tensor, b_router: torch.Tensor,
                topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None
                ) -> Tuple[torch.Tensor, torch.Tensor]:
    T, k = x.shape[0], cfg.num_experts_per_tok
    if topk_ids is None:
        topk_ids = torch.empty((T, k), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    _check(_lib.load().moe_router_topk(ctypes.byref(cfg), T, _p(x), _p(w_router), _p(b_router), _p(topk_ids),
                                       _p(topk_w), _stream(x.device)), "moe_router_topk")
    return topk_ids, topk_w


def permute(cfg: MoeConfig, topk_ids: torch.Tensor, x: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    L = _lib.load()
    T, k, dev = topk_ids.shape[0], cfg.num_experts_per_tok, topk_ids.device
    R = T * k
    out = dict(
        expert_off=torch.empty(cfg.num_local_experts + 1, dtype=torch.int32, device=dev),
        row_of_slot=torch.empty((T, k), dtype=torch.int32, device=dev),
        slot_of_row=torch.empty(R, dtype=torch.int32, device=dev),
    )
    out["x_perm"] = None if x is None else torch.empty((R, cfg.hidden_size), dtype=x.dtype, device=dev)
    nws = L.moe_permute_workspace_size(ctypes.byref(cfg), T)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    _check(L.moe_permute(ctypes.byref(cfg), T, _p(topk_ids), _p(x), _p(out["expert_off"]), _p(out["row_of_slot"]),
                         _p(out["slot_of_row"]), _p(out["x_perm"]), _p(ws), ws.numel(), _stream(dev)),
           "moe_permute")
    return out


def expert_ffn(cfg: MoeConfig, x_perm: torch.Tensor, expert_off: torch.Tensor, weights: ExpertWeights
               ) -> Tuple[torch.Tensor, torch.Tensor]:
    L = _lib.load()
    R, dev = x_perm.shape[0], x_perm.device
    T = R // cfg.num_experts_per_tok
    dt = torch_dtype(cfg)
    h = torch.empty((R, cfg.intermediate_size), dtype=dt, device=dev)
    y_perm = torch.empty((R, cfg.hidden_size), dtype=dt, device=dev)
    nws = L.moe_expert_ffn_workspace_size(ctypes.byref(cfg), T)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev) if nws else None
    ws_struct = weights.c_struct()
    _check(L.moe_expert_ffn(ctypes.byref(cfg), T, _p(x_perm), _p(expert_off), ctypes.byref(ws_struct), _p(h),
                            _p(y_perm), _p(ws), nws, _stream(dev)), "moe_expert_ffn")
    return h, y_perm


def combine(cfg: MoeConfig, y_perm: torch.Tensor, row_of_slot: torch.Tensor, topk_w: torch.Tensor) -> torch.Tensor:
    T, dev = row_of_slot.shape[0], y_perm.device
    y = torch.empty((T, cfg.hidden_size), dtype=y_perm.dtype, device=dev)
    _check(_lib.load().moe_combine(ctypes.byref(cfg), T, _p(y_perm), _p(row_of_slot), _p(topk_w), _p(y),
                                   _stream(dev)), "moe_combine")
    return y


def workspace_size(cfg: MoeConfig, T: int) -> int:
    n = _lib.load().moe_workspace_size(ctypes.byref(cfg), T)
    if n == _lib.SIZE_INVALID:
        raise MoeError(_lib.MOE_ERR_INVALID_ARG, "moe_workspace_size")
    return n


def layer_forward(cfg: MoeConfig, x: torch.Tensor, w_router: torch.Tensor, b_router: torch.Tensor,
                  weights: ExpertWeights, y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                  topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None) -> torch.Tensor:
    T, dev = x.shape[0], x.device
    if y is None:
        y = torch.empty((T, cfg.hidden_size), dtype=x.dtype, device=dev)
    if ws is None:
        ws = torch.empty(max(workspace_size(cfg, T), 16), dtype=torch.uint8, device=dev)
    wst = weights.c_struct()
    _check(_lib.load().moe_layer_forward(ctypes.byref(cfg), T, _p(x), _p(w_router), _p(b_router),
                                         ctypes.byref(wst), _p(y), _p(topk_ids), _p(topk_w), _p(ws), ws.numel(),
                                         _stream(dev)), "moe_layer_forward")
    return y


def last_device_error() -> int:
    """Reads and clears the device error word (synchronises); returns a status code."""
    return _lib.load().moe_last_device_error()


def set_expert_gemm_variant(variant: int) -> None:
    """0 = by size, 1 = single-CTA tiles, 2 = CTA-pair tiles (bf16 expert GEMMs)."""
    _check(_lib.load().moe_set_expert_gemm_variant(variant), "moe_set_expert_gemm_variant")


def set_wait_limit_ns(ns: int) -> None:
    _lib.load().moe_set_wait_limit_ns(ns)


class MoELayer:
    """A GPT-OSS MoE FFN layer resident on one GPU: weights, config and a reusable workspace."""

    def __init__(self, cfg: MoeConfig, w_router: torch.Tensor, b_router: torch.Tensor, experts: ExpertWeights):
        self.cfg, self.w_router, self.b_router, self.experts = cfg, w_router, b_router, experts
        self._ws: Optional[torch.Tensor] = None

    def workspace(self, T: int) -> torch.Tensor:
        n = max(workspace_size(self.cfg, T), 16)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, dtype=torch.uint8, device=self.w_router.device)
        return self._ws

    def __call__(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, topk_ids=None, topk_w=None) -> torch.Tensor:
        return layer_forward(self.cfg, x, self.w_router, self.b_router, self.experts, y=y,
                             ws=self.workspace(x.shape[0]), topk_ids=topk_ids, topk_w=topk_w)

    def graphed(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, topk_ids=None, topk_w=None):
        """Capture one forward on these fixed buffers into a CUDA graph; returns (replay, y).

        The library makes no host synchronisation and allocates nothing, so its
        launches are captured as they are; ``replay()`` re-runs them on whatever
        ``x`` holds at that time.  Removes host launch overhead (decode sizes).
        """
        if y is None:
            y = torch.empty((x.shape[0], self.cfg.hidden_size), dtype=x.dtype, device=x.device)
        ws = self.workspace(x.shape[0])
        self(x, y=y, topk_ids=topk_ids, topk_w=topk_w)          # warm: per-device set-up outside capture
        torch.cuda.synchronize(x.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer_forward(self.cfg, x, self.w_router, self.b_router, self.experts, y=y, ws=ws,
                          topk_ids=topk_ids, topk_w=topk_w)
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
        yd = [torch.empty((T, self.cfg.hidden_size), dtype=xs_host[0].dtype, device=dev) for _ in range(2)]
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
