"""Seeded synthetic inputs for the GPT-OSS MoE FFN layer.

This module is shared by the tests, the benchmark and the oracle-side checks.
It holds the input *recipes* only (shapes, value laws, seeds, storage formats)
and none of the layer's arithmetic: where a recipe needs the router logits
(the near-tie rejection), the caller passes a ``logits_fn``.

Storage formats handed out (numpy arrays, row-major):
  * ``bf16``  -> ``np.uint16`` holding the bf16 bit pattern (round-to-nearest-even
    from an fp32 draw);
  * ``f32``   -> ``np.float32``;
  * MXFP4     -> packed E2M1 codes ``np.uint8 [.., N, K/2]`` (element ``2i`` is the
    low nibble of byte ``i``) plus E8M0 scale bytes ``np.uint8 [.., N, K/32]``.

Layouts (reduction dim contiguous, i.e. "[N, K]" for every weight):
  x [T, D], w_router [E, D], b_router [E],
  w_gate / w_up [E, F, D], b_gate / b_up [E, F], w_down [E, D, F], b_down [E, D].

Parameter names follow the GPT-OSS weight map on the MaxText page
("MoE Router": router kernel and bias; "MOE EXPERTS": wi_0 gate, wi_1 up, wo down,
each with a bias); the layer sizes follow the GPT-OSS Config
(hidden_size, num_local_experts, num_experts_per_tok, swiglu_limit) and the
GPT-OSS 20B model card (32 experts, 4 active per token; MXFP4 expert weights).

``GlmLayerSpec`` / ``make_glm_layer`` are the recipes of the layer's GLM4-MoE-Lite
variant ("Ollama glm4_moe_lite.go"): a router without bias plus an
``e_score_correction_bias`` [E], expert weights without biases, and a shared
expert ws_gate / ws_up [F_shared, D], ws_down [D, F_shared].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Dict, Optional

import numpy as np

SWIGLU_ALPHA = 1.702


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """One synthetic layer: sizes, formats and value laws."""

    name: str
    T: int                 # tokens
    D: int                 # hidden_size
    E: int                 # num_local_experts
    k: int                 # num_experts_per_tok
    F: int                 # per-expert intermediate size
    dtype: str             # "f32" or "bf16": activations, router and dense weights
    wfmt: str = "dense"    # "dense" or "mxfp4": expert weights
    limit: float = 7.0     # swiglu_limit
    alpha: float = SWIGLU_ALPHA
    # value laws (standard deviations)
    x_std: float = 1.0
    router_w_std: Optional[float] = None   # None -> 1/sqrt(D)
    router_b: str = "zero"                 # "normal", "zero" or "zipf"
    router_b_std: float = 0.01
    zipf_s: float = 1.1
    expert_w_std: Optional[float] = None   # None -> 1/sqrt(fan_in)
    expert_b_std: float = 0.01
    dead_experts: tuple = ()               # router bias -30 for these: they receive no tokens
    cfg_id: int = 0                        # seeds the streams; distinct per recipe

    @property
    def R(self) -> int:
        return self.T * self.k

    def with_tokens(self, T: int) -> "LayerSpec":
        return dataclasses.replace(self, T=T, name=f"{self.name}_T{T}")

    def expert_flops(self) -> float:
        """Algorithmic FLOPs of the expert GEMMs (gate, up, down) for T tokens."""
        return 6.0 * self.R * self.D * self.F

    def router_flops(self) -> float:
        return 2.0 * self.T * self.D * self.E


TINY_FP32 = LayerSpec(
    name="tiny_fp32", T=64, D=256, E=8, k=2, F=512, dtype="f32",
    router_w_std=0.05, router_b="normal", router_b_std=0.01,
    expert_w_std=0.02, expert_b_std=0.01, cfg_id=1)

GPTOSS20B_PREFILL = LayerSpec(
    name="gptoss20b_prefill", T=4096, D=2880, E=32, k=4, F=2880, dtype="bf16",
    router_b="zero", cfg_id=2)

# Decode uses the very same layer (same weight streams) with few tokens.
GPTOSS20B_DECODE_T = (1, 8, 32, 64)


def gptoss20b_decode(T: int) -> LayerSpec:
    return dataclasses.replace(GPTOSS20B_PREFILL, T=T, name=f"gptoss20b_decode_T{T}")


GPTOSS20B_MXFP4 = LayerSpec(
    name="gptoss20b_mxfp4", T=8192, D=2880, E=32, k=4, F=2880, dtype="bf16",
    wfmt="mxfp4", router_b="zero", cfg_id=4)

GPTOSS120B_SKEWED = LayerSpec(
    name="gptoss120b_skewed", T=16384, D=2880, E=128, k=4, F=2880, dtype="bf16",
    router_b="zipf", zipf_s=1.1, cfg_id=5)

SPECS: Dict[str, LayerSpec] = {s.name: s for s in (
    TINY_FP32, GPTOSS20B_PREFILL, GPTOSS20B_MXFP4, GPTOSS120B_SKEWED)}
for _t in GPTOSS20B_DECODE_T:
    SPECS[f"gptoss20b_decode_T{_t}"] = gptoss20b_decode(_t)


# --------------------------------------------------------------------------- #
# storage-format helpers (format conversion only)
# --------------------------------------------------------------------------- #
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(spec: LayerSpec, seed: int, *stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, spec.cfg_id, *stream])


def _normal(rng: np.random.Generator, shape, std: float, dtype: str) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    a *= np.float32(std)
    if dtype == "bf16":
        return f32_to_bf16_bits(a)
    return a


def zipf_log_bias(E: int, s: float) -> np.ndarray:
    """Router bias b[e] = ln p_(e+1), p_i = i^-s / sum_j j^-s (expert 0 most popular)."""
    i = np.arange(1, E + 1, dtype=np.float64)
    p = i ** (-s)
    p /= p.sum()
    return np.log(p)


# stream ids
_S_X, _S_WR, _S_BR, _S_WG, _S_BG, _S_WU, _S_BU, _S_WD, _S_BD, _S_REDRAW = range(10)


def make_layer(spec: LayerSpec, seed: int = 0,
               logits_fn: Optional[Callable[[Dict[str, np.ndarray]], np.ndarray]] = None,
               min_gap: float = 1e-3, max_redraw: int = 64,
               with_experts: bool = True) -> Dict[str, np.ndarray]:
    """Draw every tensor of the layer.

    ``logits_fn(layer) -> float64 [T, E]`` turns on the near-tie rejection: any
    token whose k-th and (k+1)-th largest router logits are closer than
    ``min_gap`` has its activation row redrawn from a per-token stream
    ``(seed, cfg_id, 9, t, attempt)`` until the gap is met.
    """
    T, D, E, F, k = spec.T, spec.D, spec.E, spec.F, spec.k
    out: Dict[str, np.ndarray] = {}
    out["x"] = _normal(_rng(spec, seed, _S_X, T), (T, D), spec.x_std, spec.dtype)
    wr_std = spec.router_w_std if spec.router_w_std is not None else 1.0 / math.sqrt(D)
    out["w_router"] = _normal(_rng(spec, seed, _S_WR), (E, D), wr_std, spec.dtype)
    if spec.router_b == "normal":
        br = _rng(spec, seed, _S_BR).standard_normal(E, dtype=np.float32) * np.float32(spec.router_b_std)
    elif spec.router_b == "zipf":
        br = zipf_log_bias(E, spec.zipf_s).astype(np.float32)
    else:
        br = np.zeros(E, dtype=np.float32)
    for e in spec.dead_experts:
        br[e] = -30.0
    out["b_router"] = f32_to_bf16_bits(br) if spec.dtype == "bf16" else br.astype(np.float32)

    if with_experts:
        out.update(make_experts(spec, seed))

    if logits_fn is not None and k < E:
        _reject_near_ties(spec, seed, out, logits_fn, min_gap, max_redraw)
    return out


def make_experts(spec: LayerSpec, seed: int = 0) -> Dict[str, np.ndarray]:
    """Expert weights and biases, drawn one expert at a time (bounded host memory)."""
    D, E, F = spec.D, spec.E, spec.F
    res: Dict[str, np.ndarray] = {}
    wdt = spec.dtype
    for name, stream, n, kdim in (("gate", _S_WG, F, D), ("up", _S_WU, F, D), ("down", _S_WD, D, F)):
        if spec.wfmt == "mxfp4":
            if kdim % 32:
                raise ValueError("MXFP4 needs the reduction dim to be a multiple of 32")
            q = np.empty((E, n, kdim // 2), dtype=np.uint8)
            s = np.empty((E, n, kdim // 32), dtype=np.uint8)
            for e in range(E):
                r = _rng(spec, seed, stream, e)
                q[e] = r.integers(0, 256, size=(n, kdim // 2), dtype=np.uint8)
                s[e] = (127 + r.integers(-8, 1, size=(n, kdim // 32))).astype(np.uint8)
            res[f"w_{name}"] = q
            res[f"s_{name}"] = s
        else:
            std = spec.expert_w_std if spec.expert_w_std is not None else 1.0 / math.sqrt(kdim)
            w = np.empty((E, n, kdim), dtype=np.uint16 if wdt == "bf16" else np.float32)
            for e in range(E):
                w[e] = _normal(_rng(spec, seed, stream, e), (n, kdim), std, wdt)
            res[f"w_{name}"] = w
    for name, stream, n in (("gate", _S_BG, F), ("up", _S_BU, F), ("down", _S_BD, D)):
        res[f"b_{name}"] = _normal(_rng(spec, seed, stream), (E, n), spec.expert_b_std, wdt)
    return res


def _kth_gap(logits: np.ndarray, k: int) -> np.ndarray:
    srt = -np.sort(-logits, axis=1)
    return srt[:, k - 1] - srt[:, k]


def _reject_near_ties(spec, seed, layer, logits_fn, min_gap, max_redraw):
    lg = logits_fn(layer)
    bad = np.nonzero(_kth_gap(lg, spec.k) < min_gap)[0]
    for t in bad:
        for attempt in range(max_redraw):
            row = _normal(_rng(spec, seed, _S_REDRAW, int(t), attempt), (1, spec.D), spec.x_std, spec.dtype)
            layer["x"][t] = row[0]
            one = dict(layer)
            one["x"] = layer["x"][t:t + 1]
            if _kth_gap(logits_fn(one), spec.k)[0] >= min_gap:
                break
        else:
            raise RuntimeError(f"token {t}: no redraw met the router-logit gap")


def tiny_spec(T: int, D: int, E: int, k: int, F: int, dtype: str = "f32", wfmt: str = "dense",
              router_b: str = "normal", cfg_id: int = 100, **kw) -> LayerSpec:
    """Small ad-hoc layers (ragged tails, degenerate cases) with the tiny-config value laws."""
    return LayerSpec(name=f"tiny_T{T}_D{D}_E{E}_k{k}_F{F}_{dtype}_{wfmt}", T=T, D=D, E=E, k=k, F=F,
                     dtype=dtype, wfmt=wfmt, router_w_std=kw.pop("router_w_std", 0.05),
                     router_b=router_b, expert_w_std=kw.pop("expert_w_std", 0.02),
                     cfg_id=cfg_id, **kw)


# --------------------------------------------------------------------------- #
# GLM4-MoE-Lite variant of the layer ("Ollama glm4_moe_lite.go": Config,
# MoEGate, SwitchMLP, SharedExperts).  The page gives the config field names
# but no sizes, so the variant's layers take the GPT-OSS-shaped sizes above.
# --------------------------------------------------------------------------- #
@dataclasses.dataclass(frozen=True)
class GlmLayerSpec:
    """One synthetic GLM4-MoE-Lite-style layer: sigmoid router with a selection-only
    correction bias, SiLU experts without biases, an optional shared expert."""

    name: str
    T: int
    D: int                 # hidden_size
    E: int                 # n_routed_experts
    k: int                 # num_experts_per_tok
    F: int                 # moe_intermediate_size
    F_shared: int          # intermediate size of the shared expert (0: no shared expert)
    dtype: str             # "f32" or "bf16"
    norm_topk_prob: bool = True
    routed_scaling_factor: float = 2.5
    x_std: float = 1.0
    router_w_std: Optional[float] = None       # None -> 1/sqrt(D)
    correction_b_std: Optional[float] = 0.1    # None: no e_score_correction_bias
    expert_w_std: Optional[float] = None       # None -> 1/sqrt(fan_in)
    cfg_id: int = 300

    @property
    def R(self) -> int:
        return self.T * self.k


_S_CB, _S_SG, _S_SU, _S_SD = 10, 11, 12, 13


def make_glm_layer(spec: GlmLayerSpec, seed: int = 0,
                   scores_fn: Optional[Callable[[Dict[str, np.ndarray]], np.ndarray]] = None,
                   min_gap: float = 1e-3, max_redraw: int = 64) -> Dict[str, np.ndarray]:
    """Draw every tensor of a variant layer.

    x [T, D], w_router [E, D], e_score_correction_bias [E] (when
    ``correction_b_std`` is set), w_gate / w_up [E, F, D], w_down [E, D, F], and
    for the shared expert ws_gate / ws_up [F_shared, D], ws_down [D, F_shared].
    ``scores_fn(layer) -> float64 [T, E]`` (the scores the experts are chosen by)
    turns on the near-tie rejection, as for ``make_layer``.
    """
    T, D, E, F = spec.T, spec.D, spec.E, spec.F
    out: Dict[str, np.ndarray] = {}
    out["x"] = _normal(_rng(spec, seed, _S_X, T), (T, D), spec.x_std, spec.dtype)
    wr_std = spec.router_w_std if spec.router_w_std is not None else 1.0 / math.sqrt(D)
    out["w_router"] = _normal(_rng(spec, seed, _S_WR), (E, D), wr_std, spec.dtype)
    if spec.correction_b_std is not None:
        out["e_score_correction_bias"] = _normal(_rng(spec, seed, _S_CB), (E,), spec.correction_b_std, spec.dtype)
    for name, stream, n, kdim in (("gate", _S_WG, F, D), ("up", _S_WU, F, D), ("down", _S_WD, D, F)):
        std = spec.expert_w_std if spec.expert_w_std is not None else 1.0 / math.sqrt(kdim)
        w = np.empty((E, n, kdim), dtype=np.uint16 if spec.dtype == "bf16" else np.float32)
        for e in range(E):
            w[e] = _normal(_rng(spec, seed, stream, e), (n, kdim), std, spec.dtype)
        out[f"w_{name}"] = w
    if spec.F_shared > 0:
        Fs = spec.F_shared
        for name, stream, n, kdim in (("gate", _S_SG, Fs, D), ("up", _S_SU, Fs, D), ("down", _S_SD, D, Fs)):
            std = spec.expert_w_std if spec.expert_w_std is not None else 1.0 / math.sqrt(kdim)
            out[f"ws_{name}"] = _normal(_rng(spec, seed, stream), (n, kdim), std, spec.dtype)
    if scores_fn is not None and spec.k < E:
        _reject_near_ties(spec, seed, out, scores_fn, min_gap, max_redraw)
    return out


def glm_tiny_spec(T: int, D: int, E: int, k: int, F: int, F_shared: int, dtype: str = "f32",
                  cfg_id: int = 310, **kw) -> GlmLayerSpec:
    """Small variant layers with the tiny-config value laws."""
    return GlmLayerSpec(name=f"glm_tiny_T{T}_D{D}_E{E}_k{k}_F{F}_S{F_shared}_{dtype}", T=T, D=D, E=E, k=k, F=F,
                        F_shared=F_shared, dtype=dtype, router_w_std=kw.pop("router_w_std", 0.05),
                        expert_w_std=kw.pop("expert_w_std", 0.02), cfg_id=cfg_id, **kw)


GLM_GPTOSS20B_SHAPE = GlmLayerSpec(
    name="glm_variant_gptoss20b_shape", T=4096, D=2880, E=32, k=4, F=2880, F_shared=2880, dtype="bf16",
    cfg_id=320)
