"""Helpers for the GPU parity tests: seeded layers, uploads, error metrics.

Inputs come from ``workloads`` (near-tie rejection through the oracle's own
router); expected values come from ``oracle`` only.
"""
from __future__ import annotations

import functools

import numpy as np

import workloads as W
from oracle import moe_oracle as O

# Tolerances (stated in the layer's acceptance criteria): the max abs error of
# the layer output relative to the RMS of the reference output.
TOL_Y = {"bf16": 2e-2, "f32": 2e-2, "mxfp4": 5e-2}
# routing weights are fp32 softmaxes of fp32-accumulated logits
TOL_W = 2e-5


def logits_fn(layer):
    return O.router_logits(layer["x"], layer["w_router"], layer["b_router"])


@functools.lru_cache(maxsize=2)
def _experts(spec_key: W.LayerSpec, seed: int):
    return W.make_experts(spec_key, seed)


@functools.lru_cache(maxsize=4)
def _router_part(spec: W.LayerSpec, seed: int):
    return W.make_layer(spec, seed=seed, logits_fn=logits_fn, with_experts=False)


def layer_for(spec: W.LayerSpec, seed: int = 0, experts: bool = True):
    """Seeded layer; expert weights are shared by specs that differ only in T (prefill/decode)."""
    layer = dict(_router_part(spec, seed))
    if experts:
        import dataclasses
        layer.update(_experts(dataclasses.replace(spec, T=0, name=""), seed))
    return layer


def check_output(got: np.ndarray, ref: np.ndarray, tol: float, bf16_out: bool) -> float:
    """Layer output check: |got - ref| <= tol * RMS(ref) + (output rounding) per element.

    The output is stored in the activation dtype.  Rounding the exact fp64
    result to bf16 moves an element by up to half an ulp, <= 2^-8 |ref|, which
    on large-magnitude elements is already close to 2e-2 of the RMS (for the
    GPT-OSS-120B-shaped layer: 1.75e-2 on the sampled tokens, 2^-8 x max|y|/RMS
    = 2.3e-2 in the worst case), so that rounding is allowed on top of the bound.
    Returns the raw max |got - ref| / RMS(ref) for the record.
    """
    rms = float(np.sqrt(np.mean(np.square(ref))))
    allow = (2.0 ** -8 if bf16_out else 2.0 ** -23) * np.abs(ref)
    excess = np.abs(got - ref) - (tol * rms + allow)
    raw = float(np.max(np.abs(got - ref))) / max(rms, 1e-30)
    assert np.all(excess <= 0), f"max excess {excess.max():.3e}; raw max err / RMS = {raw:.3e}"
    print(f"max err / RMS = {raw:.3e}")
    return raw


def rel_rms(got: np.ndarray, ref: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(np.square(ref))))
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-30)


def check_stored(got: np.ndarray, ref: np.ndarray, tol: float, bf16_stored: bool) -> None:
    """Intermediates (h, y_perm) kept in the activation dtype.

    A bf16-stored value differs from its exact value by its rounding, up to
    2^-9 of its magnitude; heavy-tailed intermediates (h ~ g^2 u near 0) put
    that rounding above tol * RMS on their largest elements.  So each element
    may differ by 2^-8 |ref| (rounding plus fp32 accumulation) + tol * RMS(ref).
    """
    rms = float(np.sqrt(np.mean(np.square(ref))))
    bound = (2.0 ** -8 if bf16_stored else 0.0) * np.abs(ref) + tol * rms
    excess = np.abs(got - ref) - bound
    assert np.all(excess <= 0), f"max excess {excess.max():.3e} (rms {rms:.3e})"


def f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def tol_for(spec: W.LayerSpec) -> float:
    return TOL_Y["mxfp4"] if spec.wfmt == "mxfp4" else TOL_Y[spec.dtype]


def check_ids(gpu_ids: np.ndarray, ref_ids: np.ndarray, ref_logits: np.ndarray, order_gap: float = 1e-4):
    """Selected expert sets are bit-exact; their order too wherever neighbours differ by >= order_gap."""
    assert gpu_ids.shape == ref_ids.shape
    assert np.array_equal(np.sort(gpu_ids, axis=1), np.sort(ref_ids, axis=1)), "expert sets differ"
    sel = np.take_along_axis(ref_logits, ref_ids.astype(np.int64), axis=1)
    k = ref_ids.shape[1]
    for j in range(k):
        # position j is determined if it is separated from both neighbours
        sep = np.ones(ref_ids.shape[0], bool)
        if j > 0:
            sep &= (sel[:, j - 1] - sel[:, j]) >= order_gap
        if j < k - 1:
            sep &= (sel[:, j] - sel[:, j + 1]) >= order_gap
        assert np.array_equal(gpu_ids[sep, j], ref_ids[sep, j]), f"slot order differs at j={j}"


def pairs_of_rows(slot_of_row: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """(token, expert) held by each permuted row -- independent of the slot order within a token."""
    k = ids.shape[1]
    s = slot_of_row.astype(np.int64)
    return np.stack([s // k, ids.reshape(-1)[s]], axis=1)
