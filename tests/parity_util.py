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


def check_output(got: np.ndarray, ref: np.ndarray, tol: float) -> float:
    """Layer output check, the acceptance bound as written: max |got - ref| <= tol * RMS(ref).

    ``got`` is the fp32 layer output (the layer's y_f32 option): for a bf16 layer,
    rounding even the exact fp64 result to bf16 moves the largest elements by up
    to 2^-8 |y|, which reaches 2e-2 of the RMS on the GPT-OSS-120B-shaped layer
    (max |y| / RMS = 6.7) -- no bf16-stored output can meet the bound there, so
    the bound is asserted on the fp32 output and the bf16 output is checked to be
    exactly its rounding (``check_rounding``).  Returns the max error / RMS.
    """
    rms = float(np.sqrt(np.mean(np.square(ref))))
    raw = float(np.max(np.abs(got - ref))) / max(rms, 1e-30)
    print(f"max err / RMS = {raw:.3e} (bound {tol:g})")
    assert raw <= tol, f"max |y - y_ref| / RMS = {raw:.4e} > {tol:g}"
    return raw


def check_rounding(y_out, y32, ref: np.ndarray = None) -> None:
    """The layer output in its dtype is the round-to-nearest-even of the fp32 output, bit for bit.

    y_out, y32: torch tensors of the same layer call made with and without y_f32.
    For the record, prints the max error / RMS of the bf16 output and of the exact
    result rounded to bf16 (both include the same storage rounding).
    """
    import torch
    if y_out.dtype == torch.float32:
        assert torch.equal(y_out, y32)
        return
    want = W.f32_to_bf16_bits(y32.cpu().numpy())
    got = y_out.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want), "bf16 output is not the rounding of the fp32 output"
    if ref is not None:
        rms = float(np.sqrt(np.mean(np.square(ref))))
        exact_rounded = W.bf16_bits_to_f32(W.f32_to_bf16_bits(ref.astype(np.float32))).astype(np.float64)
        print(f"bf16 output: max err / RMS = {np.max(np.abs(f64(y_out) - ref)) / rms:.3e}; "
              f"exact result rounded to bf16: {np.max(np.abs(exact_rounded - ref)) / rms:.3e}")


def h_rounding_bound(layer, ids: np.ndarray, w: np.ndarray, h: np.ndarray) -> np.ndarray:
    """Per-element bound on how far keeping h in bf16 can move the layer output.

    Each stored h value differs from the exact one by its bf16 rounding, at most
    2^-9 |h| (plus a little fp32 arithmetic), so |delta y[t, d]| <=
    2^-9 * sum_j w[t, j] * sum_f |h[t, j, f]| |W_d[e_j][d, f]|.  Returned with the
    factor 2^-8 (twice the rounding bound) as margin for the fp32 side.
    ids, w [n, k] and h [n, k, F] are the oracle's, for the n tokens compared.
    """
    n, k = ids.shape
    out = np.zeros((n, layer["b_down"].shape[1]))
    for e in np.unique(ids):
        ii, jj = np.nonzero(ids == e)
        wd = np.abs(O.expert_weights(layer, "down", int(e)))
        out[ii] += w[ii, jj][:, None] * (np.abs(h[ii, jj]) @ wd.T)
    return 2.0 ** -8 * out


def h_rounding_bound_glm(layer, ref) -> np.ndarray:
    """h_rounding_bound for the GLM4-MoE-Lite variant: the routed experts' h (oracle, permuted
    order) and the shared expert's h, each against |W_d| of its expert."""
    from oracle import glm_moe as G
    ids, w, ros, h = ref["ids"], ref["w"], ref["row_of_slot"], ref["h"]
    T, k = ids.shape
    out = np.zeros((T, layer["w_down"].shape[1]))
    for e in np.unique(ids):
        ii, jj = np.nonzero(ids == e)
        wd = np.abs(G.decode(layer["w_down"][int(e)]))
        out[ii] += w[ii, jj][:, None] * (np.abs(h[ros[ii, jj]]) @ wd.T)
    if "ws_gate" in layer:
        x = G.decode(layer["x"])
        hs, _ = G.silu_mlp(x, G.decode(layer["ws_gate"]), G.decode(layer["ws_up"]), G.decode(layer["ws_down"]))
        out += np.abs(hs) @ np.abs(G.decode(layer["ws_down"])).T
    return 2.0 ** -8 * out


def check_h_rounding(y_default: np.ndarray, y_split: np.ndarray, bound: np.ndarray, ref: np.ndarray) -> None:
    """The layer with h in one bf16 value differs from the layer with h in two bf16 halves
    by no more than the bf16 rounding of h can explain (both outputs in fp32)."""
    rms = float(np.sqrt(np.mean(np.square(ref))))
    excess = np.abs(y_default - y_split) - (bound + 1e-4 * rms)
    assert np.all(excess <= 0), f"h-in-bf16 output off by more than its rounding: excess {excess.max():.3e}"


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
