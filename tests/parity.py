"""Comparison helpers for GPU-vs-oracle parity tests.

Tolerances (max absolute error against the fp64 oracle, element by element):
  * fp16 inputs: |dO| <= 2e-3, |dLSE| <= 1e-3;
  * bf16 inputs: |dO| <= 1.5e-2, |dLSE| <= 1e-3.

One allowance, always reported: where the exact output is so large that one
unit in the last place (ulp) of the output type is already at least the bound
(|O| >= 2 in bf16, where an ulp is 2^-6 = 0.0156; |O| >= 4 in fp16, where it is
2^-8 = 0.0039), an output beyond the bound still passes if it lies within one
ulp of the exact result rounded to the output type (round to nearest even).
The kernel rounds its fp32 result once, so half an ulp of its error is the
rounding alone and the rest is its fp32 arithmetic and the rounding of P.
Nothing else is widened. Every output that passed this way is counted per
comparison, its first locations are kept, and the session prints the counts
(`conftest.py` terminal summary), so no widening goes unseen.

LSE rows that are -inf in the oracle (no visible key) must be -inf on the GPU,
with O = 0.
"""
from __future__ import annotations

import numpy as np
import torch

TOL_O = {torch.float16: 2e-3, torch.bfloat16: 1.5e-2}
TOL_LSE = 1e-3
MANT_BITS = {torch.float16: 10, torch.bfloat16: 7}
# Smallest normal magnitude of each output type (ulp below it is constant).
MIN_NORMAL_EXP = {torch.float16: -14, torch.bfloat16: -126}

# Every comparison made in this process: (label, result dict). The terminal
# summary of the test session prints it.
RECORDS: list[tuple[str, dict]] = []


def ulp(x: np.ndarray, dtype) -> np.ndarray:
    """One unit in the last place of `dtype` at magnitude |x| (x in fp64)."""
    e_min = MIN_NORMAL_EXP[dtype]
    mag = np.maximum(np.abs(x), 2.0 ** e_min)
    return 2.0 ** (np.floor(np.log2(mag)) - MANT_BITS[dtype])


def round_to(x: np.ndarray, dtype) -> np.ndarray:
    """x (fp64) rounded to `dtype` with round-to-nearest-even, back in fp64."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).double().numpy()


def o_check(o: np.ndarray, o_ref: np.ndarray, dtype) -> dict:
    """Element-wise check of O (both fp64 arrays of the same shape).

    Returns max |dO|, the number of outputs that passed under the one-ulp
    allowance and their first locations, and the number of failures."""
    tol = TOL_O[dtype]
    err = np.abs(o - o_ref)
    over = err > tol
    res = {"max_abs_o": float(err.max(initial=0.0)), "tol_o": tol, "n_ulp_allowance": 0,
           "ulp_allowance_at": [], "n_bad": 0}
    if not over.any():
        return res
    ref_r = round_to(o_ref, dtype)
    coarse = ulp(o_ref, dtype) >= tol  # one output ulp is at least the bound here
    near = np.abs(o - ref_r) <= ulp(ref_r, dtype)
    allowed = over & coarse & near
    bad = over & ~allowed
    idx = np.argwhere(allowed)
    res["n_ulp_allowance"] = int(allowed.sum())
    res["ulp_allowance_at"] = [tuple(int(i) for i in r) for r in idx[:8]]
    res["n_bad"] = int(bad.sum())
    if bad.any():
        worst = np.unravel_index(int(np.argmax(np.where(bad, err, -1.0))), err.shape)
        res["worst_bad"] = (tuple(int(i) for i in worst), float(o_ref[worst]), float(o[worst]))
    return res


def compare(o_gpu: torch.Tensor, lse_gpu, o_ref: np.ndarray, lse_ref: np.ndarray, dtype,
            what: str = "") -> dict:
    o = o_gpu.detach().float().cpu().numpy().astype(np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    res = o_check(o, o_ref, dtype)
    assert res["n_bad"] == 0, (
        f"{what}: {res['n_bad']} outputs beyond tolerance {res['tol_o']:g} and not within one "
        f"output ulp of the rounded exact value; max |dO| = {res['max_abs_o']:.3e}; worst "
        f"(index, ref, gpu) = {res.get('worst_bad')}")
    if lse_gpu is not None:
        l = lse_gpu.detach().cpu().numpy().astype(np.float64)
        assert l.shape == lse_ref.shape
        fin = np.isfinite(lse_ref)
        assert (np.isneginf(l) == ~fin).all(), f"{what}: -inf pattern of LSE differs"
        el = np.abs(l[fin] - lse_ref[fin]).max(initial=0.0)
        assert el <= TOL_LSE, f"{what}: max |dLSE| = {el:.3e}"
        empty = ~fin
        if empty.any():
            assert (o[empty] == 0).all(), f"{what}: rows without keys must be 0"
        res["max_abs_lse"] = float(el)
    res["n_outputs"] = int(o.size)
    RECORDS.append((what or "unnamed", res))
    return res


def summary_lines() -> list[str]:
    """One line per comparison of this session (for the terminal summary)."""
    out = []
    for what, r in RECORDS:
        line = (f"{what}: max|dO| {r['max_abs_o']:.3e} (tol {r['tol_o']:g}), "
                f"max|dLSE| {r.get('max_abs_lse', float('nan')):.3e}, "
                f"ulp allowance used by {r['n_ulp_allowance']} of {r['n_outputs']} outputs")
        if r["n_ulp_allowance"]:
            line += f" at {r['ulp_allowance_at']}"
        out.append(line)
    return out
