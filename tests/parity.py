"""Comparison helpers for GPU-vs-oracle parity tests.

Tolerances (max absolute error against the fp64 oracle, element by element):
  * fp16 inputs: |dO| <= 2e-3, |dLSE| <= 1e-3;
  * bf16 inputs: |dO| <= 1.5e-2, |dLSE| <= 1e-3.
An output the exact result of which is large enough that a single rounding to
the output type already exceeds the bound (|O| >= 4 in bf16, >= 2 in fp16) is
held to one unit in the last place of that type instead: no implementation
that rounds its result could do better there. LSE rows that are -inf in the
oracle (no visible key) must be -inf on the GPU, with O = 0.
"""
from __future__ import annotations

import numpy as np
import torch

TOL_O = {torch.float16: 2e-3, torch.bfloat16: 1.5e-2}
TOL_LSE = 1e-3
MANT_BITS = {torch.float16: 10, torch.bfloat16: 7}


def ulp(x: np.ndarray, dtype) -> np.ndarray:
    mag = np.maximum(np.abs(x), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(mag)) - MANT_BITS[dtype])


def compare(o_gpu: torch.Tensor, lse_gpu, o_ref: np.ndarray, lse_ref: np.ndarray, dtype,
            what: str = "") -> dict:
    o = o_gpu.detach().float().cpu().numpy().astype(np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    err = np.abs(o - o_ref)
    bound = np.maximum(TOL_O[dtype], ulp(o_ref, dtype))
    bad = err > bound
    worst = int(np.argmax(err))
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} outputs beyond tolerance; max |dO| = {err.max():.3e} at "
        f"{np.unravel_index(worst, err.shape)} (ref {o_ref.flat[worst]:.4f}, gpu {o.flat[worst]:.4f})")
    res = {"max_abs_o": float(err.max()), "n_ulp_allowance": int((err > TOL_O[dtype]).sum())}
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
    return res
