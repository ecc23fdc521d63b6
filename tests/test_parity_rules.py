"""The comparison rule of `parity.py`, checked on planted values (CPU only).

The rule: an output passes if it is within the stated absolute bound of the
exact value; beyond it, only where one ulp of the output type is at least the
bound (|O| >= 2 in bf16, >= 4 in fp16) and only within one ulp of the exact
value rounded to that type, and every such output is counted.
"""
import numpy as np
import pytest
import torch

import parity

BF16, F16 = torch.bfloat16, torch.float16


def test_ulp_values():
    assert parity.ulp(np.array([1.0]), BF16)[0] == 2.0 ** -7
    assert parity.ulp(np.array([2.0]), BF16)[0] == 2.0 ** -6
    assert parity.ulp(np.array([-3.9]), BF16)[0] == 2.0 ** -6
    assert parity.ulp(np.array([4.0]), F16)[0] == 2.0 ** -8
    assert parity.ulp(np.array([0.0]), F16)[0] == 2.0 ** -24


def test_thresholds_where_one_ulp_reaches_the_bound():
    # bf16: one ulp reaches 1.5e-2 from |O| = 2; fp16: one ulp reaches 2e-3 from |O| = 4.
    assert parity.ulp(np.array([1.99]), BF16)[0] < parity.TOL_O[BF16] <= \
        parity.ulp(np.array([2.0]), BF16)[0]
    assert parity.ulp(np.array([3.99]), F16)[0] < parity.TOL_O[F16] <= \
        parity.ulp(np.array([4.0]), F16)[0]


def test_within_bound_passes_without_allowance():
    ref = np.array([0.5, -1.25, 3.0])
    out = ref + np.array([0.014, -0.01, 0.0149])
    r = parity.o_check(out, ref, BF16)
    assert r["n_bad"] == 0 and r["n_ulp_allowance"] == 0


def test_one_ulp_allowance_counted_and_located():
    # exact 5.01 rounds to 5.0 in bf16 (ulp 1/32); the GPU value one ulp above
    # the rounded value is 0.021 away: beyond 1.5e-2 but within one ulp.
    ref = np.array([[0.1, 5.01], [-6.2, 0.0]])
    out = ref.copy()
    out[0, 1] = 5.0 + 2.0 ** -5
    out[1, 0] = float(parity.round_to(np.array([-6.2]), BF16)[0]) - 2.0 ** -5
    r = parity.o_check(out, ref, BF16)
    assert r["n_bad"] == 0
    assert r["n_ulp_allowance"] == 2
    assert r["ulp_allowance_at"] == [(0, 1), (1, 0)]


def test_two_ulps_off_fails():
    ref = np.array([5.01])
    out = np.array([5.0 + 2 * 2.0 ** -5])
    assert parity.o_check(out, ref, BF16)["n_bad"] == 1


def test_small_outputs_get_no_allowance():
    # |O| < 2 in bf16: one ulp (<= 2^-7) is below the bound, so no widening.
    ref = np.array([1.9])
    out = np.array([1.9 + 0.016])
    r = parity.o_check(out, ref, BF16)
    assert r["n_bad"] == 1 and r["n_ulp_allowance"] == 0
    # fp16 between 2 and 4: ulp 2^-9 < 2e-3, no allowance either
    r = parity.o_check(np.array([3.0 + 0.0025]), np.array([3.0]), F16)
    assert r["n_bad"] == 1


def test_compare_records_and_asserts():
    n0 = len(parity.RECORDS)
    ref = np.array([[5.01, 0.25]])
    gpu = torch.tensor([[5.0 + 2.0 ** -5, 0.25]], dtype=torch.float64).to(BF16)
    lse_ref = np.array([1.0])
    parity.compare(gpu, torch.tensor([1.0002]), ref, lse_ref, BF16, "planted")
    assert len(parity.RECORDS) == n0 + 1
    what, r = parity.RECORDS[-1]
    assert what == "planted" and r["n_ulp_allowance"] == 1
    assert any("planted" in s and "ulp allowance used by 1" in s for s in parity.summary_lines())
    bad = torch.tensor([[5.0 + 3 * 2.0 ** -5, 0.25]], dtype=torch.float64).to(BF16)
    with pytest.raises(AssertionError):
        parity.compare(bad, None, ref, lse_ref, BF16, "planted bad")
    del parity.RECORDS[n0:]
