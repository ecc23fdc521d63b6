"""Prefill parity: the CUDA path (through the C ABI) against the fp64 oracle.

Covers the single-head fp16 workload, the causal MHA bf16 workload at full size
(every row), the 32K and 128K causal GQA workloads on seeded sampled rows, and
a sweep of ragged and degenerate shapes: tails that are not multiples of the
128-row/128-key tiles, Nq < Nk and Nq > Nk (bottom-right causal, rows with no
visible key), single rows and keys, MQA and GQA groups, d = 64 and 128.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run(eta, q, k, v, scale, causal, want_lse=True):
    fn = eta.attn_fwd_f16 if q.dtype == torch.float16 else eta.attn_fwd
    o, lse = fn(q, k, v, scale=scale, causal=causal, want_lse=want_lse)
    torch.cuda.synchronize()
    code, raw = eta.attn_get_device_status()
    assert code == eta.ATTN_OK, f"device status {code} site {raw:#x}"
    return o, lse


def test_single_head_fp16_workload(lib):
    w = workloads.PREFILL_SMALL
    q, k, v = workloads.prefill_inputs(w)
    o, lse = run(lib, q.to(DEV), k.to(DEV), v.to(DEV), w.scale, w.causal)
    o_ref, lse_ref = oracle.attention_ref(q, k, v, w.scale, w.causal)
    compare(o, lse, o_ref, lse_ref, torch.float16, w.name)


F16, BF16 = torch.float16, torch.bfloat16
SWEEP = [
    # B, Hq, Hkv, Nq, Nk, d, causal, dtype
    (2, 4, 2, 300, 300, 128, True, BF16),
    (2, 4, 2, 300, 300, 128, False, BF16),
    (1, 2, 1, 100, 333, 128, True, BF16),     # Nq < Nk
    (1, 1, 1, 129, 1000, 128, True, BF16),    # offset not a tile multiple
    (1, 2, 2, 257, 130, 128, True, BF16),     # Nq > Nk: rows without keys
    (1, 2, 2, 77, 5, 128, True, BF16),
    (1, 2, 2, 257, 130, 64, False, F16),
    (1, 1, 1, 1, 1, 128, False, BF16),
    (1, 1, 1, 1, 1, 64, True, F16),
    (1, 3, 3, 128, 128, 64, True, BF16),
    (2, 8, 1, 513, 513, 128, True, BF16),     # MQA
    (1, 4, 4, 640, 640, 128, True, F16),
    (1, 2, 2, 2048, 2048, 64, True, BF16),
    (1, 2, 1, 1000, 1000, 128, False, BF16),
    (1, 6, 2, 384, 384, 128, True, BF16),     # group of 3
    (3, 2, 2, 255, 257, 64, True, F16),
]


@pytest.mark.parametrize("shape", SWEEP, ids=lambda s: "x".join(map(str, s[:6])) +
                         ("c" if s[6] else "n") + ("h" if s[7] == F16 else "b"))
def test_prefill_sweep(lib, shape):
    B, Hq, Hkv, Nq, Nk, d, causal, dt = shape
    q, k, v = workloads.random_prefill(B, Hq, Hkv, Nq, Nk, d, dt, seed=1000 + SWEEP.index(shape))
    scale = d ** -0.5
    o, lse = run(lib, q.to(DEV), k.to(DEV), v.to(DEV), scale, causal)
    o_ref, lse_ref = oracle.attention_ref(q, k, v, scale, causal)
    compare(o, lse, o_ref, lse_ref, dt, str(shape))


def test_causal_mha_2k_every_row(lib):
    w = workloads.PREFILL_MHA_2K
    q, k, v = workloads.prefill_inputs(w, device=DEV)
    o, lse = run(lib, q, k, v, w.scale, w.causal)
    o_ref, lse_ref = oracle.attention_ref(q.cpu(), k.cpu(), v.cpu(), w.scale, w.causal)
    compare(o, lse, o_ref, lse_ref, torch.bfloat16, w.name)


def _sampled(lib, w):
    q, k, v = workloads.prefill_inputs(w, device=DEV)
    o, lse = run(lib, q, k, v, w.scale, w.causal)
    rows = workloads.sampled_rows(w)
    ridx = torch.as_tensor(rows, device=DEV)
    o_s = o[:, :, ridx].cpu()
    l_s = lse[:, :, ridx].cpu()
    qs = q[:, :, ridx].cpu()
    del o, lse, q
    kc, vc = k.cpu(), v.cpu()
    del k, v
    torch.cuda.empty_cache()
    o_ref, lse_ref = oracle.attention_ref(qs, kc, vc, w.scale, w.causal, rows=rows, nq=w.Nq)
    return compare(o_s, l_s, o_ref, lse_ref, torch.bfloat16, w.name)


def test_causal_gqa_32k_sampled_rows(lib):
    _sampled(lib, workloads.PREFILL_GQA_32K)


def test_causal_gqa_128k_sampled_rows(lib):
    w = workloads.PREFILL_GQA_128K
    assert 0 in workloads.sampled_rows(w) and w.Nq - 1 in workloads.sampled_rows(w)
    _sampled(lib, w)


def test_bitwise_deterministic_and_lse_optional(lib):
    q, k, v = workloads.random_prefill(2, 4, 2, 700, 700, 128, BF16, seed=7, device=DEV)
    o1, l1 = run(lib, q, k, v, 0.1, True)
    o2, l2 = run(lib, q, k, v, 0.1, True)
    o3, l3 = run(lib, q, k, v, 0.1, True, want_lse=False)
    assert l3 is None
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and torch.equal(o1, o3)


def test_empty_inputs(lib):
    # Nk = 0: every row is empty (O = 0, LSE = -inf); B = 0 / Nq = 0: nothing to do.
    q = torch.randn(1, 2, 10, 64, device=DEV).to(BF16)
    k = torch.empty(1, 2, 0, 64, device=DEV, dtype=BF16)
    o = torch.full_like(q, 7.0)
    lse = torch.zeros(1, 2, 10, device=DEV)
    o, lse = lib.attn_fwd(q, k, k, o=o, lse=lse, causal=True)
    torch.cuda.synchronize()
    assert (o == 0).all() and torch.isneginf(lse).all()
    q0 = torch.empty(0, 2, 10, 64, device=DEV, dtype=BF16)
    lib.attn_fwd(q0, q0, q0)
    qn = torch.empty(1, 2, 0, 64, device=DEV, dtype=BF16)
    kk = torch.randn(1, 2, 5, 64, device=DEV).to(BF16)
    lib.attn_fwd(qn, kk, kk)


def test_rejects_bad_arguments_on_gpu(lib):
    q = torch.randn(1, 2, 16, 128, device=DEV).to(BF16)
    with pytest.raises(lib.AttnError) as e:
        lib.attn_fwd(q, q, q, scale=-1.0)
    assert e.value.code == lib.ATTN_ERR_INVALID
    big = torch.randn(1, 2, 16 * 128 + 8, device=DEV).to(BF16)
    mis = big.view(-1)[4:4 + 2 * 16 * 128].view(1, 2, 16, 128)  # 8-byte aligned only
    with pytest.raises(lib.AttnError) as e:
        lib.attn_fwd(mis, q, q)
    assert e.value.code == lib.ATTN_ERR_INVALID
    q100 = torch.randn(1, 2, 16, 100, device=DEV).to(BF16)
    with pytest.raises(lib.AttnError) as e:
        lib.attn_fwd(q100, q100, q100)
    assert e.value.code == lib.ATTN_ERR_UNSUPPORTED


# The softmax applies a tile's row maximum at the next tile (the running
# reference moves one tile late, exactly, since O and l keep one reference),
# and redoes a tile whose maximum exceeds the reference by more than 32 in
# log2 units. These inputs make the maximum grow at every key tile, or jump.
MAX_CASES = [
    # B, Hq, Hkv, N, d, causal, dtype, kind
    (1, 4, 2, 1000, 128, True, BF16, "ramp"),
    (1, 4, 2, 1000, 64, True, BF16, "ramp"),
    (1, 2, 2, 700, 128, False, F16, "ramp"),
    (1, 4, 2, 1000, 128, True, BF16, "jump"),
    (1, 4, 4, 900, 64, False, BF16, "jump"),
    (2, 2, 1, 600, 64, True, F16, "drop"),
]


@pytest.mark.parametrize("case", MAX_CASES, ids=lambda c: "x".join(map(str, c[:5])) + c[7])
def test_row_maximum_moves(lib, case):
    B, Hq, Hkv, N, d, causal, dt, kind = case
    q, k, v = workloads.random_prefill(B, Hq, Hkv, N, N, d, dt, seed=1300 + MAX_CASES.index(case))
    pos = torch.arange(N, dtype=torch.float32)
    if kind == "ramp":      # every 128-key tile raises the maxima by well over 8 (log2 units)
        f = 1.0 + pos / 40.0
    elif kind == "jump":    # keys from 300 on are 40 times larger: a jump far beyond 32
        f = torch.where(pos >= 300, 40.0, 1.0)
    else:                   # large early keys, then small ones: the reference stays high
        f = torch.where(pos < 200, 12.0, 1.0)
    k = (k.float() * f[None, None, :, None]).to(dt)
    # Peaked rows put O close to single value rows; small values keep |O| in
    # the range where the stated bounds apply (this test is about the maxima).
    v = (v.float() * 0.25).to(dt)
    scale = d ** -0.5
    o, lse = run(lib, q.to(DEV), k.to(DEV), v.to(DEV), scale, causal)
    o_ref, lse_ref = oracle.attention_ref(q, k, v, scale, causal)
    compare(o, lse, o_ref, lse_ref, dt, f"moving maximum {case}")
