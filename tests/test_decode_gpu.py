"""Decode parity: split-KV decode + LSE combine against the fp64 oracle.

Covers the ragged GQA workload at full size (64 sequences, lengths uniform in
[1024, 8192]) and small cases: length 1, empty sequences, lengths that are not
multiples of the 32-key stage, MQA (one KV head for 32 query heads), MHA, a
group of 3 (padded to 4), group 8, d = 64 and fp16, a single long sequence
spread over many splits.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run(eta, q, kc, vc, sl, Hkv, scale, want_lse=True):
    fn = eta.attn_decode_f16 if q.dtype == torch.float16 else eta.attn_decode
    o, lse = fn(q, kc, vc, sl, Hkv=Hkv, scale=scale, want_lse=want_lse)
    torch.cuda.synchronize()
    code, raw = eta.attn_get_device_status()
    assert code == eta.ATTN_OK, f"device status {code} site {raw:#x}"
    return o, lse


def test_ragged_gqa_workload(lib):
    w = workloads.DECODE_GQA_RAGGED
    q, kc, vc, sl = workloads.decode_inputs(w, device=DEV)
    o, lse = run(lib, q, kc, vc, sl, w.Hkv, w.scale)
    o_ref, lse_ref = oracle.decode_ref(q.cpu(), kc.cpu(), vc.cpu(), sl.cpu(), w.scale, w.Hkv)
    compare(o, lse, o_ref, lse_ref, torch.bfloat16, w.name)


F16, BF16 = torch.float16, torch.bfloat16
CASES = [
    # B, Hq, Hkv, d, lengths, dtype
    (4, 8, 2, 128, [1, 37, 300, 0], BF16),
    (3, 4, 4, 64, [33, 64, 65], F16),          # MHA (group 1, padded)
    (2, 6, 2, 128, [500, 31], BF16),           # group 3 (padded to 4)
    (2, 32, 1, 128, [777, 1], BF16),           # MQA: 32 query heads per KV head
    (3, 16, 2, 64, [129, 2, 4096], BF16),      # group 8
    (2, 8, 8, 128, [0, 0], BF16),              # every sequence empty
    (1, 8, 2, 128, [20000], F16),              # one long sequence over many splits
    (5, 12, 4, 128, [1, 2, 3, 4, 5], BF16),
    (2, 12, 2, 64, [300, 1000], F16),          # group 6: one full chunk of 4, one of 2
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}h{c[1]}kv{c[2]}d{c[3]}")
def test_decode_cases(lib, case):
    B, Hq, Hkv, d, lens, dt = case
    sl = torch.tensor(lens, dtype=torch.int32)
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, dt, seed=2000 + CASES.index(case))
    scale = d ** -0.5
    if kc.numel() == 0:  # the ABI wants real (non-null) cache pointers even when unused
        kc = vc = torch.zeros(64, dtype=dt)
    o, lse = run(lib, q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), Hkv, scale)
    o_ref, lse_ref = oracle.decode_ref(q, kc, vc, sl, scale, Hkv)
    compare(o, lse, o_ref, lse_ref, dt, str(case))


def test_decode_deterministic_and_lse_optional(lib):
    sl = torch.tensor([1000, 3000, 17], dtype=torch.int32)
    q, kc, vc, sl = workloads.random_decode(3, 32, 8, 128, sl, BF16, seed=9, device=DEV)
    o1, l1 = run(lib, q, kc, vc, sl, 8, 0.08)
    o2, l2 = run(lib, q, kc, vc, sl, 8, 0.08)
    o3, l3 = run(lib, q, kc, vc, sl, 8, 0.08, want_lse=False)
    assert l3 is None
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and torch.equal(o1, o3)


def test_decode_matches_prefill_single_query(lib):
    # decode of one sequence equals prefill with Nq = 1 over the same keys
    L, Hq, Hkv, d = 700, 8, 2, 128
    sl = torch.tensor([L], dtype=torch.int32)
    q, kc, vc, sl = workloads.random_decode(1, Hq, Hkv, d, sl, BF16, seed=11, device=DEV)
    o, lse = run(lib, q, kc, vc, sl, Hkv, 0.09)
    k4 = kc.view(1, Hkv, L, d)
    v4 = vc.view(1, Hkv, L, d)
    op, lp = lib.attn_fwd(q.view(1, Hq, 1, d).contiguous(), k4, v4, scale=0.09, causal=False)
    torch.cuda.synchronize()
    assert (o.float() - op.view(1, Hq, d).float()).abs().max().item() <= 2 * 2 ** -8
    assert (lse - lp.view(1, Hq)).abs().max().item() <= 1e-4


def test_decode_rejects_bad_arguments(lib):
    q = torch.randn(2, 6, 128, device=DEV).to(BF16)
    kc = torch.randn(4 * 128 * 4, device=DEV).to(BF16)
    sl = torch.tensor([1, 1], dtype=torch.int32, device=DEV)
    with pytest.raises(lib.AttnError) as e:
        lib.attn_decode(q, kc, kc, sl, Hkv=4)  # 6 % 4 != 0
    assert e.value.code == lib.ATTN_ERR_INVALID
    with pytest.raises(lib.AttnError) as e:
        lib.attn_decode(q, kc, kc, sl, Hkv=2, scale=float("nan"))
    assert e.value.code == lib.ATTN_ERR_INVALID
