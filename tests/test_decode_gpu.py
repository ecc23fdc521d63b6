"""Decode parity: split-KV decode + LSE combine against the fp64 oracle.

Covers the ragged GQA workload at full size (64 sequences, lengths uniform in
[1024, 8192]) and small cases: length 1, empty sequences, lengths that are not
multiples of the 32-key stage, MQA (one KV head for 32 query heads), MHA, a
group of 3 (padded to 4), group 8, d = 64 and fp16, a single long sequence
spread over many splits; for the persistent tensor-core pass (groups of 2 to
32 with d = 128), tile tails, padded groups, MQA, the workload's scale with
groups of 8, keys that move the running maximum at every tile, and segments
cut between CTAs; bitwise repeatability of the persistent pass over many calls
on ragged workloads; and batches of twenty thousand short sequences, whose
token offsets come from one prefix sum per call, on every decode path.
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


# Groups of 2 to 32 query heads per KV head with d = 128 take the persistent
# tensor-core pass (scores and P V as tcgen05 products, keys on tensor-memory
# lanes).
TC_CASES = [
    # B, Hq, Hkv, d, lengths, dtype
    (4, 16, 2, 128, [1, 127, 128, 129], BF16),         # tile tails around 128 keys
    (3, 32, 4, 128, [5000, 0, 260], F16),              # group 8, long + empty
    (2, 32, 2, 128, [2049, 777], BF16),                # group 16 (no padding)
    (2, 48, 2, 128, [1500, 300], BF16),                # group 24 (padded to 32)
    (2, 32, 1, 128, [4100, 64], F16),                  # MQA, group 32
    (64, 64, 8, 128, "ragged", BF16),                  # group 8 at the workload's scale
]


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: f"B{c[0]}h{c[1]}kv{c[2]}")
def test_decode_tensor_core_groups(lib, case):
    B, Hq, Hkv, d, lens, dt = case
    if lens == "ragged":
        sl = workloads.decode_seqlens(B, 1024, 8192, 2300)
    else:
        sl = torch.tensor(lens, dtype=torch.int32)
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, dt,
                                            seed=2100 + TC_CASES.index(case))
    scale = d ** -0.5
    o, lse = run(lib, q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), Hkv, scale)
    o_ref, lse_ref = oracle.decode_ref(q, kc, vc, sl, scale, Hkv)
    compare(o, lse, o_ref, lse_ref, dt, str(case[:4]))


def test_decode_tensor_core_running_max_moves(lib):
    # Keys grow along each sequence, so every 128-key tile raises the heads'
    # maxima by far more than the lazy-rescale threshold (8 in log2 units) and
    # the accumulated O^T is rescaled in tensor memory tile after tile.
    B, Hq, Hkv, d = 2, 16, 2, 128
    sl = torch.tensor([1300, 700], dtype=torch.int32)
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, BF16, seed=2200)
    rows = []
    for b in range(B):
        L = int(sl[b])
        ramp = 1.0 + torch.arange(L, dtype=torch.float32) / 40.0
        rows.append(ramp.repeat(Hkv))
    kc = (kc.float().view(-1, d) * torch.cat(rows)[:, None]).to(BF16).view(kc.shape)
    o, lse = run(lib, q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), Hkv, d ** -0.5)
    o_ref, lse_ref = oracle.decode_ref(q, kc, vc, sl, d ** -0.5, Hkv)
    compare(o, lse, o_ref, lse_ref, BF16, "growing keys")


def test_decode_tensor_core_single_split_writes_output(lib):
    # Many short segments: most are whole in one CTA, whose epilogue writes O
    # and LSE itself (no partials). Includes empty and very short sequences,
    # fp16, and the call without LSE.
    B, Hq, Hkv, d = 40, 64, 8, 128
    sl = workloads.decode_seqlens(B, 0, 300, 2400)
    sl[3] = 0
    sl[7] = 1
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, F16, seed=2401)
    assert lib.attn_decode_num_splits(B, Hq, Hkv, d) == 1
    args = (q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), Hkv, d ** -0.5)
    o, lse = run(lib, *args)
    o_ref, lse_ref = oracle.decode_ref(q, kc, vc, sl, d ** -0.5, Hkv)
    compare(o, lse, o_ref, lse_ref, F16, "single split")
    o2, none = run(lib, *args, want_lse=False)
    assert none is None and torch.equal(o, o2)


# The persistent pass divides all (sequence, KV head) tiles of 128 keys into
# equal contiguous ranges, one per CTA; segments cut between CTAs are merged by
# the gather kernel. These cases stress the cuts.
PS_CASES = [
    # B, Hq, Hkv, d, lengths, dtype
    (1, 8, 1, 128, [1000], BF16),                 # 8 tiles over every CTA: most CTAs own none
    (3, 32, 2, 128, [70000, 5, 300], BF16),       # one long segment cut over many CTAs
    (300, 16, 2, 128, "short", F16),              # many short sequences, empties between
    (64, 32, 1, 128, "ragged", BF16),             # MQA at the workload's scale
    (64, 128, 8, 128, "ragged", BF16),            # group 16 at the workload's scale
    # d = 64: the same pass with a 64-dim K tile and the P V product's upper
    # 64 rows reading a zeroed box
    (5, 6, 3, 64, [1, 127, 128, 129, 0], BF16),   # group 2, tile tails
    (1, 8, 1, 64, [1000], F16),                   # group 8, most CTAs own no tile
    (3, 32, 2, 64, [70000, 5, 300], F16),         # group 16, one segment cut over many CTAs
    (300, 8, 2, 64, "short", BF16),               # group 4, many short sequences
    (64, 32, 1, 64, "ragged", BF16),              # MQA at the workload's scale
    (64, 32, 8, 64, "ragged", BF16),              # group 4 at the workload's scale
]


@pytest.mark.parametrize("case", PS_CASES, ids=lambda c: f"B{c[0]}h{c[1]}kv{c[2]}d{c[3]}")
def test_decode_persistent_cuts(lib, case):
    B, Hq, Hkv, d, lens, dt = case
    if lens == "short":
        sl = workloads.decode_seqlens(B, 0, 200, 2500)
        sl[::7] = 0
    elif lens == "ragged":
        sl = workloads.decode_seqlens(B, 1024, 8192, 2501)
    else:
        sl = torch.tensor(lens, dtype=torch.int32)
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, dt,
                                            seed=2600 + PS_CASES.index(case))
    scale = d ** -0.5
    o, lse = run(lib, q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), Hkv, scale)
    o2, lse2 = run(lib, q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), Hkv, scale)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)  # fixed assignment: bitwise repeatable
    o_ref, lse_ref = oracle.decode_ref(q, kc, vc, sl, scale, Hkv)
    compare(o, lse, o_ref, lse_ref, dt, f"persistent {case[:4]}")


# Repeated calls on the same inputs must give bitwise-identical outputs: the
# persistent pass's tile assignment is fixed, so any difference is a race
# (for instance an end-of-piece wait that passes before the last P V product
# has run). Ragged workloads at full scale, where the K/V copies, the softmax
# and the products overlap the most.
REPEAT_CASES = [
    # B, Hq, Hkv, d, dtype
    (64, 32, 8, 128, BF16),   # group 4 (the bench's decode workload shape)
    (64, 64, 8, 128, BF16),   # group 8
    (64, 32, 8, 64, BF16),    # group 4, d = 64
    (64, 32, 1, 128, F16),    # MQA
]


@pytest.mark.parametrize("case", REPEAT_CASES, ids=lambda c: f"B{c[0]}h{c[1]}kv{c[2]}d{c[3]}")
def test_decode_persistent_repeatable(lib, case):
    B, Hq, Hkv, d, dt = case
    sl = workloads.decode_seqlens(B, 1024, 8192, 2800 + REPEAT_CASES.index(case))
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, dt,
                                            seed=2810 + REPEAT_CASES.index(case), device=DEV)
    scale = d ** -0.5
    o1, l1 = run(lib, q, kc, vc, sl, Hkv, scale)
    for _ in range(12):
        o, l = run(lib, q, kc, vc, sl, Hkv, scale)
        assert torch.equal(o, o1) and torch.equal(l, l1), f"decode {case[:4]}: outputs differ"


# Batches above 1024 sequences: each sequence's offset in the packed cache
# comes from one prefix-sum kernel per call (the plan kernel on the persistent
# pass above 2048 sequences) instead of each CTA summing the lengths before its
# own; up to 2048 sequences the persistent pass's CTAs scan the lengths
# themselves (several per thread at 2048).
BIG_B_CASES = [
    # B, Hq, Hkv, d, dtype; lengths uniform in [0, 48], every 11th empty
    (20000, 4, 4, 128, BF16),   # MHA: CUDA-core split pass
    (20000, 4, 4, 64, F16),     # d = 64, MHA: CUDA-core split pass
    (20000, 8, 2, 64, BF16),    # d = 64, group 4: persistent pass
    (20000, 4, 2, 96, BF16),    # d = 96: generic kernel
    (20000, 16, 2, 128, BF16),  # group 8: persistent pass (plan kernel)
    (2048, 16, 2, 128, BF16),   # group 8: the largest batch whose CTAs find their ranges themselves
    (2048, 32, 1, 64, F16),     # MQA, d = 64, the same
]


def big_batch(case, seed):
    B, Hq, Hkv, d, dt = case
    sl = workloads.decode_seqlens(B, 0, 48, seed)
    sl[::11] = 0
    return workloads.random_decode(B, Hq, Hkv, d, sl, dt, seed=seed + 1)


@pytest.mark.parametrize("case", BIG_B_CASES, ids=lambda c: f"B{c[0]}h{c[1]}kv{c[2]}d{c[3]}")
def test_decode_large_batch_offsets(lib, case):
    B, Hq, Hkv, d, dt = case
    q, kc, vc, sl = big_batch(case, 2700 + BIG_B_CASES.index(case))
    scale = d ** -0.5
    o, lse = run(lib, q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), Hkv, scale)
    o_ref, lse_ref = oracle.decode_ref(q, kc, vc, sl, scale, Hkv)
    compare(o, lse, o_ref, lse_ref, dt, f"large batch {case[:4]}")
