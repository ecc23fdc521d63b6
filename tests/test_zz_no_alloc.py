"""attn_decode_noalloc: decode with the scratch in a fixed library array.

Some callers cannot allocate device memory where they run decode (an engine
that has handed almost all of HBM to its own KV-cache pool, a latency-critical
path where an allocator call may lock or synchronise, a runtime whose memory
plan is fixed up front). The no-allocation entry point serves them; these tests
check, through the C ABI, that it gives the allocating entry point's results
within the parity tolerances on consecutive calls, that a later call is not
affected by what an earlier one left in the shared scratch, and that sizes the
scratch cannot hold are refused with their own error code.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import TOL_LSE, TOL_O, compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _agree(o, lse, o_ref, lse_ref):
    d_o = (o.float() - o_ref.float()).abs().max().item()
    fin = torch.isfinite(lse_ref)
    assert torch.equal(torch.isfinite(lse), fin)
    d_l = (lse[fin] - lse_ref[fin]).abs().max().item() if fin.any() else 0.0
    assert d_o <= TOL_O[torch.bfloat16], d_o
    assert d_l <= TOL_LSE, d_l


def _call_pair(lib, q, kc, vc, sl, Hkv):
    o_ref, lse_ref = lib.attn_decode(q, kc, vc, sl, Hkv=Hkv)
    for _ in range(2):  # two calls in a row, fresh outputs each time
        o = torch.full_like(q, float("nan"))
        lse = torch.full(lse_ref.shape, float("nan"), device=DEV)
        lib.attn_decode_noalloc(q, kc, vc, sl, Hkv=Hkv, o=o, lse=lse)
        torch.cuda.synchronize()
        assert lib.attn_get_device_status()[0] == lib.ATTN_OK
        _agree(o, lse, o_ref, lse_ref)


def test_noalloc_matches_allocating_decode_on_ragged_workload(lib):
    w = workloads.DECODE_GQA_RAGGED
    q, kc, vc, sl = workloads.decode_inputs(w, device=DEV)
    _call_pair(lib, q, kc, vc, sl, w.Hkv)


def test_noalloc_after_a_larger_call_and_with_empty_sequences(lib):
    # A smaller problem after the big one: stale scratch contents must not leak.
    sl = torch.tensor([5, 0, 1300, 64], dtype=torch.int32)
    q, kc, vc, sl = workloads.random_decode(4, 16, 2, 64, sl, torch.bfloat16, seed=31,
                                            device=DEV)
    _call_pair(lib, q, kc, vc, sl, 2)


def _oracle_sample(q, kc, vc, sl, Hkv, o, lse, seqs, what):
    """Compare sequences `seqs` of a no-alloc result with the fp64 oracle."""
    lens = sl.cpu().tolist()
    offs = np.concatenate([[0], np.cumsum(lens)])
    d = q.shape[-1]
    per = Hkv * d
    qc, kcc, vcc = q.cpu(), kc.cpu(), vc.cpu()
    for b in seqs:
        a, e = int(offs[b]) * per, int(offs[b + 1]) * per
        o_ref, l_ref = oracle.decode_ref(qc[b:b + 1], kcc[a:e], vcc[a:e], sl.cpu()[b:b + 1],
                                         d ** -0.5, Hkv)
        compare(o[b:b + 1], lse[b:b + 1], o_ref, l_ref, torch.bfloat16, f"{what} seq {b}")


def test_noalloc_persistent_partials_fill_most_of_the_scratch(lib):
    # The persistent pass (d = 128, 2..32 query heads per KV head) keeps its
    # plan and the partials of segments cut between CTAs in the scratch:
    # (B * Hkv + CTAs - 1) slots of G rows of d + 1 floats, one CTA per SM.
    # B=44, Hq=256, Hkv=8 (group 32) needs about 7.9 MiB of the 8 MiB.
    B, Hq, Hkv, d = 44, 256, 8, 128
    G = Hq // Hkv
    slots = B * Hkv + torch.cuda.get_device_properties(0).multi_processor_count - 1
    assert slots * G * (d + 1) < 2_097_152 < (slots + 40) * G * (d + 1)
    sl = workloads.decode_seqlens(B, 1, 3000, 47)
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, torch.bfloat16, seed=47,
                                            device=DEV)
    _call_pair(lib, q, kc, vc, sl, Hkv)
    o, lse = lib.attn_decode_noalloc(q, kc, vc, sl, Hkv=Hkv)
    torch.cuda.synchronize()
    _oracle_sample(q, kc, vc, sl, Hkv, o, lse, range(0, B, 5), "noalloc persistent group 32")


def test_noalloc_tensor_core_single_split_beyond_scratch(lib):
    # Groups of 2..32 heads at d = 128 run on the persistent pass, whose
    # partials would need (4096 * 4 + 147) * 8 * 129 floats here, about 8 times
    # the array: every CTA then takes whole segments and writes its results
    # directly, with only the per-sequence plan in the scratch.
    B, Hq, Hkv, d = 4096, 32, 4, 128
    assert B * Hq * (d + 1) > 2_097_152
    assert lib.attn_decode_num_splits(B, Hq, Hkv, d) == 1
    sl = workloads.decode_seqlens(B, 0, 48, 53)
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, torch.bfloat16, seed=53,
                                            device=DEV)
    _call_pair(lib, q, kc, vc, sl, Hkv)
    o, lse = lib.attn_decode_noalloc(q, kc, vc, sl, Hkv=Hkv)
    torch.cuda.synchronize()
    _oracle_sample(q, kc, vc, sl, Hkv, o, lse, range(0, B, 61), "noalloc tensor-core B=4096")


def test_noalloc_refuses_sizes_beyond_its_scratch(lib):
    # B * Hq * (d + 1) floats per split on the CUDA-core pass (one query head
    # per KV head); 16384 * 8 * 129 is above 2,097,152.
    B, Hq, Hkv, d = 16384, 8, 8, 128
    q = torch.zeros(B, Hq, d, device=DEV, dtype=torch.bfloat16)
    kc = torch.zeros(64, device=DEV, dtype=torch.bfloat16)
    sl = torch.zeros(B, device=DEV, dtype=torch.int32)
    with pytest.raises(lib.AttnError) as e:
        lib.attn_decode_noalloc(q, kc, kc, sl, Hkv=Hkv)
    assert e.value.code == lib.ATTN_ERR_SCRATCH


@pytest.mark.parametrize("B,Hq,Hkv,lens", [
    (3, 32, 4, [2000, 10, 700]),   # persistent pass, one segment cut over many CTAs
    (40, 64, 8, None),             # persistent pass, short segments mostly whole in one CTA
])
def test_noalloc_tensor_core_groups(lib, B, Hq, Hkv, lens):
    sl = torch.tensor(lens, dtype=torch.int32) if lens else workloads.decode_seqlens(B, 0, 400, 41)
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, 128, sl, torch.bfloat16, seed=43,
                                            device=DEV)
    _call_pair(lib, q, kc, vc, sl, Hkv)


@pytest.mark.parametrize("B,Hq,Hkv,d", [
    (3000, 1, 1, 128),    # CUDA-core split pass: offsets, then a few splits in the scratch
    (20000, 4, 2, 96),    # generic kernel: only the offsets in the scratch
    (20000, 16, 2, 128),  # persistent pass: plan only, whole segments per CTA
])
def test_noalloc_large_batch_offsets(lib, B, Hq, Hkv, d):
    # Above 1024 sequences the token offsets come from one prefix sum per call,
    # kept in the scratch ahead of whatever else the pass needs there.
    sl = workloads.decode_seqlens(B, 0, 48, 57)
    sl[::11] = 0
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, torch.bfloat16, seed=59,
                                            device=DEV)
    _call_pair(lib, q, kc, vc, sl, Hkv)
    o, lse = lib.attn_decode_noalloc(q, kc, vc, sl, Hkv=Hkv)
    torch.cuda.synchronize()
    _oracle_sample(q, kc, vc, sl, Hkv, o, lse, list(range(0, B, 97)) + [B - 1],
                   f"noalloc B={B} d={d}")
