"""The data-parallel partition run through the CUDA library on one GPU.

Each shard of `exact_tiled_attention_38_b200.sharding` is one library call, as
it would be on its own GPU. Prefill shards by (batch, KV head) must give
bit-for-bit the unsharded call's output (every (batch, head) is computed by
the same tile sequence wherever it runs); decode shards by sequence are
checked against the fp64 oracle (their split counts differ from the
unsharded call's, so only rounding may differ).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from exact_tiled_attention_38_b200 import sharding
from parity import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("world", [2, 3, 8])
def test_prefill_shards_bitwise_equal_whole_call(lib, world):
    B, Hq, Hkv, N, d = 2, 16, 4, 700, 128
    q, k, v = workloads.random_prefill(B, Hq, Hkv, N, N, d, torch.bfloat16, seed=91, device=DEV)
    o_all, l_all = lib.attn_fwd(q, k, v, causal=True)
    o = torch.full_like(o_all, float("nan"))
    lse = torch.full_like(l_all, float("nan"))
    G = Hq // Hkv
    for r in range(world):
        qs, ks, vs, units = sharding.prefill_shard(q, k, v, world, r)
        if qs.shape[1] == 0:
            continue
        os_, ls_ = lib.attn_fwd(qs, ks, vs, causal=True)
        sharding.prefill_place(o, lse, os_, ls_, units, G)
    torch.cuda.synchronize()
    assert torch.equal(o, o_all) and torch.equal(lse, l_all)


def test_decode_shards_match_the_oracle(lib):
    w = workloads.DECODE_GQA_RAGGED
    q, kc, vc, sl = workloads.decode_inputs(w, device=DEV)
    lens = sl.cpu().tolist()
    world = 4
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.Hq), float("nan"), device=DEV)
    for r in range(world):
        qs, kcs, vcs, sls, (b0, b1) = sharding.decode_shard(q, kc, vc, lens, w.Hkv, world, r,
                                                            seqlens_dev=sl)
        os_, ls_ = lib.attn_decode(qs, kcs, vcs, sls, w.Hkv)
        o[b0:b1] = os_
        lse[b0:b1] = ls_
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.decode_ref(q.cpu(), kc.cpu(), vc.cpu(), sl.cpu(), w.scale, w.Hkv)
    compare(o, lse, o_ref, l_ref, torch.bfloat16, f"{w.name} in {world} shards")
    shares = [sum(lens[c0:c1]) for c0, c1 in zip(*(lambda c: (c[:-1], c[1:]))(
        sharding.decode_cuts(lens, world)))]
    assert max(shares) <= sum(lens) / world + max(lens)
    assert np.isfinite(lse.cpu().numpy()).all()
