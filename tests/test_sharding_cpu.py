"""Data-parallel partition of one workload over ranks (CPU, gloo world size 2).

Prefill is split by (batch, KV head) and decode by sequence
(`exact_tiled_attention_38_b200.sharding`). Each rank here runs the fp64
oracle on its shard, exactly as a GPU rank would run one library call on it;
the gathered shards must equal the unsharded oracle result, and the index
arithmetic (coverage, contiguity, balance) is checked on its own.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from exact_tiled_attention_38_b200 import sharding  # noqa: E402


def test_split_even_covers_every_unit_once():
    for n in range(0, 23):
        for world in range(1, 6):
            spans = [sharding.split_even(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1


def test_prefill_shard_views_are_the_units_heads():
    B, Hq, Hkv, N, d = 3, 6, 2, 5, 8
    q = torch.arange(B * Hq * N * d, dtype=torch.float32).reshape(B, Hq, N, d)
    k = -torch.arange(B * Hkv * N * d, dtype=torch.float32).reshape(B, Hkv, N, d)
    G = Hq // Hkv
    seen = []
    for r in range(4):
        qs, ks, vs, (u0, u1) = sharding.prefill_shard(q, k, k, 4, r)
        assert qs.is_contiguous() and ks.is_contiguous()
        assert qs.shape == (1, (u1 - u0) * G, N, d) and ks.shape == (1, u1 - u0, N, d)
        for i, u in enumerate(range(u0, u1)):
            b, g = divmod(u, Hkv)
            assert torch.equal(ks[0, i], k[b, g])
            for j in range(G):  # query head h of the shard reads its KV head h // G
                assert torch.equal(qs[0, i * G + j], q[b, g * G + j])
            seen.append(u)
    assert seen == list(range(B * Hkv))


def test_decode_cuts_cover_and_balance_tokens():
    gen = np.random.default_rng(5)
    for _ in range(50):
        B = int(gen.integers(1, 40))
        lens = gen.integers(-2, 300, size=B)
        for world in (1, 2, 3, 8):
            cuts = sharding.decode_cuts(lens, world)
            assert cuts[0] == 0 and cuts[-1] == B and len(cuts) == world + 1
            assert all(a <= b for a, b in zip(cuts, cuts[1:]))
            pos = np.clip(lens, 0, None)
            share = [pos[cuts[r]:cuts[r + 1]].sum() for r in range(world)]
            # each rank is within one sequence of an equal share of the tokens
            assert max(share) <= pos.sum() / world + pos.max(initial=0) + 1e-9


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import oracle
    import workloads
    from exact_tiled_attention_38_b200 import sharding as sh

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # prefill: causal GQA, 3 batches x 4 KV heads (group 2), split by unit
        B, Hq, Hkv, N, d = 3, 8, 4, 40, 16
        q, k, v = workloads.random_prefill(B, Hq, Hkv, N, N, d, torch.bfloat16, seed=77)
        qs, ks, vs, units = sh.prefill_shard(q, k, v, world, rank)
        o_s, l_s = oracle.attention_ref(qs, ks, vs, d ** -0.5, True)
        pre = [None] * world
        dist.all_gather_object(pre, (units, o_s, l_s))
        # decode: ragged cache split by sequence at equal token shares
        lens = torch.tensor([17, 0, 90, 3, 44, 61, 1], dtype=torch.int32)
        dq, kc, vc, sl = workloads.random_decode(7, 8, 2, 16, lens, torch.bfloat16, seed=78)
        qd, kcs, vcs, sls, seqs = sh.decode_shard(dq, kc, vc, lens.tolist(), 2, world, rank,
                                                  seqlens_dev=lens)
        od, ld = oracle.decode_ref(qd, kcs, vcs, sls, 16 ** -0.5, 2)
        dec = [None] * world
        dist.all_gather_object(dec, (seqs, od, ld))
        if rank == 0:
            out.put((pre, dec))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gathered_shards_equal_the_unsharded_oracle():
    import oracle
    import workloads

    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    pre, dec = out.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    B, Hq, Hkv, N, d = 3, 8, 4, 40, 16
    G = Hq // Hkv
    q, k, v = workloads.random_prefill(B, Hq, Hkv, N, N, d, torch.bfloat16, seed=77)
    o_ref, l_ref = oracle.attention_ref(q, k, v, d ** -0.5, True)
    o = np.full(o_ref.shape, np.nan)
    lse = np.full(l_ref.shape, np.nan)
    for units, o_s, l_s in pre:
        u0, u1 = units
        o.reshape(B * Hq, N, d)[u0 * G:u1 * G] = o_s[0]
        lse.reshape(B * Hq, N)[u0 * G:u1 * G] = l_s[0]
    assert sorted(u for units, _, _ in pre for u in range(*units)) == list(range(B * Hkv))
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(lse, l_ref)

    lens = torch.tensor([17, 0, 90, 3, 44, 61, 1], dtype=torch.int32)
    dq, kc, vc, sl = workloads.random_decode(7, 8, 2, 16, lens, torch.bfloat16, seed=78)
    od_ref, ld_ref = oracle.decode_ref(dq, kc, vc, lens, 16 ** -0.5, 2)
    od = np.full(od_ref.shape, np.nan)
    ld = np.full(ld_ref.shape, np.nan)
    for (b0, b1), o_s, l_s in dec:
        od[b0:b1] = o_s
        ld[b0:b1] = l_s
    np.testing.assert_array_equal(od, od_ref)
    np.testing.assert_array_equal(ld, ld_ref)


def test_prefill_place_inverts_the_shard():
    B, Hq, Hkv, N, d = 2, 4, 2, 3, 8
    G = Hq // Hkv
    full = torch.randn(B, Hq, N, d)
    lse = torch.randn(B, Hq, N)
    o = torch.zeros_like(full)
    lo = torch.zeros_like(lse)
    for r in range(3):
        qs, _, _, units = sharding.prefill_shard(full, full[:, :Hkv], full[:, :Hkv], 3, r)
        ls = lse.reshape(B * Hq, N)[units[0] * G:units[1] * G].unsqueeze(0)
        sharding.prefill_place(o, lo, qs, ls, units, G)
    assert torch.equal(o, full) and torch.equal(lo, lse)


def test_bad_arguments():
    with pytest.raises(ValueError):
        sharding.split_even(4, 0, 0)
    with pytest.raises(ValueError):
        sharding.prefill_units(1, 6, 4, 2, 0)
