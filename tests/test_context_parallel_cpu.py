"""Context-parallel prefill host logic on the CPU.

Covers the zigzag sharding, the ring schedule (every visible chunk pair once,
the right mask for each, equal work per rank and step) and the ring exchange
over gloo with world sizes 2 and 4. The per-pair attention and the merge are
injected here as fp64 oracle operations (test infrastructure); on a GPU the
same schedule runs the library's kernels (tests/test_context_parallel_gpu.py).
The expected result is the oracle's attention over the whole sequence: the
ring reaches it exactly up to rounding because softmax over the union of
disjoint key blocks is the LSE merge of the blocks (aikaboom page "11.4d
FlashAttention", "Online Softmax").
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

import oracle
import workloads
from exact_tiled_attention_38_b200 import context_parallel as cp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleOps:
    """fp64 stand-ins for the two kernels the ring calls."""

    def attention(self, q, k, v, scale, causal, o, lse):
        o_ref, lse_ref = oracle.attention_ref(q, k, v, scale, causal)
        o.copy_(torch.from_numpy(o_ref))
        lse.copy_(torch.from_numpy(lse_ref))

    def merge(self, o_acc, lse_acc, o_part, lse_part, o_out):
        acc = o_acc.double().numpy().copy()
        empty = np.isneginf(lse_acc.double().numpy())
        acc[empty] = 0.0  # the accumulator of an empty row is not read
        om, lm = oracle.combine_partials(np.stack([acc, o_part.double().numpy()]),
                                         np.stack([lse_acc.double().numpy(),
                                                   lse_part.double().numpy()]))
        o_acc.copy_(torch.from_numpy(om))
        lse_acc.copy_(torch.from_numpy(lm))
        if o_out is not None:
            o_out.copy_(torch.from_numpy(om))


def _inputs(B, Hq, Hkv, N, d, seed):
    q, k, v = workloads.random_prefill(B, Hq, Hkv, N, N, d, torch.bfloat16, seed=seed)
    return q.double(), k.double(), v.double()


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_zigzag_roundtrip(world):
    x = torch.arange(2 * 3 * (8 * world) * 2, dtype=torch.float64).view(2, 3, 8 * world, 2)
    shards = [cp.shard_zigzag(x, r, world) for r in range(world)]
    assert all(s.shape == (2, 2, 3, 4, 2) and s.is_contiguous() for s in shards)
    assert torch.equal(cp.unshard_zigzag(shards), x)
    # rank r holds chunks r and 2W-1-r
    assert torch.equal(shards[0][0], x[:, :, 0:4])
    assert torch.equal(shards[0][1], x[:, :, (2 * world - 1) * 4:])
    with pytest.raises(ValueError):
        cp.shard_zigzag(x[:, :, :-1], 0, world)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_plan_covers_each_visible_pair_once(world, causal):
    for r in range(world):
        mine = cp.zigzag_chunk_ids(r, world)
        seen = {}
        plan = cp.ring_plan(r, world, causal)
        assert [s.src for s in plan] == [(r - s) % world for s in range(world)]
        for step in plan:
            theirs = cp.zigzag_chunk_ids(step.src, world)
            for qi, ki, kind in step.pairs:
                key = (mine[qi], theirs[ki])
                assert key not in seen
                seen[key] = kind
        want = {}
        for qc in mine:
            for kc in range(2 * world):
                if not causal:
                    want[(qc, kc)] = "full"
                elif kc < qc:
                    want[(qc, kc)] = "full"
                elif kc == qc:
                    want[(qc, kc)] = "diag"
        assert seen == want


@pytest.mark.parametrize("world", [2, 3, 4, 8])
def test_ring_plan_balanced_when_causal(world):
    # work of a step in c x c blocks: a full pair is 1, a diagonal pair 1/2
    for r in range(world):
        for step in cp.ring_plan(r, world, True):
            work = sum(1.0 if kind == "full" else 0.5 for _, _, kind in step.pairs)
            assert work == 2.0


def test_pair_kind():
    assert cp.pair_kind(3, 1, True) == "full"
    assert cp.pair_kind(3, 3, True) == "diag"
    assert cp.pair_kind(3, 5, True) == "skip"
    assert cp.pair_kind(3, 5, False) == "full"


@pytest.mark.parametrize("world,causal", [(1, True), (1, False), (3, True), (2, False)])
def test_ring_attention_local_ring_matches_full_oracle(world, causal):
    B, Hq, Hkv, d = 1, 4, 2, 16
    N = 2 * world * 12
    q, k, v = _inputs(B, Hq, Hkv, N, d, seed=7100 + world)
    scale = d ** -0.5
    ks = [cp.shard_zigzag(k, r, world) for r in range(world)]
    vs = [cp.shard_zigzag(v, r, world) for r in range(world)]
    outs, lses = [], []
    for r in range(world):
        ex = cp.LocalRing(r, ks, vs) if world > 1 else None
        o, lse = cp.ring_attention(cp.shard_zigzag(q, r, world), ks[r], vs[r], causal, scale,
                                   exchange=ex, ops=OracleOps())
        outs.append(o)
        lses.append(lse)
    o_ref, lse_ref = oracle.attention_ref(q, k, v, scale, causal)
    np.testing.assert_allclose(cp.unshard_zigzag(outs).numpy(), o_ref, atol=1e-6, rtol=0)
    np.testing.assert_allclose(cp.unshard_zigzag(lses).numpy(), lse_ref, atol=1e-6, rtol=0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _ring_worker(rank, world, port, causal, out_q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, Hq, Hkv, d = 1, 4, 1, 16
        N = 2 * world * 10
        q, k, v = _inputs(B, Hq, Hkv, N, d, seed=7200 + world)
        ex = cp.RingExchange()
        o, lse = cp.ring_attention(cp.shard_zigzag(q, rank, world), cp.shard_zigzag(k, rank, world),
                                   cp.shard_zigzag(v, rank, world), causal, d ** -0.5,
                                   exchange=ex, ops=OracleOps())
        o_ref, lse_ref = oracle.attention_ref(q, k, v, d ** -0.5, causal)
        mine_o = cp.shard_zigzag(torch.from_numpy(o_ref), rank, world).numpy()
        mine_l = cp.shard_zigzag(torch.from_numpy(lse_ref).unsqueeze(-1), rank, world)[..., 0]
        err_o = float(np.abs(o.numpy() - mine_o).max())
        err_l = float(np.abs(lse.numpy() - mine_l.numpy()).max())
        dist.barrier()
        out_q.put((rank, err_o, err_l))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (4, True), (2, False)])
def test_ring_exchange_over_gloo(world, causal):
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ring_worker, args=(r, world, port, causal, out_q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [out_q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(r for r, _, _ in res) == list(range(world))
    for rank, err_o, err_l in res:
        assert err_o < 1e-6 and err_l < 1e-6, (rank, err_o, err_l)


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(world=st.integers(1, 4), c=st.integers(1, 5), Hkv=st.integers(1, 2),
       group=st.integers(1, 3), causal=st.booleans(), seed=st.integers(0, 1000))
def test_property_ring_matches_full_oracle(world, c, Hkv, group, causal, seed):
    # Any world size and chunk length: every rank's output, put back in order,
    # equals the oracle over the whole sequence.
    N, d = 2 * world * c, 8
    q, k, v = _inputs(1, Hkv * group, Hkv, N, d, seed=seed)
    ks = [cp.shard_zigzag(k, r, world) for r in range(world)]
    vs = [cp.shard_zigzag(v, r, world) for r in range(world)]
    outs, lses = [], []
    for r in range(world):
        ex = cp.LocalRing(r, ks, vs) if world > 1 else None
        o, lse = cp.ring_attention(cp.shard_zigzag(q, r, world), ks[r], vs[r], causal, 0.3,
                                   exchange=ex, ops=OracleOps())
        outs.append(o)
        lses.append(lse)
    o_ref, lse_ref = oracle.attention_ref(q, k, v, 0.3, causal)
    np.testing.assert_allclose(cp.unshard_zigzag(outs).numpy(), o_ref, atol=1e-6, rtol=0)
    np.testing.assert_allclose(cp.unshard_zigzag(lses).numpy(), lse_ref, atol=1e-6, rtol=0)
