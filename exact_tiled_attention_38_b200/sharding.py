"""Partition of one attention workload over several GPUs (data parallel).

The hot path has no exchange step when it is split along independent units,
so each GPU computes its shard end to end with one library call and no
collective on the data path:

  * prefill by (batch, KV head): a KV head and the group of Hq / Hkv query
    heads that read it (the GQA grouping of the sicorps page's last
    paragraph) form one unit; units are numbered u = b * Hkv + g, and a rank
    takes a contiguous run of them. In the BHSD layout a contiguous unit run
    is one contiguous block of q / o rows ([u0 * G, u1 * G) of the B * Hq
    heads) and of k / v ([u0, u1) of the B * Hkv heads), so the shard is a
    single attn_fwd call with B = 1, Hq = n * G, Hkv = n (query head h of the
    shard reads its KV head h / G, the same map as the whole problem).
  * decode by sequence: a rank takes a contiguous run of sequences
    [b0, b1); in the packed cache their keys and values are one contiguous
    slice (tokens sum(L[:b0]) .. sum(L[:b1]) times Hkv * d elements), so the
    shard is a single attn_decode call on views. Runs are cut at equal shares
    of the total cached tokens, which is the decode work (the first page:
    generating a token re-reads the whole cache of its sequence).

Only index arithmetic and tensor views live here; every number is computed
by the library's kernels.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple


def split_even(n: int, world: int, rank: int) -> Tuple[int, int]:
    """[lo, hi) of `n` equal-cost units for `rank` of `world` (sizes differ by <= 1)."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad split")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def prefill_units(B: int, Hq: int, Hkv: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous (batch, KV-head) units [u0, u1) of rank `rank`; u = b * Hkv + g."""
    if Hkv < 1 or Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return split_even(B * Hkv, world, rank)


def prefill_shard(q, k, v, world: int, rank: int):
    """Views of q [B,Hq,Nq,d], k, v [B,Hkv,Nk,d] for this rank's units, shaped
    as one attn_fwd problem: q [1, n*G, Nq, d], k, v [1, n, Nk, d]. Also
    returns (u0, u1) so results can be placed back (`prefill_place`)."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    u0, u1 = prefill_units(B, Hq, Hkv, world, rank)
    qs = q.reshape(B * Hq, Nq, d)[u0 * G:u1 * G].unsqueeze(0)
    ks = k.reshape(B * Hkv, Nk, d)[u0:u1].unsqueeze(0)
    vs = v.reshape(B * Hkv, Nk, d)[u0:u1].unsqueeze(0)
    return qs, ks, vs, (u0, u1)


def prefill_place(full_o, full_lse, shard_o, shard_lse, units, G: int):
    """Write a shard's o [1, n*G, Nq, d] and lse [1, n*G, Nq] into the whole
    problem's o [B,Hq,Nq,d] and lse [B,Hq,Nq]."""
    u0, u1 = units
    B, Hq, Nq, d = full_o.shape
    full_o.reshape(B * Hq, Nq, d)[u0 * G:u1 * G] = shard_o[0]
    if full_lse is not None:
        full_lse.reshape(B * Hq, Nq)[u0 * G:u1 * G] = shard_lse[0]


def decode_cuts(seqlens: Sequence[int], world: int) -> List[int]:
    """Sequence boundaries b_0 = 0 <= b_1 <= ... <= b_world = B: rank r takes
    sequences [b_r, b_{r+1}). Cut where the running token count first reaches
    r / world of the total (lengths below 0 count as 0)."""
    if world < 1:
        raise ValueError("bad world size")
    lens = [max(0, int(x)) for x in seqlens]
    B = len(lens)
    total = sum(lens)
    cuts = [0]
    run, b = 0, 0
    for r in range(1, world):
        target = total * r / world
        while b < B and run + lens[b] / 2 < target:  # a sequence goes where most of it falls
            run += lens[b]
            b += 1
        cuts.append(max(b, cuts[-1]))
    cuts.append(B)
    return cuts


def decode_shard(q, kcache, vcache, seqlens_host: Sequence[int], Hkv: int, world: int,
                 rank: int, seqlens_dev=None):
    """Views for this rank's sequences: q [b1-b0, Hq, d], the packed caches'
    slice, and the lengths (a view of `seqlens_dev` if given, the device copy
    the kernels read). Returns (q, kcache, vcache, seqlens, (b0, b1))."""
    cuts = decode_cuts(seqlens_host, world)
    b0, b1 = cuts[rank], cuts[rank + 1]
    lens = [max(0, int(x)) for x in seqlens_host]
    d = q.shape[-1]
    per = Hkv * d
    t0, t1 = sum(lens[:b0]) * per, sum(lens[:b1]) * per
    sl = seqlens_dev[b0:b1] if seqlens_dev is not None else seqlens_host[b0:b1]
    return q[b0:b1], kcache.reshape(-1)[t0:t1], vcache.reshape(-1)[t0:t1], sl, (b0, b1)
