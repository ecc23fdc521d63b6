"""Context-parallel prefill: one long sequence sharded over a ring of ranks.

Attention over a sequence too long for one GPU's time budget is split along
the sequence. Every rank holds a slice of Q, K and V; K/V blocks travel round
a ring of ranks by point-to-point sends, and each rank folds the partial
result of its query slice against every K/V block it sees into a running
(O, LSE) state. The fold is the log-sum-exp merge of the running softmax
statistics (aikaboom page "11.4d FlashAttention", "Online Softmax") applied
to whole key blocks, done by the library's ``attn_merge`` kernel; the
per-block attention is the library's prefill kernel. Long contexts of 32K to
128K tokens are the workloads the pages name for the tiled method (aikaboom
page, "The Core Problem" and "Real-World Impact").

Sharding (zigzag): the sequence of N tokens is cut into 2W chunks of
c = N / (2W) tokens; rank r holds chunks r and 2W-1-r, stored chunk-major as
``[2, B, H, c, d]`` so every chunk is one contiguous attn_fwd operand. With
causal attention each rank then does the same work at every ring step: at
step s it holds the K/V chunks of rank (r - s) mod W, and
  * step 0 (its own chunks): (r, r) and (2W-1-r, 2W-1-r) on the diagonal
    (causal, Nq = Nk = c), (2W-1-r, r) full;
  * a source rank below r: both query chunks against the source's low chunk,
    full;
  * a source rank above r: the high query chunk against both source chunks,
    full;
the remaining pairs lie wholly above the diagonal and are skipped. Without a
causal mask every pair is full.

Plumbing only in Python: the exchange is torch.distributed point-to-point
(NCCL over NVLink on GPUs; no collective, no multicast), double-buffered so
the next block's transfer overlaps the current block's kernels; all
arithmetic runs in the CUDA library.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple


def zigzag_chunk_ids(rank: int, world: int) -> Tuple[int, int]:
    """Sequence chunks (of 2 * world) that ``rank`` holds: (low, high)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return rank, 2 * world - 1 - rank


def pair_kind(q_chunk: int, k_chunk: int, causal: bool) -> str:
    """'full', 'diag' (causal, same chunk) or 'skip' (keys all in the future)."""
    if not causal or k_chunk < q_chunk:
        return "full"
    return "diag" if k_chunk == q_chunk else "skip"


@dataclass
class RingStep:
    src: int                                   # rank whose K/V chunks are held
    pairs: List[Tuple[int, int, str]] = field(default_factory=list)  # (q slot, kv slot, kind)


def ring_plan(rank: int, world: int, causal: bool) -> List[RingStep]:
    """The chunk pairs rank computes at each of the ``world`` ring steps."""
    mine = zigzag_chunk_ids(rank, world)
    plan = []
    for s in range(world):
        src = (rank - s) % world
        theirs = zigzag_chunk_ids(src, world)
        step = RingStep(src)
        for qi in (0, 1):
            for ki in (0, 1):
                kind = pair_kind(mine[qi], theirs[ki], causal)
                if kind != "skip":
                    step.pairs.append((qi, ki, kind))
        plan.append(step)
    return plan


def shard_zigzag(x, rank: int, world: int):
    """This rank's two chunks of x [B, H, N, ...] along N, as [2, B, H, c, ...]."""
    import torch

    N = x.shape[2]
    if N % (2 * world) != 0:
        raise ValueError(f"sequence length {N} is not a multiple of 2 * world = {2 * world}")
    c = N // (2 * world)
    lo, hi = zigzag_chunk_ids(rank, world)
    return torch.stack([x[:, :, lo * c:(lo + 1) * c], x[:, :, hi * c:(hi + 1) * c]]).contiguous()


def unshard_zigzag(shards):
    """Inverse of shard_zigzag: per-rank [2, B, H, c, ...] shards -> [B, H, N, ...]."""
    import torch

    world = len(shards)
    chunks = [None] * (2 * world)
    for r, sh in enumerate(shards):
        lo, hi = zigzag_chunk_ids(r, world)
        chunks[lo], chunks[hi] = sh[0], sh[1]
    return torch.cat(chunks, dim=2)


class RingExchange:
    """Send the held K/V block to rank + 1, receive rank - 1's, in one batch of
    torch.distributed point-to-point operations (NCCL on GPUs, gloo on CPUs)."""

    def __init__(self, group=None):
        import torch.distributed as dist

        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self._reqs = []

    def _global(self, r):
        return r if self.group is None else self.dist.get_global_rank(self.group, r)

    def start(self, send_k, send_v, recv_k, recv_v) -> None:
        d = self.dist
        nxt = self._global((self.rank + 1) % self.world)
        prv = self._global((self.rank - 1) % self.world)
        ops = [d.P2POp(d.isend, send_k, nxt, self.group), d.P2POp(d.irecv, recv_k, prv, self.group),
               d.P2POp(d.isend, send_v, nxt, self.group), d.P2POp(d.irecv, recv_v, prv, self.group)]
        self._reqs = d.batch_isend_irecv(ops)

    def wait(self) -> None:
        for r in self._reqs:
            r.wait()
        self._reqs = []


class LocalRing:
    """Stand-in for RingExchange inside one process: rank ``rank`` of a ring
    whose every rank's K/V shard is at hand. It hands over, at each step, the
    block the real ring would deliver, so one GPU can run any rank's exact
    sequence of kernel calls."""

    def __init__(self, rank: int, shards_k, shards_v):
        self.rank = rank
        self.world = len(shards_k)
        self._k, self._v = shards_k, shards_v
        self._step = 0

    def start(self, send_k, send_v, recv_k, recv_v) -> None:
        self._step += 1
        src = (self.rank - self._step) % self.world
        recv_k.copy_(self._k[src])
        recv_v.copy_(self._v[src])

    def wait(self) -> None:
        pass


class CudaOps:
    """The library's kernels: prefill on one chunk pair with O kept in float32,
    and the LSE merge of such a partial into the running accumulator."""

    def attention(self, q, k, v, scale, causal, o, lse):
        from . import attn_fwd_partial

        return attn_fwd_partial(q, k, v, o=o, lse=lse, scale=scale, causal=causal)

    def merge(self, o_acc, lse_acc, o_part, lse_part, o_out):
        from . import attn_merge

        attn_merge(o_acc, lse_acc, o_part, lse_part, o_out=o_out)


def ring_attention(q, k, v, causal: bool = True, scale: Optional[float] = None,
                   exchange=None, ops=None):
    """Attention of this rank's query chunks against the whole sequence.

    q [2, B, Hq, c, d], k and v [2, B, Hkv, c, d]: this rank's zigzag shard
    (``shard_zigzag``), bf16 or fp16, on this rank's GPU. ``exchange`` is a
    RingExchange (None: a single rank holding the whole sequence). Returns
    (o [2, B, Hq, c, d] in q's dtype, lse [2, B, Hq, c] float32), this rank's
    rows of the full-sequence result.
    """
    import math

    import torch

    if q.dim() != 5 or k.dim() != 5 or q.shape[0] != 2 or k.shape != v.shape:
        raise ValueError("q, k, v must be zigzag shards [2, B, H, c, d]")
    ops = ops or CudaOps()
    world = exchange.world if exchange is not None else 1
    rank = exchange.rank if exchange is not None else 0
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    plan = ring_plan(rank, world, causal)
    last = {}
    for s, step in enumerate(plan):
        for n, (qi, _, _) in enumerate(step.pairs):
            last[qi] = (s, n)

    o = torch.empty_like(q)
    o_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse_acc = torch.full(q.shape[:-1], float("-inf"), dtype=torch.float32, device=q.device)
    # Every partial O stays unrounded (float32; wider inputs keep their own
    # type), so the 2W - 1 folds of a query chunk round its output once.
    part_dt = torch.float32 if q.dtype in (torch.bfloat16, torch.float16) else q.dtype
    part_o = torch.empty(q.shape[1:], dtype=part_dt, device=q.device)
    part_lse = torch.empty(q.shape[1:-1], dtype=torch.float32, device=q.device)
    cur_k, cur_v = k, v
    nxt_k, nxt_v = (torch.empty_like(k), torch.empty_like(v)) if world > 1 else (None, None)
    for s, step in enumerate(plan):
        if s + 1 < world:
            exchange.start(cur_k, cur_v, nxt_k, nxt_v)
        for n, (qi, ki, kind) in enumerate(step.pairs):
            ops.attention(q[qi], cur_k[ki], cur_v[ki], scale, kind == "diag", part_o, part_lse)
            ops.merge(o_acc[qi], lse_acc[qi], part_o, part_lse,
                      o[qi] if last[qi] == (s, n) else None)
        if s + 1 < world:
            exchange.wait()
            if s == 0:  # the caller's k, v are never written: recycle a fresh pair
                cur_k, cur_v, nxt_k, nxt_v = nxt_k, nxt_v, torch.empty_like(k), torch.empty_like(v)
            else:
                cur_k, cur_v, nxt_k, nxt_v = nxt_k, nxt_v, cur_k, cur_v
    return o, lse_acc
