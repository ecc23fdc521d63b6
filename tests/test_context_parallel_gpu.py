"""Context-parallel prefill on the GPU against the fp64 oracle.

* attn_merge: folding partial results one by one into an fp32 accumulator
  gives the oracle's combine of all of them (the log-sum-exp identity of the
  aikaboom page "11.4d FlashAttention", "Online Softmax"), including rows that
  are empty in some or all partials; an empty accumulator row is never read
  (it is filled with NaN here).
* ring_attention: every rank of a W-rank zigzag ring is run on this one GPU
  with LocalRing handing over the K/V block the real ring would deliver at
  each step, so the kernels see exactly the calls of a multi-GPU run. The
  ranks' outputs, put back in sequence order, must match the oracle's
  attention over the whole sequence.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from exact_tiled_attention_38_b200 import context_parallel as cp
from parity import compare, ulp

pytestmark = pytest.mark.gpu

DEV = "cuda"
BF16, F16 = torch.bfloat16, torch.float16


@pytest.mark.parametrize("d", [8, 64, 96, 128, 256])
@pytest.mark.parametrize("dt", [BF16, F16])
def test_merge_matches_oracle_combine(lib, d, dt):
    gen = torch.Generator().manual_seed(7300 + d)
    shape = (2, 3, 77)
    parts_o = [torch.randn(*shape, d, generator=gen).to(dt) for _ in range(3)]
    parts_l = [torch.rand(*shape, generator=gen) * 6 - 3 for _ in range(3)]
    parts_l[0][0, 0, :5] = float("-inf")        # empty in one partial
    for p in parts_l:
        p[1, 2, 10] = float("-inf")             # empty in every partial
    parts_l[2][1, 1, 20] = 40.0                 # one partial dominates
    o_acc = torch.full((*shape, d), float("nan"), device=DEV)
    lse_acc = torch.full(shape, float("-inf"), device=DEV)
    o_out = torch.empty(*shape, d, dtype=dt, device=DEV)
    for i in range(3):
        lib.attn_merge(o_acc, lse_acc, parts_o[i].to(DEV), parts_l[i].to(DEV),
                       o_out=o_out if i == 2 else None)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.combine_partials(torch.stack(parts_o), torch.stack(parts_l))
    acc = o_acc.cpu().double().numpy()
    assert np.isfinite(acc).all()
    np.testing.assert_allclose(acc, o_ref, atol=2e-6, rtol=2e-6)
    l = lse_acc.cpu().double().numpy()
    assert (np.isneginf(l) == np.isneginf(l_ref)).all()
    fin = np.isfinite(l_ref)
    np.testing.assert_allclose(l[fin], l_ref[fin], atol=2e-6, rtol=0)
    out = o_out.cpu().double().numpy()
    assert (np.abs(out - o_ref) <= ulp(o_ref, dt) * 0.5 + 4e-6).all()  # rounded to nearest
    assert (out[1, 2, 10] == 0).all()


RING = [
    # world, causal, Hq, Hkv, N, d, dtype
    (1, True, 2, 1, 1000, 128, BF16),
    (2, True, 4, 2, 1200, 128, BF16),   # chunks of 300: ragged 128-row tiles
    (4, True, 8, 2, 2048, 128, BF16),
    (3, False, 4, 4, 1536, 64, F16),
    (2, True, 4, 1, 1024, 64, F16),     # MQA
    (2, True, 4, 2, 800, 96, BF16),     # generic head size
]


@pytest.mark.parametrize("case", RING, ids=lambda c: "w{}{}h{}kv{}n{}d{}".format(
    c[0], "c" if c[1] else "n", *c[2:6]))
def test_ring_attention_emulated(lib, case):
    world, causal, Hq, Hkv, N, d, dt = case
    q, k, v = workloads.random_prefill(1, Hq, Hkv, N, N, d, dt, seed=7400 + RING.index(case))
    scale = d ** -0.5
    ks = [cp.shard_zigzag(k, r, world).to(DEV) for r in range(world)]
    vs = [cp.shard_zigzag(v, r, world).to(DEV) for r in range(world)]
    outs, lses = [], []
    for r in range(world):
        ex = cp.LocalRing(r, ks, vs) if world > 1 else None
        o, lse = cp.ring_attention(cp.shard_zigzag(q, r, world).to(DEV), ks[r], vs[r], causal,
                                   scale, exchange=ex)
        outs.append(o.cpu())
        lses.append(lse.cpu())
    torch.cuda.synchronize()
    code, raw = lib.attn_get_device_status()
    assert code == lib.ATTN_OK, f"device status {code} site {raw:#x}"
    o_ref, lse_ref = oracle.attention_ref(q, k, v, scale, causal)
    compare(cp.unshard_zigzag(outs), cp.unshard_zigzag(lses), o_ref, lse_ref, dt, str(case))


# Partial results kept in fp32: attn_fwd_partial writes O unrounded, and
# attn_merge folds such partials (attn_merge_partial[_f16]).
PARTIAL = [
    # B, Hq, Hkv, Nq, Nk, d, causal, dtype
    (2, 4, 2, 300, 300, 128, True, BF16),
    (1, 2, 1, 129, 1000, 128, True, BF16),    # Nq < Nk, bottom-right causal
    (1, 2, 2, 257, 130, 64, True, F16),       # rows without keys
    (1, 3, 3, 200, 333, 64, False, BF16),
    (1, 2, 1, 100, 100, 96, True, BF16),      # generic head size
]


@pytest.mark.parametrize("case", PARTIAL, ids=lambda c: "x".join(map(str, c[:6])))
def test_fwd_partial_unrounded_output(lib, case):
    B, Hq, Hkv, Nq, Nk, d, causal, dt = case
    q, k, v = workloads.random_prefill(B, Hq, Hkv, Nq, Nk, d, dt, seed=7500 + PARTIAL.index(case))
    scale = d ** -0.5
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o32, lse = lib.attn_fwd_partial(qd, kd, vd, scale=scale, causal=causal)
    fn = lib.attn_fwd_f16 if dt == F16 else lib.attn_fwd
    o16, lse16 = fn(qd, kd, vd, scale=scale, causal=causal)
    torch.cuda.synchronize()
    assert o32.dtype == torch.float32
    # the same arithmetic before the final rounding: rounding o32 gives attn_fwd's O
    assert torch.equal(o32.to(dt), o16) and torch.equal(lse, lse16)
    o_ref, lse_ref = oracle.attention_ref(q, k, v, scale, causal)
    compare(o32, lse, o_ref, lse_ref, dt, f"partial {case[:7]}")


@pytest.mark.parametrize("dt", [BF16, F16])
def test_merge_of_fp32_partials(lib, dt):
    gen = torch.Generator().manual_seed(7600)
    shape, d = (3, 50), 128
    parts_o = [torch.randn(*shape, d, generator=gen) for _ in range(4)]
    parts_l = [torch.rand(*shape, generator=gen) * 6 - 3 for _ in range(4)]
    parts_l[1][0, :7] = float("-inf")
    o_acc = torch.full((*shape, d), float("nan"), device=DEV)
    lse_acc = torch.full(shape, float("-inf"), device=DEV)
    o_out = torch.empty(*shape, d, dtype=dt, device=DEV)
    for i in range(4):
        lib.attn_merge(o_acc, lse_acc, parts_o[i].to(DEV), parts_l[i].to(DEV),
                       o_out=o_out if i == 3 else None)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.combine_partials(torch.stack(parts_o).double(),
                                           torch.stack(parts_l).double())
    np.testing.assert_allclose(o_acc.cpu().double().numpy(), o_ref, atol=2e-6, rtol=2e-6)
    np.testing.assert_allclose(lse_acc.cpu().double().numpy(), l_ref, atol=2e-6, rtol=0)
    out = o_out.cpu().double().numpy()
    assert (np.abs(out - o_ref) <= ulp(o_ref, dt) * 0.5 + 4e-6).all()


def _ring_rows(q, k, v, world, causal, scale, rows):
    """Every rank of a `world`-rank ring on this GPU; the result's `rows`."""
    ks = [cp.shard_zigzag(k, r, world).to(DEV) for r in range(world)]
    vs = [cp.shard_zigzag(v, r, world).to(DEV) for r in range(world)]
    outs, lses = [], []
    for r in range(world):
        ex = cp.LocalRing(r, ks, vs) if world > 1 else None
        o, lse = cp.ring_attention(cp.shard_zigzag(q, r, world).to(DEV), ks[r], vs[r], causal,
                                   scale, exchange=ex)
        outs.append(o.cpu())
        lses.append(lse.cpu())
    torch.cuda.synchronize()
    o = cp.unshard_zigzag(outs)
    lse = cp.unshard_zigzag(lses)
    return o[:, :, rows], lse[:, :, rows]


def test_ring_of_eight_at_16k_error_does_not_grow(lib):
    # One 16K causal GQA sequence over rings of 2, 4 and 8 ranks (chunks of
    # 4096, 2048 and 1024 tokens): a query chunk's output is folded from up to
    # 2W - 1 partials, each kept in fp32, so the output is rounded once and its
    # error against the oracle must not grow with W.
    N, Hq, Hkv, d = 16384, 8, 2, 128
    q, k, v = workloads.random_prefill(1, Hq, Hkv, N, N, d, BF16, seed=7700)
    scale = d ** -0.5
    rows = np.sort(np.random.default_rng(7701).choice(N, size=96, replace=False))
    rows[0], rows[-1] = 0, N - 1
    o_ref, lse_ref = oracle.attention_ref(q[:, :, rows], k, v, scale, True, rows=rows, nq=N)
    errs = {}
    for world in (2, 4, 8):
        o, lse = _ring_rows(q, k, v, world, True, scale, rows)
        res = compare(o, lse, o_ref, lse_ref, BF16, f"ring of {world} at 16K, sampled rows")
        errs[world] = res["max_abs_o"]
    code, raw = lib.attn_get_device_status()
    assert code == lib.ATTN_OK, f"device status {code} site {raw:#x}"
    assert errs[8] <= 1.5 * errs[2] + 2e-4, errs
