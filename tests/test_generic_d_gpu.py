"""Head sizes off the tensor-core path (multiples of 8 in [8, 256] other than
64 and 128) against the fp64 oracle.

These run on the generic CUDA-core kernel through the same entry points as
d = 64 / 128 (sicorps page: the head size is a model parameter; the tiled
method of the aikaboom page "11.4d FlashAttention" does not depend on it).
Cases cover causal, non-causal and sliding-window prefill, GQA and MQA,
Nq < Nk and Nq > Nk, ragged tails of the 16-row and 32-key tiles, fp16 and
bf16, and decode (plain, windowed and no-alloc) over a ragged cache with an
empty sequence.
"""
import pytest
import torch

import oracle
import workloads
from parity import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"
BF16, F16 = torch.bfloat16, torch.float16

PREFILL = [
    # B, Hq, Hkv, Nq, Nk, d, causal, window, dtype
    (1, 2, 1, 37, 37, 8, True, 0, BF16),
    (2, 4, 2, 100, 100, 32, True, 0, F16),
    (1, 4, 4, 77, 150, 40, False, 0, BF16),
    (2, 8, 2, 257, 257, 80, True, 0, BF16),
    (1, 6, 3, 129, 300, 96, True, 0, F16),      # Nq < Nk
    (1, 2, 2, 200, 60, 96, True, 0, BF16),      # Nq > Nk: rows without keys
    (1, 4, 1, 333, 333, 160, False, 0, BF16),   # MQA
    (1, 2, 1, 190, 190, 256, True, 0, BF16),
    (1, 2, 1, 96, 140, 256, False, 0, F16),
    (1, 4, 2, 300, 300, 80, True, 45, BF16),    # sliding window
    (1, 2, 2, 100, 100, 96, True, 1, F16),      # each row sees only its own key
]


@pytest.mark.parametrize("case", PREFILL, ids=lambda c: "x".join(map(str, c[:8])))
def test_prefill_generic_d(lib, case):
    B, Hq, Hkv, Nq, Nk, d, causal, W, dt = case
    q, k, v = workloads.random_prefill(B, Hq, Hkv, Nq, Nk, d, dt, seed=6000 + PREFILL.index(case))
    scale = d ** -0.5
    if W:
        o, lse = lib.attn_fwd_window(q.to(DEV), k.to(DEV), v.to(DEV), W, scale=scale)
    else:
        fn = lib.attn_fwd_f16 if dt == F16 else lib.attn_fwd
        o, lse = fn(q.to(DEV), k.to(DEV), v.to(DEV), scale=scale, causal=causal)
    torch.cuda.synchronize()
    code, raw = lib.attn_get_device_status()
    assert code == lib.ATTN_OK, f"device status {code} site {raw:#x}"
    o_ref, lse_ref = oracle.attention_ref(q, k, v, scale, causal, window=W)
    compare(o, lse, o_ref, lse_ref, dt, str(case))


def test_prefill_generic_d_empty_keys(lib):
    q = torch.randn(1, 2, 20, 48, device=DEV).to(BF16)
    k = torch.empty(1, 2, 0, 48, device=DEV, dtype=BF16)
    o, lse = lib.attn_fwd(q, k, k, causal=False)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


DECODE = [
    # B, Hq, Hkv, d, lengths, window, dtype
    (4, 8, 2, 96, [1, 37, 300, 0], 0, BF16),
    (3, 16, 2, 80, [1000, 33, 2049], 0, F16),
    (2, 4, 1, 256, [500, 31], 0, BF16),
    (3, 8, 8, 32, [64, 65, 7], 20, BF16),
]


@pytest.mark.parametrize("case", DECODE, ids=lambda c: f"B{c[0]}h{c[1]}kv{c[2]}d{c[3]}w{c[5]}")
def test_decode_generic_d(lib, case):
    B, Hq, Hkv, d, lens, W, dt = case
    sl = torch.tensor(lens, dtype=torch.int32)
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, dt, seed=6100 + DECODE.index(case))
    scale = d ** -0.5
    args = (q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), Hkv)
    if W:
        o, lse = lib.attn_decode_window(*args, W, scale=scale)
    else:
        fn = lib.attn_decode_f16 if dt == F16 else lib.attn_decode
        o, lse = fn(*args, scale=scale)
    torch.cuda.synchronize()
    code, raw = lib.attn_get_device_status()
    assert code == lib.ATTN_OK, f"device status {code} site {raw:#x}"
    o_ref, lse_ref = oracle.decode_ref(q, kc, vc, sl, scale, Hkv, window=W)
    compare(o, lse, o_ref, lse_ref, dt, str(case))
    if not W and dt == BF16:
        o2, lse2 = lib.attn_decode_noalloc(*args, scale=scale)
        torch.cuda.synchronize()
        assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_generic_d_more_heads_than_one_grid_dimension(lib):
    # B * Hq = 70,000 (batch, head) pairs: more than a grid dimension of
    # 65,535 blocks holds, so the kernel runs in z slices; tiny rows keep the
    # oracle fast. Prefill (causal, GQA) and decode (ragged, with empties).
    B, Hq, Hkv, N, d = 35000, 2, 1, 8, 8
    q, k, v = workloads.random_prefill(B, Hq, Hkv, N, N, d, BF16, seed=6200)
    o, lse = lib.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), scale=d ** -0.5, causal=True)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_ref(q, k, v, d ** -0.5, True)
    compare(o, lse, o_ref, lse_ref, BF16, "z-sliced prefill")

    sl = workloads.decode_seqlens(B, 0, 6, 6201)
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, BF16, seed=6202)
    o, lse = lib.attn_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), Hkv,
                             scale=d ** -0.5)
    torch.cuda.synchronize()
    code, raw = lib.attn_get_device_status()
    assert code == lib.ATTN_OK, f"device status {code} site {raw:#x}"
    o_ref, lse_ref = oracle.decode_ref(q, kc, vc, sl, d ** -0.5, Hkv)
    compare(o, lse, o_ref, lse_ref, BF16, "z-sliced decode")
