"""Sliding-window prefill and decode on the GPU against the fp64 oracle.

Reading (zimaspace page, "Reduced IO Is Not the Same as Eliminating KV Cache",
windowing as a runtime scheme): causal query i keeps keys j with
i + (Nk - Nq) - W < j <= i + (Nk - Nq); decode keeps the last W cached tokens.
Cases cover windows narrower than a tile, windows that start inside a tile,
windows wider than the sequence (plain causal), Nq < Nk and Nq > Nk, and the
bf16 and fp16 entry points.
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
    # B, Hq, Hkv, Nq, Nk, d, window, dtype
    (2, 4, 2, 300, 300, 128, 64, BF16),
    (1, 2, 1, 700, 700, 128, 1, BF16),       # each row sees only its own key
    (1, 2, 2, 513, 513, 128, 200, BF16),     # window starts inside a key tile
    (1, 4, 4, 256, 1000, 128, 130, BF16),    # Nq < Nk (chunk of a longer cache)
    (1, 2, 2, 400, 150, 64, 40, F16),        # Nq > Nk: rows without keys
    (1, 2, 1, 1024, 1024, 64, 5000, BF16),   # window wider than every row: plain causal
    (1, 8, 2, 2048, 2048, 128, 384, BF16),   # several items, windows of 3 key tiles
]


@pytest.mark.parametrize("case", PREFILL, ids=lambda c: "x".join(map(str, c[:7])))
def test_prefill_window(lib, case):
    B, Hq, Hkv, Nq, Nk, d, W, dt = case
    q, k, v = workloads.random_prefill(B, Hq, Hkv, Nq, Nk, d, dt, seed=5000 + PREFILL.index(case))
    scale = d ** -0.5
    o, lse = lib.attn_fwd_window(q.to(DEV), k.to(DEV), v.to(DEV), W, scale=scale)
    torch.cuda.synchronize()
    code, raw = lib.attn_get_device_status()
    assert code == lib.ATTN_OK, f"device status {code} site {raw:#x}"
    o_ref, lse_ref = oracle.attention_ref(q, k, v, scale, True, window=W)
    compare(o, lse, o_ref, lse_ref, dt, str(case))


def test_prefill_window_wider_than_keys_equals_causal(lib):
    q, k, v = workloads.random_prefill(1, 4, 2, 600, 600, 128, BF16, seed=5100, device=DEV)
    o1, l1 = lib.attn_fwd_window(q, k, v, 600)
    o2, l2 = lib.attn_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


DECODE = [
    # B, Hq, Hkv, d, lengths, window, dtype
    (4, 8, 2, 128, [1, 37, 300, 0], 32, BF16),
    (3, 32, 8, 128, [5000, 100, 2049], 1000, BF16),
    (2, 16, 2, 64, [129, 4096], 129, F16),
    (2, 8, 1, 128, [777, 20], 1, BF16),
    (5, 64, 4, 128, [9000, 0, 130, 4000, 257], 1100, BF16),  # group 16, persistent pass
    (3, 32, 1, 64, [3000, 5, 700], 500, BF16),               # MQA, d = 64, persistent pass
]


@pytest.mark.parametrize("case", DECODE, ids=lambda c: f"B{c[0]}h{c[1]}kv{c[2]}d{c[3]}w{c[5]}")
def test_decode_window(lib, case):
    B, Hq, Hkv, d, lens, W, dt = case
    sl = torch.tensor(lens, dtype=torch.int32)
    q, kc, vc, sl = workloads.random_decode(B, Hq, Hkv, d, sl, dt, seed=5200 + DECODE.index(case))
    scale = d ** -0.5
    o, lse = lib.attn_decode_window(q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), Hkv, W,
                                    scale=scale)
    torch.cuda.synchronize()
    code, raw = lib.attn_get_device_status()
    assert code == lib.ATTN_OK, f"device status {code} site {raw:#x}"
    o_ref, lse_ref = oracle.decode_ref(q, kc, vc, sl, scale, Hkv, window=W)
    compare(o, lse, o_ref, lse_ref, dt, str(case))
