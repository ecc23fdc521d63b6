"""Bounded device waits, exercised on the GPU without a fault.

attn_fwd_stall_test enqueues the prefill kernel with its TMA producers issuing
no copies, so the first waits for data can never complete. Every wait in the
kernel has a time limit; the test checks that the launch ends on its own
within a few limits, that the status word reports a timeout at a known wait
site, and that the same CUDA context then runs an ordinary prefill that
matches the oracle.
"""
import time

import pytest
import torch

import oracle
import workloads
from parity import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"
# Wait sites of the prefill kernel that can give up first when no copy lands:
# Q full, K/V full (MMA warp), S ready (softmax warps).
STALL_SITES = {1, 3, 5}


def test_stalled_prefill_times_out_and_context_recovers(lib):
    B, Hq, Hkv, N, d = 1, 2, 1, 300, 128
    scale = d ** -0.5
    q, k, v = workloads.random_prefill(B, Hq, Hkv, N, N, d, torch.bfloat16, seed=4242)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o = torch.empty_like(qd)
    lse = torch.empty(B, Hq, N, device=DEV, dtype=torch.float32)
    assert lib.attn_get_device_status()[0] == lib.ATTN_OK

    wait_us = 2000
    t0 = time.perf_counter()
    rc = lib.load_library().attn_fwd_stall_test(
        qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv,
        N, N, d, scale, 1, wait_us, None)
    assert rc == lib.ATTN_OK
    code, raw = lib.attn_get_device_status()
    elapsed = time.perf_counter() - t0
    assert code == lib.ATTN_ERR_TIMEOUT, (code, hex(raw))
    assert raw & ~0xFFF == 0x1000 and (raw & 0xFFF) in STALL_SITES, hex(raw)
    assert elapsed < 2.0, elapsed  # a few 2 ms limits plus polling, not the 2 s default
    assert lib.attn_get_device_status()[0] == lib.ATTN_OK  # reading cleared the word

    o2, lse2 = lib.attn_fwd(qd, kd, vd, scale=scale, causal=True)
    torch.cuda.synchronize()
    assert lib.attn_get_device_status()[0] == lib.ATTN_OK
    o_ref, lse_ref = oracle.attention_ref(q, k, v, scale, True)
    compare(o2, lse2, o_ref, lse_ref, torch.bfloat16, "after stalled launch")

