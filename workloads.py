"""Seeded synthetic workloads for exact tiled attention.

This module only draws random inputs and names the workload shapes; it holds
none of the attention arithmetic. Both the CUDA path (through the tests and
``bench.py``) and the fp64 oracle consume the tensors it returns, bit for bit.

Recipe (all inputs synthetic; the pages name no dataset):
  * Q, K, V entries are i.i.d. N(0, 1) (times ``std``) drawn in fp32 by a
    ``torch.Generator`` seeded with the workload's seed, in the order q, k, v,
    then rounded to the storage dtype (round-to-nearest-even).
  * Decode sequence lengths are integers uniform in [lmin, lmax], drawn by a
    CPU ``torch.Generator`` seeded with the workload's seed, before the caches.
  * Sampled query rows for the long prompts are drawn without replacement by
    ``numpy.random.default_rng(seed + 100)`` and sorted.

The generator device is part of the recipe: CPU and CUDA generators give
different streams for the same seed, so a caller draws once and hands the same
tensor to both sides.

Workloads (the score-matrix sizes they imply follow "The Core Problem" on the
aikaboom page "11.4d FlashAttention"; the 32K and 128K contexts are the ones
that page's "Performance Impact" list names):
  * prefill_f16_b1_h1_n256_d64: single-head non-causal fp16, B=1, H=1,
    N=256, d=64.
  * prefill_causal_mha_b4_h16_n2048_d128: causal MHA bf16, B=4, Hq=Hkv=16,
    N=2048, d=128.
  * prefill_causal_gqa_b1_h32kv8_n32k_d128: causal GQA bf16, B=1, Hq=32,
    Hkv=8, N=32768, d=128; 256 sampled rows per head.
  * decode_gqa_b64_h32kv8_d128_ragged: one query token per sequence, B=64,
    Hq=32, Hkv=8, d=128, per-sequence KV length uniform in [1024, 8192].
  * prefill_causal_gqa_b1_h32kv8_n128k_d128: causal GQA bf16 at 128K context,
    B=1, Hq=32, Hkv=8, N=131072, d=128, data N(0,1)*0.5; 64 sampled rows per
    head including the first and the last row.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

SEED_BASE = 38_000
ROW_SEED_OFFSET = 100


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    dtype: str  # "bf16" or "f16"
    causal: bool
    seed: int
    std: float = 1.0
    sample_rows: Optional[int] = None  # None: every row is checked
    include_ends: bool = False  # sampled rows always contain 0 and Nq-1

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    lmin: int
    lmax: int
    dtype: str
    seed: int
    std: float = 1.0

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


PREFILL_SMALL = PrefillWorkload(
    "prefill_f16_b1_h1_n256_d64", B=1, Hq=1, Hkv=1, Nq=256, Nk=256, d=64,
    dtype="f16", causal=False, seed=SEED_BASE + 0)
PREFILL_MHA_2K = PrefillWorkload(
    "prefill_causal_mha_b4_h16_n2048_d128", B=4, Hq=16, Hkv=16, Nq=2048, Nk=2048,
    d=128, dtype="bf16", causal=True, seed=SEED_BASE + 1)
PREFILL_GQA_32K = PrefillWorkload(
    "prefill_causal_gqa_b1_h32kv8_n32k_d128", B=1, Hq=32, Hkv=8, Nq=32768, Nk=32768,
    d=128, dtype="bf16", causal=True, seed=SEED_BASE + 2, sample_rows=256)
DECODE_GQA_RAGGED = DecodeWorkload(
    "decode_gqa_b64_h32kv8_d128_ragged", B=64, Hq=32, Hkv=8, d=128, lmin=1024,
    lmax=8192, dtype="bf16", seed=SEED_BASE + 3)
PREFILL_GQA_128K = PrefillWorkload(
    "prefill_causal_gqa_b1_h32kv8_n128k_d128", B=1, Hq=32, Hkv=8, Nq=131072,
    Nk=131072, d=128, dtype="bf16", causal=True, seed=SEED_BASE + 4, std=0.5,
    sample_rows=64, include_ends=True)

WORKLOADS = [PREFILL_SMALL, PREFILL_MHA_2K, PREFILL_GQA_32K, DECODE_GQA_RAGGED,
             PREFILL_GQA_128K]


def _randn(shape, gen, device, std, dtype):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def prefill_inputs(w: PrefillWorkload, device="cpu", seed: Optional[int] = None):
    """Return (q, k, v) in BHSD layout, contiguous, in the workload dtype."""
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed if seed is None else seed)
    q = _randn((w.B, w.Hq, w.Nq, w.d), gen, device, w.std, w.torch_dtype)
    k = _randn((w.B, w.Hkv, w.Nk, w.d), gen, device, w.std, w.torch_dtype)
    v = _randn((w.B, w.Hkv, w.Nk, w.d), gen, device, w.std, w.torch_dtype)
    return q, k, v


def random_prefill(B, Hq, Hkv, Nq, Nk, d, dtype=torch.bfloat16, seed=0,
                   device="cpu", std=1.0):
    """Ad-hoc seeded prefill inputs for parity sweeps (same recipe as above)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = _randn((B, Hq, Nq, d), gen, device, std, dtype)
    k = _randn((B, Hkv, Nk, d), gen, device, std, dtype)
    v = _randn((B, Hkv, Nk, d), gen, device, std, dtype)
    return q, k, v


def decode_seqlens(B, lmin, lmax, seed) -> torch.Tensor:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return torch.randint(lmin, lmax + 1, (B,), generator=gen, dtype=torch.int32)


def decode_inputs(w: DecodeWorkload, device="cpu", seqlens: Optional[torch.Tensor] = None,
                  seed: Optional[int] = None):
    """Return (q [B,Hq,d], kcache, vcache, seqlens int32 [B]).

    The caches are packed: sequence b starts at token offset sum(seqlens[:b]) and
    is laid out [Hkv][L_b][d], so each (b, kv head) is one contiguous run. The
    caches are returned flat (1-D) in the workload dtype.
    """
    s = w.seed if seed is None else seed
    if seqlens is None:
        seqlens = decode_seqlens(w.B, w.lmin, w.lmax, s)
    return random_decode(w.B, w.Hq, w.Hkv, w.d, seqlens, w.torch_dtype, s, device, w.std)


def random_decode(B, Hq, Hkv, d, seqlens, dtype=torch.bfloat16, seed=0, device="cpu",
                  std=1.0):
    seqlens = torch.as_tensor(seqlens, dtype=torch.int32).cpu()
    assert seqlens.numel() == B
    total = int(seqlens.clamp(min=0).sum())
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 1)
    q = _randn((B, Hq, d), gen, device, std, dtype)
    kc = _randn((total * Hkv * d,), gen, device, std, dtype)
    vc = _randn((total * Hkv * d,), gen, device, std, dtype)
    return q, kc, vc, seqlens.to(device)


def sampled_rows(w: PrefillWorkload) -> np.ndarray:
    """Seeded query rows the oracle evaluates for a long prompt (sorted, unique)."""
    if w.sample_rows is None:
        return np.arange(w.Nq)
    rng = np.random.default_rng(w.seed + ROW_SEED_OFFSET)
    rows = rng.choice(w.Nq, size=w.sample_rows, replace=False)
    if w.include_ends:
        rows[0] = 0
        rows[1] = w.Nq - 1
        rows = np.unique(rows)
        while rows.size < w.sample_rows:  # refill if the ends were drawn already
            extra = rng.choice(w.Nq, size=w.sample_rows - rows.size, replace=False)
            rows = np.unique(np.concatenate([rows, extra]))
    return np.sort(rows)
