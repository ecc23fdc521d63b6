#!/usr/bin/env python
"""Benchmark of the exact tiled attention hot path on B200.

One step = one pass of the whole path over one batch of each synthetic
workload, inputs resident in HBM:
  * prefill, causal GQA bf16 at 128K context: B=1, Hq=32, Hkv=8, N=131072,
    d=128 (O and LSE) -- the headline: `value` is its TFLOP/s;
  * prefill, causal GQA bf16, long prompt: B=1, Hq=32, Hkv=8, N=32768, d=128;
  * prefill, causal MHA bf16: B=4, Hq=Hkv=16, N=2048, d=128;
  * decode, GQA bf16: 64 sequences, Hq=32, Hkv=8, d=128, KV lengths uniform
    in [1024, 8192] (split-KV pass + LSE combine).
Prefill throughput is algorithmic FLOPs (4*d per visible query/key pair) over
the kernel's CUDA-event time, summed over ranks (weak scaling: every rank runs
its own batch); decode is reported in GB/s of KV cache read. L2 is flushed
before every kernel (a 256 MiB write, then a 256 MiB read that evicts the
written lines); the flush is outside the kernel events. The small fp16
single-head workload is a parity case only (about 9 us of launch-bound work),
not a bench line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With --impl reference the fp64 CPU oracle runs a bounded sample of the same
workload on the host cores (rank 0 only) and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "prefill attn TFLOP/s & decode KV-cache GB/s, as % of B200 roofline"
HEADLINE = workloads.PREFILL_GQA_128K
PREFILLS = (workloads.PREFILL_GQA_128K, workloads.PREFILL_GQA_32K, workloads.PREFILL_MHA_2K)
PREFILL_KEYS = {workloads.PREFILL_GQA_128K.name: "128k", workloads.PREFILL_GQA_32K.name: "32k",
                workloads.PREFILL_MHA_2K.name: "2k"}
PREFILL = workloads.PREFILL_MHA_2K
DECODE = workloads.DECODE_GQA_RAGGED
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Spec-sheet figures for one B200, for context beside the measured peaks: dense
# bf16 tensor throughput (without 2:4 sparsity) and HGX HBM3e bandwidth.
NOMINAL_PEAKS = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
# Sources each measured kernel is compiled from (its traffic figure is valid
# only while they hash to the value recorded with it).
KERNEL_SOURCES = {
    k: [os.path.join(ROOT, "exact_tiled_attention_38_b200", "csrc", f) for f in files]
    for k, files in {
        "attn_prefill_kernel": ("prefill_sm100.cuh", "common.cuh", "ptx.cuh"),
        "attn_decode_persistent_kernel": ("decode_ps_sm100.cuh",
                                          "decode_sm100.cuh", "common.cuh", "ptx.cuh"),
    }.items()
}


# ----------------------------------------------------------------------------- accounting
def visible_pairs(nq: int, nk: int, causal: bool) -> int:
    """(query, key) pairs a row-wise softmax sees; causal is bottom-right aligned."""
    if not causal:
        return nq * nk
    per_row = np.clip(np.arange(nq, dtype=np.int64) + (nk - nq) + 1, 0, nk)
    return int(per_row.sum())


def prefill_flops(w) -> float:
    return 4.0 * w.d * w.B * w.Hq * visible_pairs(w.Nq, w.Nk, w.causal)


def decode_kv_bytes(seqlens, Hkv: int, d: int, elem: int = 2) -> int:
    total = int(np.clip(np.asarray(seqlens, dtype=np.int64), 0, None).sum())
    return 2 * total * Hkv * d * elem


def decode_bytes(seqlens, B, Hq, Hkv, d, elem=2) -> int:
    """Algorithmic HBM bytes of one decode call: KV read + q read + O/LSE write."""
    return decode_kv_bytes(seqlens, Hkv, d, elem) + 2 * B * Hq * d * elem + B * Hq * 4


def prefill_bytes(w) -> int:
    e = 2
    q = w.B * w.Hq * w.Nq * w.d * e
    kv = 2 * w.B * w.Hkv * w.Nk * w.d * e
    return 2 * q + kv + w.B * w.Hq * w.Nq * 4


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[kernel]:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summaries, if the kernel's sources have not changed since the capture; else
    None."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    ent = d.get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("per_workload", {}).get(workload)


# ----------------------------------------------------------------------------- ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def reduce_max(values, group=None):
    """Element-wise max over ranks of a list of floats (identity on one rank)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else "cpu"
    t = torch.tensor(list(values), dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t.cpu().tolist()


def aggregate_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: units all ranks processed / slowest rank's time (per s)."""
    return units_per_rank * world / (max_ms * 1e-3)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clocks and clock-event (throttle) reasons through NVML, read
    only, every `period_s` while the timed loop runs. The GPU is matched by PCI
    bus id so that NVML and CUDA indices need not agree. While sampling, the
    interpreter's thread switch interval is shortened to a fifth of the period:
    otherwise the launching thread keeps the interpreter lock for up to 5 ms at
    a time and a short timed region gets a single sample."""

    REASONS = {  # NVML clocks-event reason bits that reject or annotate a run
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4,
    }

    def __init__(self, cuda_index: int, period_s: float = 0.005):
        self.cuda_index = cuda_index
        self.period = period_s
        self.sm = []
        self.max_sm = None
        self.reasons = set()
        self.error = None
        self._stop = threading.Event()
        self._t = None
        self._h = None
        self._nvml = None
        self._switch = None

    def _handle(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        self._nvml = pynvml
        props = torch.cuda.get_device_properties(self.cuda_index)
        bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id,
                                    props.pci_device_id)
        try:
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _run(self):
        nv = self._nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while True:
            try:
                self.sm.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = get_reasons(self._h)
                for name, bit in self.REASONS.items():
                    if bits & bit:
                        self.reasons.add(name)
            except Exception as e:  # pragma: no cover
                self.error = str(e)
                return
            if self._stop.wait(self.period):
                return

    def __enter__(self):
        try:
            self._h = self._handle()
            self.max_sm = self._nvml.nvmlDeviceGetMaxClockInfo(self._h, self._nvml.NVML_CLOCK_SM)
            self._switch = sys.getswitchinterval()
            sys.setswitchinterval(min(self._switch, self.period / 5))
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception as e:
            self.error = str(e)
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join(timeout=10)
        if self._switch is not None:
            sys.setswitchinterval(self._switch)

    def summary(self):
        out = {"sm_mhz": statistics.median(self.sm) if self.sm else None,
               "sm_max_mhz": self.max_sm, "reasons": sorted(self.reasons),
               "samples": len(self.sm), "source": "nvml"}
        if self.error:
            out["error"] = self.error
        return out


def merged_clocks(samplers):
    """One clock record over several sampled regions (median of all samples)."""
    sm = [x for c in samplers for x in c.sm]
    reasons = sorted(set().union(*(c.reasons for c in samplers))) if samplers else []
    out = {"sm_mhz": statistics.median(sm) if sm else None,
           "sm_max_mhz": samplers[0].max_sm if samplers else None, "reasons": reasons,
           "samples": len(sm), "source": "nvml",
           "per_phase": [c.summary() for c in samplers]}
    errs = [c.error for c in samplers if c.error]
    if errs:
        out["error"] = errs[0]
    return out


# ----------------------------------------------------------------------------- CPU oracle
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def headline_head_inputs():
    """One (batch, KV head) of the 128K workload on the host, drawn with its seed
    and recipe (the oracle's cost per row does not depend on the values): q of
    query head 0, k and v of KV head 0."""
    import torch

    w = HEADLINE
    gen = torch.Generator().manual_seed(w.seed)
    shape = (1, 1, w.Nq, w.d)
    q = (torch.randn(shape, generator=gen) * w.std).to(w.torch_dtype)
    k = (torch.randn(shape, generator=gen) * w.std).to(w.torch_dtype)
    v = (torch.randn(shape, generator=gen) * w.std).to(w.torch_dtype)
    return q, k, v


def oracle_rows_sample(q, k, v, rows):
    """fp64 oracle on query rows `rows` of one head of the 128K workload.
    Returns (seconds, algorithmic FLOPs of those rows)."""
    import oracle

    w = HEADLINE
    rows = np.asarray(rows, dtype=np.int64)
    t0 = time.perf_counter()
    oracle.attention_ref(q[:, :, rows], k, v, w.scale, w.causal, rows=rows, nq=w.Nq)
    sec = time.perf_counter() - t0
    vis = np.clip(rows + (w.Nk - w.Nq) + 1, 0, w.Nk)
    return sec, 4.0 * w.d * float(vis.sum())


def oracle_decode_sample(q, kc, vc, sl, seqs):
    import oracle

    t0 = time.perf_counter()
    lens = sl.tolist()
    offs = np.concatenate([[0], np.cumsum(lens)])
    per = DECODE.Hkv * DECODE.d
    for b in seqs:
        a, e = int(offs[b]) * per, int(offs[b + 1]) * per
        oracle.decode_ref(q[b:b + 1], kc[a:e], vc[a:e], sl[b:b + 1], DECODE.scale, DECODE.Hkv)
    return time.perf_counter() - t0


def cores_used() -> dict:
    return {"cores": blas_threads(), "host_cpu_count": os.cpu_count(),
            "cores_note": "cores = BLAS threads of the oracle's matrix products (the rest of "
                          "the oracle is single-threaded numpy); host_cpu_count = os.cpu_count()"}


def cpu_baseline(budget_s: float = 12.0):
    """Time the oracle, as it stands, on a bounded sample of the headline
    workload (seeded random query rows of one head of the 128K prefill; the
    rate is those rows' algorithmic FLOPs over the oracle's time), plus a
    sample of the decode workload."""
    q, k, v = headline_head_inputs()
    rng = np.random.default_rng(HEADLINE.seed + 200)
    rows, spent, flops = [], 0.0, 0.0
    while spent < budget_s * 0.75:
        batch = rng.integers(0, HEADLINE.Nq, size=8)
        sec, fl = oracle_rows_sample(q, k, v, batch)
        spent += sec
        flops += fl
        rows.extend(int(r) for r in batch)
    _, dq, dkc, dvc, dsl = (None,) + workloads.decode_inputs(DECODE, device="cpu")
    seqs, dspent = [], 0.0
    while dspent < budget_s * 0.25 and len(seqs) < DECODE.B:
        dspent += oracle_decode_sample(dq, dkc, dvc, dsl, [len(seqs)])
        seqs.append(len(seqs))
    kv = decode_kv_bytes(dsl[: len(seqs)].numpy(), DECODE.Hkv, DECODE.d)
    out = {"value": flops / spent / 1e12, "unit": "TFLOP/s", "kind": "oracle",
           "sample": f"prefill: {len(rows)} seeded random query rows of one head of "
                     f"{HEADLINE.name} against its {HEADLINE.Nk} keys in {spent:.1f} s "
                     f"(algorithmic FLOPs of those rows / oracle time); decode: {len(seqs)} "
                     f"of {DECODE.B} sequences of {DECODE.name} in {dspent:.1f} s",
           "decode": {"value": kv / dspent / 1e9, "unit": "GB/s"}}
    out.update(cores_used())
    return out


def run_oracle_timing(budget_s: float = 10.0) -> int:
    """CPU only: the fp64 oracle, as it stands, on the small fp16 workload (whole)
    and on the 32K and 128K causal GQA workloads (a bounded set of query rows of
    one head, with the time for every row of every head extrapolated from the
    oracle's own cost per row, which is proportional to Nk: it scores a row
    against every key and then masks). Inputs have the workloads' shapes; the
    timing does not depend on their values. One JSON line per workload."""
    import torch

    import oracle

    cores = blas_threads()
    w0 = workloads.PREFILL_SMALL
    q, k, v = workloads.prefill_inputs(w0, device="cpu")
    t0 = time.perf_counter()
    oracle.attention_ref(q, k, v, w0.scale, w0.causal)
    sec = time.perf_counter() - t0
    print(json.dumps({"variant": f"oracle_cpu_{w0.name}", "kind": "oracle", "cores": cores,
                      "sample": "whole workload", "seconds": round(sec, 4),
                      "value": round(prefill_flops(w0) / sec / 1e9, 3), "unit": "GFLOP/s"}),
          flush=True)
    for w in (workloads.PREFILL_GQA_32K, workloads.PREFILL_GQA_128K):
        gen = torch.Generator().manual_seed(w.seed)
        kh = torch.randn(1, 1, w.Nk, w.d, generator=gen).to(torch.bfloat16)
        vh = torch.randn(1, 1, w.Nk, w.d, generator=gen).to(torch.bfloat16)
        rows, spent = [], 0.0
        rng = np.random.default_rng(w.seed + 100)
        while spent < budget_s / 2 and len(rows) < w.Nq:
            r = int(rng.integers(0, w.Nq))
            qh = torch.randn(1, 1, 1, w.d, generator=gen).to(torch.bfloat16)
            t0 = time.perf_counter()
            oracle.attention_ref(qh, kh, vh, w.scale, w.causal, rows=[r], nq=w.Nq)
            spent += time.perf_counter() - t0
            rows.append(r)
        full_rows = w.B * w.Hq * w.Nq
        print(json.dumps({
            "variant": f"oracle_cpu_{w.name}", "kind": "oracle", "cores": cores,
            "sample": f"{len(rows)} query rows of one head against all {w.Nk} keys",
            "seconds": round(spent, 3),
            "extrapolated_full_seconds": round(spent / len(rows) * full_rows, 1),
            "extrapolation": "per-row time x every row of every head (cost per row ~ Nk)"}),
            flush=True)
    return 0


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle, as it stands, on the host cores, on
    the same metric (TFLOP/s of the 128K causal GQA prefill); each step is a
    bounded sample (8 seeded random query rows of one head) of that workload,
    plus one decode sequence for the decode side."""
    if rank != 0:
        return 0
    q, k, v = headline_head_inputs()
    dq, dkc, dvc, dsl = workloads.decode_inputs(DECODE, device="cpu")
    rng = np.random.default_rng(HEADLINE.seed + 300)
    for _ in range(args.warmup):
        oracle_rows_sample(q, k, v, rng.integers(0, HEADLINE.Nq, size=8))
    pt = dt = fl = 0.0
    kv = 0
    for i in range(args.steps):
        sec, f = oracle_rows_sample(q, k, v, rng.integers(0, HEADLINE.Nq, size=8))
        pt += sec
        fl += f
        b = i % DECODE.B
        dt += oracle_decode_sample(dq, dkc, dvc, dsl, [b])
        kv += decode_kv_bytes(dsl[b:b + 1].numpy(), DECODE.Hkv, DECODE.d)
    value = fl / pt / 1e12
    sample = (f"each step: 8 seeded random query rows of one head of {HEADLINE.name} against "
              f"its {HEADLINE.Nk} keys (algorithmic FLOPs of those rows / oracle time), and 1 "
              f"of {DECODE.B} sequences of {DECODE.name}; fp64 numpy")
    cb = {"value": value, "unit": "TFLOP/s", "kind": "oracle", "sample": sample}
    cb.update(cores_used())
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": (pt + dt) / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{HEADLINE.name} (bounded sample per step)",
                   "parallelism": "rank 0 host cores"},
        "decode": {"value": kv / dt / 1e9, "unit": "GB/s"},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def prefill_roofline(w, ms, peaks, src, primary: str):
    """Roofline object of one prefill launch: algorithmic FLOPs / event time
    against the measured dense bf16 rate; `primary` picks which measured rate
    is `peak` (burst for a short launch, sustained for a launch long enough to
    sit at the power-capped clock), and both fractions are reported."""
    flops = prefill_flops(w)
    ach = flops / (ms * 1e-3) / 1e12
    burst = peaks["bf16_tflops"]
    sus = peaks.get("bf16_tflops_sustained", burst)
    peak = sus if primary == "sustained" else burst
    return {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
            "frac": ach / peak, "frac_burst": ach / burst, "frac_sustained": ach / sus,
            "traffic": profiled_traffic("attn_prefill_kernel", w.name),
            "kernel": f"attn_prefill_kernel<{w.d},bf16,{'causal' if w.causal else 'full'}>",
            "workload": w.name, "algorithmic_flops": flops, "ms_per_launch": ms,
            "peak_source": f"{src} bf16 dense matmul ({primary})",
            "nominal": {"peak": NOMINAL_PEAKS["bf16_tflops"],
                        "frac": ach / NOMINAL_PEAKS["bf16_tflops"]}}


def run_ours(args, world, rank, local):
    import torch
    import torch.distributed as dist

    import exact_tiled_attention_38_b200 as eta

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    eta.load_library()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    seed_off = 1000 * rank
    stream = torch.cuda.current_stream()
    # Device memory the library itself holds (device-wide free bytes before and
    # after the first call of each, once the module is loaded): prefill
    # allocates nothing; decode keeps its split workspace cached in the
    # library's pool. A materialised fp32 score matrix would take
    # B * Hq * Nq * Nk * 4 bytes.
    eta.attn_get_device_status(stream)  # loads the library's module (code, static arrays)
    memory = {"how": "device-wide free memory before and after the first call"}
    data = {}  # kernel name -> its inputs and outputs, set up when its phase starts

    def setup(name):
        torch.cuda.synchronize()
        if name == "decode":
            sl_cpu = workloads.decode_seqlens(DECODE.B, DECODE.lmin, DECODE.lmax,
                                              DECODE.seed + seed_off)
            dq, dkc, dvc, dsl = workloads.decode_inputs(DECODE, device=dev, seqlens=sl_cpu,
                                                        seed=DECODE.seed + seed_off)
            do = torch.empty_like(dq)
            dlse = torch.empty(DECODE.B, DECODE.Hq, device=dev, dtype=torch.float32)
            torch.cuda.synchronize()
            free0 = torch.cuda.mem_get_info(dev)[0]
            eta.attn_decode(dq, dkc, dvc, dsl, DECODE.Hkv, o=do, lse=dlse, scale=DECODE.scale,
                            stream=stream)
            torch.cuda.synchronize()
            memory["decode_library_bytes"] = free0 - torch.cuda.mem_get_info(dev)[0]
            data[name] = (sl_cpu, dq, dkc, dvc, dsl, do, dlse)
            return
        w = next(x for x in PREFILLS if PREFILL_KEYS[x.name] == name)
        q, k, v = workloads.prefill_inputs(w, device=dev, seed=w.seed + seed_off)
        o = torch.empty_like(q)
        lse = torch.empty(w.B, w.Hq, w.Nq, device=dev, dtype=torch.float32)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info(dev)[0]
        eta.attn_fwd(q, k, v, o=o, lse=lse, scale=w.scale, causal=w.causal, stream=stream)
        torch.cuda.synchronize()
        memory[f"prefill_{name}_library_bytes"] = free0 - torch.cuda.mem_get_info(dev)[0]
        memory[f"prefill_{name}_score_matrix_fp32_bytes"] = w.B * w.Hq * w.Nq * w.Nk * 4
        data[name] = (w, q, k, v, o, lse)

    # L2 flush before every kernel: write 256 MiB (> 126 MB L2), then read
    # another 256 MiB so that the dirty lines of the write are evicted (written
    # back) before the timed kernel starts rather than during it.
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.int32, device=dev)
    flush_rd = torch.zeros(64 * 1024 * 1024, dtype=torch.int32, device=dev)

    def flush_l2():
        flush.zero_()
        flush_rd.max()

    kernel_names = [PREFILL_KEYS[w.name] for w in PREFILLS] + ["decode"]

    def launch(name):
        if name == "decode":
            _, dq, dkc, dvc, dsl, do, dlse = data[name]
            eta.attn_decode(dq, dkc, dvc, dsl, DECODE.Hkv, o=do, lse=dlse, scale=DECODE.scale,
                            stream=stream)
            return
        w, q, k, v, o, lse = data[name]
        eta.attn_fwd(q, k, v, o=o, lse=lse, scale=w.scale, causal=w.causal, stream=stream)

    # The step's kernels are timed in phases, shortest first, and each phase
    # sets up its own workloads just before it: a launch of about 0.13 s (the
    # 128K prefill) holds the GPU at its power-capped clock for a while
    # afterwards, which would slow the short kernels if they followed it. Each
    # phase has its own warm-up and clock record (the short phase sampled
    # every millisecond); a step is one pass of every phase's kernels over
    # their batch, so ms_per_step is the sum of the phases' per-step times.
    phases = [("decode", "2k"), ("32k",), ("128k",)]
    ms, phase_ms, phase_clocks = {}, {}, {}
    for names in phases:
        for name in names:
            setup(name)

        def step(evs=None):
            for i, name in enumerate(names):
                flush_l2()
                if evs:
                    evs[2 * i].record(stream)
                launch(name)
                if evs:
                    evs[2 * i + 1].record(stream)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        code, raw = eta.attn_get_device_status(stream)
        if code != eta.ATTN_OK:
            raise RuntimeError(f"device status {code} ({raw:#x}) after warm-up of {names}")
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(names))]
               for _ in range(args.steps)]
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        period = 0.001 if names == phases[0] else 0.005
        with ClockSampler(local, period_s=period) as clocks:
            t_start.record(stream)
            for i in range(args.steps):
                step(evs[i])
            t_end.record(stream)
            torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        code, raw = eta.attn_get_device_status(stream)
        if code != eta.ATTN_OK:
            raise RuntimeError(f"device status {code} ({raw:#x}) in the timed loop of {names}")
        for i, name in enumerate(names):
            ms[name] = sum(e[2 * i].elapsed_time(e[2 * i + 1]) for e in evs) / args.steps
        phase_ms["+".join(names)] = t_start.elapsed_time(t_end) / args.steps
        phase_clocks["+".join(names)] = clocks
    pre = [data[PREFILL_KEYS[w.name]] for w in PREFILLS]
    n_ev = len(PREFILLS) + 1
    sl_cpu, dq, dkc, dvc, dsl, do, dlse = data["decode"]
    order = kernel_names + list(phase_ms)
    red = reduce_max([ms[n] for n in kernel_names] + [phase_ms[n] for n in phase_ms])
    ms_max = dict(zip(order, red))
    step_ms_max = sum(ms_max[n] for n in phase_ms)

    # ---- end to end through the public API, host buffers in pinned memory:
    # every step copies each workload's inputs host -> device, runs the call
    # and copies O and LSE back.
    e2e_steps = max(1, min(args.steps, 3))
    host = []
    for w, q, k, v, o, lse in pre:
        host.append(([t.cpu().pin_memory() for t in (q, k, v)],
                     [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (o, lse)],
                     [torch.empty_like(t) for t in (q, k, v)]))
    hdec = ([t.cpu().pin_memory() for t in (dq, dkc, dvc, dsl)],
            [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (do, dlse)],
            [torch.empty_like(t) for t in (dq, dkc, dvc, dsl)])
    nbytes = lambda ts: sum(t.numel() * t.element_size() for t in ts)  # noqa: E731
    seg_h2d = [nbytes(h[0]) for h in host] + [nbytes(hdec[0])]
    seg_d2h = [nbytes(h[1]) for h in host] + [nbytes(hdec[1])]

    def e2e_step(ev=None):
        for i, ((w, *_), (hin, hout, dbuf)) in enumerate(zip(pre, host)):
            if ev:
                ev[2 * i].record(stream)
            for dst, src in zip(dbuf, hin):
                dst.copy_(src, non_blocking=True)
            oo, ll = eta.attn_fwd(dbuf[0], dbuf[1], dbuf[2], scale=w.scale, causal=w.causal,
                                  stream=stream)
            hout[0].copy_(oo, non_blocking=True)
            hout[1].copy_(ll, non_blocking=True)
            if ev:
                ev[2 * i + 1].record(stream)
        hin, hout, dbuf = hdec
        if ev:
            ev[2 * n_ev - 2].record(stream)
        for dst, src in zip(dbuf, hin):
            dst.copy_(src, non_blocking=True)
        oo, ll = eta.attn_decode(dbuf[0], dbuf[1], dbuf[2], dbuf[3], DECODE.Hkv,
                                 scale=DECODE.scale, stream=stream)
        hout[0].copy_(oo, non_blocking=True)
        hout[1].copy_(ll, non_blocking=True)
        if ev:
            ev[2 * n_ev - 1].record(stream)

    e2e_step()
    torch.cuda.synchronize()
    eev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n_ev)]
           for _ in range(e2e_steps)]
    if world > 1:
        dist.barrier()
    for i in range(e2e_steps):
        e2e_step(eev[i])
    torch.cuda.synchronize()
    e2e_ms = reduce_max([sum(e[2 * i].elapsed_time(e[2 * i + 1]) for e in eev) / e2e_steps
                         for i in range(n_ev)])

    peaks, src = load_peaks()
    kv_bytes = decode_kv_bytes(sl_cpu.numpy(), DECODE.Hkv, DECODE.d)
    dbytes = decode_bytes(sl_cpu.numpy(), DECODE.B, DECODE.Hq, DECODE.Hkv, DECODE.d)
    dec_ms = ms["decode"]
    dec_ach = dbytes / (dec_ms * 1e-3) / 1e9
    hl_flops = prefill_flops(HEADLINE)
    value = aggregate_throughput(hl_flops, world, ms_max["128k"]) / 1e12
    # The 128K launch (about 0.13 s, most of a step's time) runs long enough to
    # sit at the power-capped clock: its fraction is taken of the sustained
    # measured rate, the shorter launches' of the burst rate; both are given.
    rl = {PREFILL_KEYS[w.name]: prefill_roofline(w, ms[PREFILL_KEYS[w.name]], peaks, src,
                                                 "sustained" if w is HEADLINE else "burst")
          for w, *_ in pre}
    prefill_lines = {PREFILL_KEYS[w.name]: {
        "value": aggregate_throughput(prefill_flops(w), world, ms_max[PREFILL_KEYS[w.name]]) / 1e12,
        "unit": "TFLOP/s", "ms_per_launch": ms[PREFILL_KEYS[w.name]],
        "clocks": phase_clocks[next(n for n in phase_clocks
                                    if PREFILL_KEYS[w.name] in n.split("+"))].summary()}
        for w, *_ in pre}
    e2e_seg = {PREFILL_KEYS[w.name]: {
        "value": aggregate_throughput(prefill_flops(w), world, e2e_ms[i]) / 1e12,
        "unit": "TFLOP/s", "h2d_bytes": seg_h2d[i], "d2h_bytes": seg_d2h[i]}
        for i, (w, *_) in enumerate(pre)}
    e2e_seg["decode"] = {"value": aggregate_throughput(kv_bytes, world, e2e_ms[-1]) / 1e9,
                         "unit": "GB/s", "h2d_bytes": seg_h2d[-1], "d2h_bytes": seg_d2h[-1]}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": HEADLINE.name,
            "prefill": {PREFILL_KEYS[w.name]: {
                "name": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.Nq, "d": w.d,
                "causal": w.causal, "std": w.std, "flops": prefill_flops(w)} for w in PREFILLS},
            "decode": {"name": DECODE.name, "B": DECODE.B, "Hq": DECODE.Hq, "Hkv": DECODE.Hkv,
                       "d": DECODE.d, "kv_tokens": int(sl_cpu.sum()), "kv_bytes": kv_bytes,
                       "nsplit": eta.attn_decode_num_splits(DECODE.B, DECODE.Hq, DECODE.Hkv,
                                                            DECODE.d)},
            "step": "decode and prefill 2K, then prefill 32K, then prefill 128K, each in its "
                    "own timed phase of `steps` iterations (shortest first, so that the 128K "
                    "launches' power-capped clock does not carry over into the short kernels); "
                    "each kernel timed with CUDA events on its stream",
            "l2": "flushed before every kernel (256 MiB write, then a 256 MiB read that "
                  "evicts its dirty lines; outside the kernel events); the 128K and 32K "
                  "inputs and the decode cache are also larger than L2",
            "parallelism": f"replicas x{world} (independent batches per GPU)",
            "memory": memory,
        },
        # The dominant kernel of a step is the 128K prefill launch (about 95 %
        # of the step's kernel time).
        "roofline": rl["128k"],
        "roofline_prefill_128k": rl["128k"],
        "roofline_prefill_32k": rl["32k"],
        "roofline_prefill_2k": rl["2k"],
        "roofline_decode": {
            "bound": "hbm", "achieved": dec_ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": dec_ach / peaks["hbm_gbs"],
            "traffic": profiled_traffic("attn_decode_persistent_kernel", DECODE.name),
            "kernel": "attn_decode_persistent_kernel<16,4,1,128,bf16> + attn_decode_gather_kernel "
                      "(one attn_decode call, timed together; batches of up to 2048 sequences "
                      "need no plan kernel)",
            "workload": DECODE.name, "algorithmic_bytes": dbytes, "ms_per_launch": dec_ms,
            "peak_source": f"{src} copy bandwidth (burst)",
            "nominal": {"peak": NOMINAL_PEAKS["hbm_gbs"],
                        "frac": dec_ach / NOMINAL_PEAKS["hbm_gbs"]}},
        "prefill": prefill_lines,
        "decode": {"value": aggregate_throughput(kv_bytes, world, ms_max["decode"]) / 1e9,
                   "unit": "GB/s (KV cache read)", "ms_per_call": dec_ms,
                   "clocks": phase_clocks["decode+2k"].summary()},
        "e2e": {"value": e2e_seg["128k"]["value"], "unit": "TFLOP/s",
                "h2d_bytes_per_step": seg_h2d[0], "d2h_bytes_per_step": seg_d2h[0],
                "what": "the 128K prefill through the public binding: H2D of q, k, v from "
                        "pinned host memory, attn_fwd, D2H of O and LSE, per step",
                "segments": e2e_seg, "steps": e2e_steps},
        "clocks": merged_clocks(list(phase_clocks.values())),
        "phases_ms_per_step": phase_ms,
        # 3 prefill launches + decode stream and gather per step
        "gpu_launches": (len(PREFILLS) + 2) * args.steps,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_profile(args, local):
    """Launch one phase of the step `warmup + steps` times with no timing or
    output: the target of an ncu capture (a small, self-contained command)."""
    import torch

    import exact_tiled_attention_38_b200 as eta

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    eta.load_library()
    if args.profile.startswith("prefill"):
        w = {"prefill": PREFILL, "prefill_32k": workloads.PREFILL_GQA_32K,
             "prefill_128k": workloads.PREFILL_GQA_128K,
             "prefill_d64": variant_by_name("prefill_causal_mha_b4_h16_n2048_d64")}[args.profile]
        q, k, v = workloads.prefill_inputs(w, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty(w.B, w.Hq, w.Nq, device=dev, dtype=torch.float32)
        for _ in range(args.warmup + args.steps):
            eta.attn_fwd(q, k, v, o=o, lse=lse, scale=w.scale, causal=w.causal)
    else:
        dq, dkc, dvc, dsl = workloads.decode_inputs(DECODE, device=dev)
        do = torch.empty_like(dq)
        dlse = torch.empty(DECODE.B, DECODE.Hq, device=dev, dtype=torch.float32)
        for _ in range(args.warmup + args.steps):
            eta.attn_decode(dq, dkc, dvc, dsl, DECODE.Hkv, o=do, lse=dlse, scale=DECODE.scale)
    torch.cuda.synchronize()
    code, raw = eta.attn_get_device_status()
    if code != eta.ATTN_OK:
        raise RuntimeError(f"device status {code} ({raw:#x})")
    return 0


def variant_by_name(name):
    return next(w for w in variant_workloads() if w.name == name)


def variant_workloads():
    """Extra shapes measured by --variants: the other head groupings, head sizes
    and dtypes of the same kernels (the 2K, 32K and 128K prefill configs and the
    ragged decode config are in the bench step itself)."""
    P, D, sb = workloads.PrefillWorkload, workloads.DecodeWorkload, workloads.SEED_BASE + 20
    return [
        P("prefill_noncausal_mha_b4_h16_n4096_d128", 4, 16, 16, 4096, 4096, 128, "bf16", False, sb),
        P("prefill_causal_mha_b4_h16_n2048_d64", 4, 16, 16, 2048, 2048, 64, "bf16", True, sb + 1),
        P("prefill_causal_mha_b4_h16_n2048_d128_f16", 4, 16, 16, 2048, 2048, 128, "f16", True,
          sb + 2),
        P("prefill_causal_mqa_b2_h32kv1_n4096_d128", 2, 32, 1, 4096, 4096, 128, "bf16", True,
          sb + 3),
        P("prefill_chunk_gqa_b1_h32kv8_nq2048_nk32768_d128", 1, 32, 8, 2048, 32768, 128, "bf16",
          True, sb + 4),
        D("decode_mqa_b64_h32kv1_d128_ragged", 64, 32, 1, 128, 1024, 8192, "bf16", sb + 5),
        D("decode_gqa8_b64_h64kv8_d128_ragged", 64, 64, 8, 128, 1024, 8192, "bf16", sb + 6),
        D("decode_mha_b64_h8kv8_d128_ragged", 64, 8, 8, 128, 1024, 8192, "bf16", sb + 7),
        D("decode_gqa_b64_h32kv8_d128_ragged_f16", 64, 32, 8, 128, 1024, 8192, "f16", sb + 8),
        D("decode_gqa_b64_h32kv8_d64_ragged", 64, 32, 8, 64, 1024, 8192, "bf16", sb + 9),
        D("decode_gqa16_b64_h128kv8_d128_ragged", 64, 128, 8, 128, 1024, 8192, "bf16", sb + 10),
    ]


def run_variants(args, local):
    """One JSON line per extra workload: median CUDA-event time of single
    launches, L2 flushed before each, against the measured peaks."""
    import torch

    import exact_tiled_attention_38_b200 as eta

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    eta.load_library()
    peaks, _ = load_peaks()
    flush = torch.empty(64 << 20, dtype=torch.int32, device=dev)
    flush_rd = torch.empty(64 << 20, dtype=torch.int32, device=dev)
    for w in variant_workloads():
        f16 = w.dtype == "f16"
        if isinstance(w, workloads.PrefillWorkload):
            q, k, v = workloads.prefill_inputs(w, device=dev)
            o = torch.empty_like(q)
            lse = torch.empty(w.B, w.Hq, w.Nq, device=dev, dtype=torch.float32)
            fn = eta.attn_fwd_f16 if f16 else eta.attn_fwd

            def call():
                fn(q, k, v, o=o, lse=lse, scale=w.scale, causal=w.causal)

            work, unit, peak = prefill_flops(w), "TFLOP/s", peaks["bf16_tflops"]
            scale_units = 1e9
        else:
            q, kc, vc, sl = workloads.decode_inputs(w, device=dev)
            o = torch.empty_like(q)
            lse = torch.empty(w.B, w.Hq, device=dev, dtype=torch.float32)
            fn = eta.attn_decode_f16 if f16 else eta.attn_decode

            def call():
                fn(q, kc, vc, sl, w.Hkv, o=o, lse=lse, scale=w.scale)

            work, unit, peak = decode_kv_bytes(sl.cpu(), w.Hkv, w.d), "GB/s", peaks["hbm_gbs"]
            scale_units = 1e6
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        reps = 5 if work > 5e13 else 15
        ts = []
        with ClockSampler(local) as clocks:
            for _ in range(reps):
                flush.zero_()
                flush_rd.max()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                call()
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
        code, raw = eta.attn_get_device_status()
        if code != eta.ATTN_OK:
            raise RuntimeError(f"{w.name}: device status {code} ({raw:#x})")
        ms = statistics.median(ts)
        val = work / ms / scale_units
        line = {"variant": w.name, "value": round(val, 1), "unit": unit,
                "ms_per_launch": round(ms, 4), "frac": round(val / peak, 4), "peak": peak,
                "launches": reps, "clocks": clocks.summary()}
        if unit == "TFLOP/s" and "bf16_tflops_sustained" in peaks:
            line["frac_sustained"] = round(val / peaks["bf16_tflops_sustained"], 4)
        print(json.dumps(line), flush=True)
        del q, o, lse
        torch.cuda.empty_cache()
    run_ring_variant(eta, dev, local, peaks, flush, flush_rd)
    return 0


def run_ring_variant(eta, dev, local, peaks, flush, flush_rd, world=8):
    """Context-parallel prefill of the 128K causal GQA workload over an
    8-rank zigzag ring: rank 0's whole call sequence (8 steps, 2 chunk pairs
    each, plus the LSE merges) on this one GPU, with LocalRing's device copies
    standing in for the K/V transfers. Every rank does the same work, so the
    per-rank rate is what each GPU of an 8-GPU ring would compute."""
    import torch

    from exact_tiled_attention_38_b200 import context_parallel as cp

    w = workloads.PREFILL_GQA_128K
    q, k, v = workloads.prefill_inputs(w, device=dev)
    ks = [cp.shard_zigzag(k, r, world) for r in range(world)]
    vs = [cp.shard_zigzag(v, r, world) for r in range(world)]
    q0 = cp.shard_zigzag(q, 0, world)
    del q, k, v
    torch.cuda.empty_cache()
    c = w.Nq // (2 * world)
    flops = 4.0 * w.d * w.Hq * w.B * (2 * world * c * c + c)  # one rank's visible pairs

    def call():
        cp.ring_attention(q0, ks[0], vs[0], True, w.scale, exchange=cp.LocalRing(0, ks, vs))

    call()
    torch.cuda.synchronize()
    ts = []
    with ClockSampler(local) as clocks:
        for _ in range(3):
            flush.zero_()
            flush_rd.max()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
    code, raw = eta.attn_get_device_status()
    if code != eta.ATTN_OK:
        raise RuntimeError(f"ring: device status {code} ({raw:#x})")
    ms = statistics.median(ts)
    val = flops / ms / 1e9
    print(json.dumps({"variant": f"prefill_ring_w{world}_rank0_causal_gqa_b1_h32kv8_n128k_d128",
                      "value": round(val, 1), "unit": "TFLOP/s", "ms_per_launch": round(ms, 4),
                      "frac": round(val / peaks["bf16_tflops"], 4), "peak": peaks["bf16_tflops"],
                      "launches": len(ts), "chunk": c, "clocks": clocks.summary(),
                      "frac_sustained": round(val / peaks.get("bf16_tflops_sustained",
                                                              peaks["bf16_tflops"]), 4)}),
          flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=("prefill", "prefill_32k", "prefill_128k", "prefill_d64", "decode"), default=None,
                    help="only launch this phase (an ncu target); prints nothing")
    ap.add_argument("--oracle-timing", action="store_true",
                    help="CPU only: time the fp64 oracle on the small, 32K and 128K workloads "
                         "(sampled rows, extrapolated)")
    ap.add_argument("--variants", action="store_true",
                    help="measure the extra shapes (long context, head groupings, d, dtype), "
                         "one JSON line each, instead of the step")
    args = ap.parse_args(argv)
    if args.warmup < 3 and not args.profile:
        ap.error("--warmup must be >= 3")
    if args.oracle_timing:
        return run_oracle_timing()
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.profile:
        return run_profile(args, local)
    if args.variants:
        return run_variants(args, local)
    return run_ours(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
