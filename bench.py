#!/usr/bin/env python
"""Benchmark: paged decode attention KV-read GB/s and tokens/s on B200.

Workload (one "step" = one pass of the whole hot path over one batch):
  long-context split-K decode -- batch 4, seqlen_q 1, context 131072 tokens
  each, Hq 32 / Hkv 8, head_dim 128, bf16 N(0,1) data, contiguous paged cache
  with block_size 16 and a seeded randperm block table [4, 8192], fixed split
  chunk 4096 tokens merged in global block order.  A step appends the newest
  token's K/V (position 131071) and runs decode attention over the
  131072-token contexts (split kernel + merge kernel), the append fused into
  the same call (paged_decode_attn_append).

value   = algorithmic KV bytes (every visible token read once per KV head, K
          and V, bf16) of all ranks / device time of the K timed steps (max
          over ranks), in GB/s.  The 2.15 GB cache is larger than L2, so no
          flush is needed between steps.
e2e     = the same metric through the public API with pinned host buffers:
          each step copies q, the new K/V, the sequence lengths and the block
          table host->device (packed in one pinned buffer, one copy) and the
          output and lse device->host (one copy), on a copy stream with two
          buffer sets so that step k + 1's inputs and step k's results move
          while the neighbouring step computes.
roofline: the decode call's KV bytes / its mean CUDA-event duration, against
          the measured HBM copy bandwidth.
cpu_baseline: the CPU fp64 oracle on a bounded sample of the same workload.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: torchrun --nproc-per-node N bench.py --gpus N  (weak scaling: each
rank runs its own batch; there is no collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode attention KV-read GB/s (% of HBM peak) and tokens/s at 1 B200"
WORKLOAD = ("long-context split-K decode: batch 4, seqlen_q 1, context 131072, Hq 32, Hkv 8, "
            "head_dim 128, bf16, contiguous paged cache block_size 16, randperm block_table "
            "[4, 8192], split chunk 4096 tokens")
FALLBACK_HBM_GBS = 6650.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
L2_BYTES = 126 * 1024 * 1024  # B200 L2


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--context", type=int, default=131072,
                    help="tokens per sequence (a smaller workload for profiling captures)")
    ap.add_argument("--batch", type=int, default=4)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the secondary objects (prefill, varlen, backward, other decode "
                         "workloads): the decode step alone, for launch-list captures")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the prefill backward and print its result object")
    ap.add_argument("--varlen-only", action="store_true",
                    help="time only the packed mixed-batch call and print its result object")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only the chunked causal prefill (--steps repetitions, "
                         "2 warm-up passes) and print its result object")
    return ap.parse_args()


def dist_env():
    from paged_kv_decode_31_b200 import dist as pdist
    return pdist.rank_env()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_decode_31_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per decode call from the committed ncu summary, or None if
    the kernels changed since those counters were taken."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            t = json.load(f)
        if t.get("kernel_digest") == kernel_source_digest():
            return int(t["dram_bytes_per_call"])
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML (read-only) while the
    timed region runs."""

    REASONS = {
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sync_boost": 0x10,
        "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                self.reasons |= int(n.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        names = [k for k, bit in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def cpu_baseline(di_dev, n_seq: int = 4):
    """The fp64 oracle on a bounded sample -- the first n_seq sequences (all
    four by default: the whole workload), every KV head, full context -- on
    every host core (one oracle task per query row).  Returns the cpu_baseline
    object."""
    import oracle
    from paged_kv_decode_31_b200 import inputs as I
    host_cores = os.cpu_count() or 1
    oracle.set_num_threads(host_cores)
    host = I.DecodeInputs(di_dev.q[:n_seq].cpu(), di_dev.cache.to("cpu"),
                          di_dev.block_table[:n_seq].cpu(), di_dev.seqlens[:n_seq].cpu(),
                          di_dev.Hq, di_dev.Hkv, di_dev.D, di_dev.scale, di_dev.causal)
    t0 = time.perf_counter()
    oracle.paged_attn(host.q, host.cache.k, host.cache.v, host.block_table, host.seqlens,
                      host.scale, host.causal)
    dt = time.perf_counter() - t0
    gbs = host.kv_bytes() / dt / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": oracle.num_threads(),
            "host_cores": host_cores, "kind": "oracle",
            "sample": f"{n_seq} of {di_dev.batch} sequences, all {di_dev.Hkv} KV heads, full "
                      f"131072-token context ({host.kv_bytes()} KV bytes) in {dt:.2f} s",
            "tokens_per_s": round(n_seq / dt, 4)}


def prefill_secondary(dev, reps: int = 20):
    """Chunked causal prefill of the parity workload (batch 8, Hq 16 / Hkv 4,
    D 128, block_size 16): 4 chunks of 512 tokens, each appended and attended
    by one paged_decode_attn_append call (an append launch, then the row-major
    attention kernel).  Algorithmic flops: 4 * D per (query row, visible key) for
    Q K^T and P V.  Returns the secondary result object."""
    import paged_kv_decode_31_b200 as pkv
    from paged_kv_decode_31_b200 import inputs as I
    cache, table, q_all, k_all, v_all = I.config_parity_cache(device=dev)
    B, Hq, D, chunk = 8, 16, 128, 512
    outs = [torch.empty(B, chunk, Hq, D, dtype=torch.bfloat16, device=dev) for _ in range(4)]
    lses = [torch.empty(B, Hq, chunk, dtype=torch.float32, device=dev) for _ in range(4)]
    ws = torch.empty(pkv.workspace_size(B, chunk, Hq, D, 2048), dtype=torch.uint8, device=dev)
    seqs = [torch.full((B,), chunk * (c + 1), dtype=torch.int32, device=dev) for c in range(4)]

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(reps)]

    def prefill(marks=None):
        for c in range(4):
            if marks is not None:
                marks[c].record()
            s, e = chunk * c, chunk * (c + 1)
            pkv.paged_decode_attn_append(q_all[:, s:e], k_all[:, s:e], v_all[:, s:e], cache.k,
                                         cache.v, table, seqs[c], max_seqlen_k=e, causal=True,
                                         out=outs[c], lse=lses[c], workspace=ws)
        if marks is not None:
            marks[4].record()

    for _ in range(2):
        prefill()
    torch.cuda.synchronize()
    for r in range(reps):
        prefill(ev[r])
    torch.cuda.synchronize()
    chunk_ms = [sum(ev[r][c].elapsed_time(ev[r][c + 1]) for r in range(reps)) / reps
                for c in range(4)]
    ms = sum(ev[r][0].elapsed_time(ev[r][4]) for r in range(reps)) / reps
    pairs = sum(p + 1 for p in range(4 * chunk))          # (query token, visible key)
    flops = 4.0 * D * pairs * B * Hq
    tflops = flops / (ms / 1e3) / 1e12
    return {"workload": "chunked causal prefill, batch 8 x 2048 tokens in 4 chunks of 512, "
                        "Hq 16, Hkv 4, D 128, block_size 16 (append + attention per chunk)",
            "ms_per_prefill": round(ms, 4), "tflops": round(tflops, 2),
            "chunk_us": [round(1e3 * x, 1) for x in chunk_ms],
            "algorithmic_flops": flops}


# Packed mixed batch for the varlen measurement: (requests, queries each, context)
VARLEN_MIX = [(16, 1, 16384), (8, 4, 8192), (6, 256, 2048), (2, 1024, 4096)]


def varlen_secondary(dev, reps: int = 10):
    """One packed multi-request call (paged_varlen_attn) over a mix of decode
    steps, multi-token steps and prefill chunks (VARLEN_MIX; Hq 32 / Hkv 8,
    D 128, block_size 16, causal), with each request's final row selected as
    well.  Reports the call time, queries/s, the unique K/V bytes / time and
    the algorithmic flops (4 * D per (query row, visible key)) / time."""
    import paged_kv_decode_31_b200 as pkv
    from paged_kv_decode_31_b200 import inputs as I
    Hq, Hkv, D, bs = 32, 8, 128, 16
    lengths, ctx = [], []
    for count, n, c in VARLEN_MIX:
        lengths += [n] * count
        ctx += [c] * count
    B = len(ctx)
    gen = torch.Generator().manual_seed(2024)
    nblk = [(c + bs - 1) // bs for c in ctx]
    gen_d = torch.Generator(device=dev).manual_seed(2025)
    cache = I.make_cache(sum(nblk) + 64, bs, Hkv, D, "contiguous", gen_d, device=dev)
    perm = torch.randperm(sum(nblk) + 64, generator=gen)[:sum(nblk)].to(torch.int32)
    table = torch.zeros(B, max(nblk), dtype=torch.int32)
    o = 0
    for b, k in enumerate(nblk):
        table[b, :k] = perm[o:o + k]
        o += k
    table = table.to(dev)
    seqlens = torch.tensor(ctx, dtype=torch.int32, device=dev)
    cu = torch.tensor([0] + torch.tensor(lengths).cumsum(0).tolist(), dtype=torch.int32,
                      device=dev)
    total_q = int(sum(lengths))
    q = I.randn_bf16((total_q, Hq, D), gen).to(dev)
    out = torch.empty(total_q, Hq, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(Hq, total_q, dtype=torch.float32, device=dev)
    fo = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
    fl = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ws = torch.empty(pkv.varlen_workspace_size(total_q, Hq, D, max(ctx)), dtype=torch.uint8,
                     device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        pkv.paged_varlen_attn(q, cache.k, cache.v, table, seqlens, cu, max(lengths),
                              max_seqlen_k=max(ctx), causal=True, out=out, lse=lse,
                              final_out=fo, final_lse=fl, workspace=ws, err=err)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        call()
    b_.record()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"varlen call set device error bits {int(err.item())}")
    ms = a.elapsed_time(b_) / reps
    kv_bytes = sum(c * Hkv * 2 * D * 2 for c in ctx)
    pairs = sum(sum(c - n + i + 1 for i in range(n)) for n, c in zip(lengths, ctx))
    flops = 4.0 * D * pairs * Hq
    return {"workload": "packed causal batch of " + ", ".join(
                f"{k} x {n} queries at context {c}" for k, n, c in VARLEN_MIX) +
                f" ({B} requests, {total_q} query tokens), Hq 32, Hkv 8, D 128, block_size 16, "
                "final rows selected",
            "ms_per_call": round(ms, 4), "queries_per_s": round(total_q / (ms / 1e3), 1),
            "kv_gbs": round(kv_bytes / (ms / 1e3) / 1e9, 2), "kv_bytes": kv_bytes,
            "tflops": round(flops / (ms / 1e3) / 1e12, 2), "algorithmic_flops": flops}


def backward_secondary(dev, reps: int = 20):
    """Deterministic backward of the full causal prefill of the parity
    workload (batch 8 x 2048 tokens, Hq 16 / Hkv 4, D 128, block_size 16):
    one forward for out / lse, then paged_prefill_attn_bwd timed alone.
    Algorithmic flops: 10 * D per (query row, visible key) -- the five
    products S, dP, dV, dK, dQ; the kernels' recompute of S and dP for dQ is
    not counted."""
    import paged_kv_decode_31_b200 as pkv
    from paged_kv_decode_31_b200 import inputs as I
    cache, table, q_all, k_all, v_all = I.config_parity_cache(device=dev)
    B, Hq, D, T = 8, 16, 128, 2048
    seq = torch.full((B,), T, dtype=torch.int32, device=dev)
    pkv.kv_append(k_all[:, :T], v_all[:, :T], cache.k, cache.v, table, seq - T)
    q = q_all[:, :T].contiguous()
    out, lse = pkv.paged_prefill_attn(q, cache.k, cache.v, table, seq, max_seqlen_k=T,
                                      causal=True)
    gen = torch.Generator(device=dev).manual_seed(77)
    dout = torch.randn(B, T, Hq, D, generator=gen, device=dev).to(torch.bfloat16)
    dq = torch.empty_like(q)
    dk = torch.zeros(tuple(cache.k.shape), dtype=torch.bfloat16, device=dev)
    dv = torch.zeros(tuple(cache.v.shape), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def bwd():
        pkv.paged_prefill_attn_bwd(q, cache.k, cache.v, table, seq, out, lse, dout,
                                   max_seqlen_k=T, causal=True, dq=dq, dk_cache=dk, dv_cache=dv,
                                   err=err)

    for _ in range(2):
        bwd()
    torch.cuda.synchronize()
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        bwd()
    b_.record()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"backward set device error bits {int(err.item())}")
    ms = a.elapsed_time(b_) / reps
    pairs = sum(p + 1 for p in range(T))
    flops = 10.0 * D * pairs * B * Hq
    return {"workload": "deterministic backward of causal prefill, batch 8 x 2048 tokens, "
                        "Hq 16, Hkv 4, D 128, block_size 16 (dq and the cache gradients)",
            "ms_per_call": round(ms, 4), "tflops": round(flops / (ms / 1e3) / 1e12, 2),
            "algorithmic_flops": flops}


def decode_workload_secondary(dev, name: str, reps: int = 200, warmup: int = 20):
    """The other timed decode workloads: `gqa_shard` (batch 32 x 4096, Hq 32 /
    Hkv 8, D 128, block_size 16, contiguous) and `ragged` (batch 64, contexts
    U[1, 32768], Hq 16 / Hkv 4, D 128, block_size 256, interleaved, NaN tails
    and spare blocks).  One paged_decode_attn call per step, 20 warm-up and
    200 timed steps with CUDA events per call; K/V bytes per call /
    device time (mean, median, best); then 200 more steps back to back
    between one event pair (`gbs_loop`, the steady-state rate the headline
    `value` measures, without the per-call events in the stream).  Inputs are
    larger than L2."""
    import paged_kv_decode_31_b200 as pkv
    from paged_kv_decode_31_b200 import inputs as I
    # drawn on the host (the generators are CPU ones), then moved
    di = (I.config_gqa_shard if name == "gqa_shard" else I.config_ragged)().to(dev)
    msk = int(di.seqlens.max().item())
    ws = torch.empty(pkv.workspace_size(di.q.shape[0], 1, di.Hq, di.D, msk), dtype=torch.uint8,
                     device=dev)
    out = torch.empty(tuple(di.q.shape), dtype=torch.bfloat16, device=dev)
    lse = torch.empty(di.q.shape[0], di.Hq, 1, dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        pkv.paged_decode_attn(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens,
                              max_seqlen_k=msk, scale=di.scale, causal=False, out=out, lse=lse,
                              workspace=ws, err=err)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for a, b in ev:
        a.record()
        call()
        b.record()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())}")
    t = sorted(a.elapsed_time(b) for a, b in ev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        call()
    e1.record()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())}")
    loop = e0.elapsed_time(e1) / reps
    kv = di.kv_bytes()
    mean = sum(t) / len(t)
    return {"workload": name, "kv_bytes": kv, "ms_mean": round(mean, 5),
            "ms_median": round(t[len(t) // 2], 5), "ms_best": round(t[0], 5),
            "gbs_mean": round(kv / (mean / 1e3) / 1e9, 2),
            "gbs_best": round(kv / (t[0] / 1e3) / 1e9, 2),
            "ms_loop": round(loop, 5), "gbs_loop": round(kv / (loop / 1e3) / 1e9, 2)}


def packed_layout(tensors):
    """Byte offsets of `tensors` laid end to end in one buffer, each start
    16-byte aligned, and the buffer's size."""
    offs, off = [], 0
    for t in tensors:
        offs.append(off)
        off += (t.numel() * t.element_size() + 15) // 16 * 16
    return offs, off


def packed_views(buf, like, offs):
    """Views of the uint8 buffer `buf` with the dtypes and shapes of `like`
    (contiguous), at the offsets of packed_layout."""
    return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(tuple(t.shape))
            for t, o in zip(like, offs)]


def run_ours(args):
    import torch.distributed as dist
    import paged_kv_decode_31_b200 as pkv
    from paged_kv_decode_31_b200 import dist as pdist
    from paged_kv_decode_31_b200 import inputs as I

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        pdist.init("nccl", device=dev)
    di = I.config_long_context(seed=1000 + rank, device=dev, batch=args.batch,
                               seqlen=args.context)
    B, ctx, Hq, Hkv, D = di.batch, int(di.seqlens[0].item()), di.Hq, di.Hkv, di.D
    gen = torch.Generator(device=dev).manual_seed(2000 + rank)
    k_new = torch.randn(B, 1, Hkv, D, generator=gen, device=dev).to(torch.bfloat16)
    v_new = torch.randn(B, 1, Hkv, D, generator=gen, device=dev).to(torch.bfloat16)
    seq = di.seqlens
    out = torch.empty(B, 1, Hq, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, Hq, 1, dtype=torch.float32, device=dev)
    ws = torch.empty(pkv.workspace_size(B, 1, Hq, D, ctx), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    kv_bytes = di.kv_bytes()

    def step(ev0=None, ev1=None):
        # kv_append of the newest token fused into the decode call
        if ev0 is not None:
            ev0.record(stream)
        pkv.paged_decode_attn_append(di.q, k_new, v_new, di.cache.k, di.cache.v, di.block_table,
                                     seq, max_seqlen_k=ctx, scale=di.scale, causal=False, out=out,
                                     lse=lse, workspace=ws, err=err)
        if ev1 is not None:
            ev1.record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())}")

    # per-launch durations for the roofline: events around every tenth step
    # of the timed loop (an event pair around every step costs the loop ~1 %)
    ev_every = 10 if args.steps >= 20 else 1
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           if k % ev_every == 0 else (None, None) for k in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t_start.record(stream)
        for k in range(args.steps):
            step(*evs[k])
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = t_start.elapsed_time(t_end)
    decode_ms = [a.elapsed_time(b) for a, b in evs if a is not None]
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())}")

    # e2e through the public API with pinned host buffers: the step's inputs
    # (q, the new K/V, the lengths, the block table) travel in one pinned
    # buffer and its results (out, lse) come back in another -- one copy each
    # way per step, the call itself taking views of the device buffers.  Two
    # sets of device buffers and a copy stream: step k + 1's inputs go in and
    # step k's results come out while step k / k + 1 computes, as a serving
    # loop would run it; every step's own copies stay inside the timed region.
    e2e = None
    if not args.no_e2e:
        ins = (di.q, k_new, v_new, seq, di.block_table)
        in_offs, h2d = packed_layout(ins)
        h_in = torch.empty(h2d, dtype=torch.uint8).pin_memory()
        for t, hv in zip(ins, packed_views(h_in, ins, in_offs)):
            hv.copy_(t.cpu())
        res = (out, lse)
        res_offs, d2h = packed_layout(res)
        d_in = [torch.empty(h2d, dtype=torch.uint8, device=dev) for _ in range(2)]
        v_in = [packed_views(d, ins, in_offs) for d in d_in]
        d_res = [torch.empty(d2h, dtype=torch.uint8, device=dev) for _ in range(2)]
        v_res = [packed_views(d, res, res_offs) for d in d_res]
        h_res = [torch.empty(d2h, dtype=torch.uint8).pin_memory() for _ in range(2)]
        cs = torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]    # slot's inputs landed
        ev_done = [torch.cuda.Event() for _ in range(2)]  # slot's call finished
        ev_out = [torch.cuda.Event() for _ in range(2)]   # slot's results copied out

        def copy_in(k):
            j = k & 1
            if k >= 2:
                cs.wait_event(ev_done[j])  # step k - 2 no longer reads d_in[j]
            with torch.cuda.stream(cs):
                d_in[j].copy_(h_in, non_blocking=True)
            ev_in[j].record(cs)

        def call(k):
            j = k & 1
            stream.wait_event(ev_in[j])
            if k >= 2:
                stream.wait_event(ev_out[j])  # step k - 2's results left d_res[j]
            d_q, d_kn, d_vn, d_s, d_bt = v_in[j]
            e_out, e_lse = v_res[j]
            pkv.paged_decode_attn_append(d_q, d_kn, d_vn, di.cache.k, di.cache.v, d_bt, d_s,
                                         max_seqlen_k=ctx, scale=di.scale, causal=False,
                                         out=e_out, lse=e_lse, workspace=ws, err=err)
            ev_done[j].record(stream)

        def copy_out(k):
            j = k & 1
            cs.wait_event(ev_done[j])
            with torch.cuda.stream(cs):
                h_res[j].copy_(d_res[j], non_blocking=True)
            ev_out[j].record(cs)

        def e2e_steps(n):
            cs.wait_stream(stream)
            copy_in(0)
            for k in range(n):
                if k + 1 < n:
                    copy_in(k + 1)
                call(k)
                copy_out(k)
            stream.wait_stream(cs)

        e2e_steps(max(3, args.warmup))
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_steps(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        if int(err.item()) != 0:
            raise RuntimeError(f"device error bits {int(err.item())}")
        # both host slots hold the call's results for the same inputs: the bits
        # of the device-timed steps' out
        out_bits = out.view(torch.int16).cpu()
        for j in range(2):
            h_out = packed_views(h_res[j], res, res_offs)[0]
            if not torch.equal(h_out.view(torch.int16), out_bits):
                raise RuntimeError("e2e results differ from the device-timed steps' out")
        e2e_ms = pdist.max_over_ranks(e0.elapsed_time(e1), device=dev)
        e2e = {"value": round(pdist.weak_scaling_rate(kv_bytes, world, args.steps, e2e_ms) / 1e9, 2),
               "unit": "GB/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e2e_ms / args.steps, 5),
               "copies": "one pinned host->device and one device->host copy per step on a "
                         "copy stream, overlapping the neighbouring steps' calls (two buffer sets)"}

    ms_total = pdist.max_over_ranks(ms_total, device=dev)
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    peak, peak_kind = measured_peaks()
    ms_step = ms_total / args.steps
    value = pdist.weak_scaling_rate(kv_bytes, world, args.steps, ms_total) / 1e9
    dec_ms = statistics.mean(decode_ms)
    achieved = kv_bytes / (dec_ms / 1e3) / 1e9
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": B, "seqlen_q": 1, "seqlen_k": ctx,
                   "Hq": Hq, "Hkv": Hkv, "head_dim": D, "block_size": 16,
                   "split_tokens": pkv.SPLIT_TOKENS,
                   "step": "paged_decode_attn_append: kv_append of 1 token/sequence fused into the decode call",
                   "l2": (f"inputs larger than L2 ({kv_bytes / 1e9:.3g} GB of K/V per rank), no flush"
                          if kv_bytes > L2_BYTES else
                          f"inputs NOT larger than L2 ({kv_bytes / 1e9:.3g} GB of K/V per rank): "
                          "a profiling size, not a bench number"),
                   "parallelism": f"dp{world}"},
        "tokens_per_s": round(B * world * args.steps / (ms_total / 1e3), 1),
        "hbm_frac": round(value / world / peak, 4),
        "hbm_frac_basis": f"{peak_kind} HBM copy bandwidth {peak} GB/s",
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     # the ncu figure belongs to the full-size workload only
                     "traffic": profiled_traffic() if (args.context, args.batch) == (131072, 4) else None,
                     "kernel": "paged_decode_attn_append (attn_split_kernel<128,16,3,2> + merge_kernel<128>)",
                     "algorithmic_bytes_per_launch": kv_bytes,
                     "launch_ms_mean": round(dec_ms, 5),
                     "launch_ms_median": round(statistics.median(decode_ms), 5),
                     "launch_ms_min": round(min(decode_ms), 5),
                     "launches_timed": len(decode_ms),
                     "peak_basis": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback 6.65 TB/s"},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks.summary(),
        "e2e": e2e,
    }
    if (args.context, args.batch) != (131072, 4):
        result["config"]["workload"] = (f"profiling size: batch {B}, context {ctx} "
                                        "(otherwise as the long-context workload)")
    if world == 1 and (args.context, args.batch) == (131072, 4) and not args.no_secondary:
        bf16_peak = None
        try:
            with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
                bf16_peak = float(json.load(f)["bf16_tflops"])
        except Exception:
            bf16_peak = 1590.0

        def prefill_obj():
            pre = prefill_secondary(dev)
            pre["tensor_peak_tflops"] = bf16_peak
            pre["frac_of_tensor_peak"] = round(pre["tflops"] / bf16_peak, 4)
            return pre

        def varlen_obj():
            vl = varlen_secondary(dev)
            vl["hbm_frac"] = round(vl["kv_gbs"] / peak, 4)
            vl["frac_of_tensor_peak"] = round(vl["tflops"] / bf16_peak, 4)
            return vl

        def backward_obj():
            bw = backward_secondary(dev)
            bw["frac_of_tensor_peak"] = round(bw["tflops"] / bf16_peak, 4)
            return bw

        def decode_obj(name):
            dw = decode_workload_secondary(dev, name)
            dw["hbm_frac"] = round(dw["gbs_loop"] / peak, 4)
            dw["hbm_frac_basis"] = "gbs_loop"
            return dw

        secondary = [("prefill", prefill_obj), ("varlen", varlen_obj), ("backward", backward_obj),
                     ("gqa_shard", lambda: decode_obj("gqa_shard")),
                     ("ragged", lambda: decode_obj("ragged"))]
        for key, fn in secondary:
            try:
                result[key] = fn()
            except Exception as exc:  # the headline line is printed regardless
                result[key] = {"error": f"{type(exc).__name__}: {str(exc)[:200]}"}
    if not args.no_cpu_baseline and world == 1:
        result["cpu_baseline"] = cpu_baseline(di)
    print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_reference(args):
    """The CPU fp64 oracle, timed on every host core, on this workload's config
    and metric: each step is the whole workload (four sequences, every KV head,
    the full 131072-token context)."""
    rank, world, local = dist_env()
    if rank != 0:
        return
    import oracle
    from paged_kv_decode_31_b200 import inputs as I
    di = I.config_long_context(seed=1000, device="cpu")
    Hkv = di.Hkv
    host_cores = os.cpu_count() or 1
    oracle.set_num_threads(host_cores)
    sample_bytes = int(di.seqlens.sum()) * Hkv * di.D * 4

    def step():
        oracle.paged_attn(di.q, di.cache.k, di.cache.v, di.block_table, di.seqlens, di.scale,
                          False)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = sample_bytes * args.steps / dt / 1e9
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": 4, "seqlen_q": 1, "seqlen_k": 131072,
                   "Hq": 32, "Hkv": 8, "head_dim": 128, "block_size": 16,
                   "split_tokens": 4096, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                         "host_cores": host_cores, "kind": "oracle",
                         "sample": f"per step: all {di.batch} sequences, all {Hkv} KV heads, "
                                   f"full 131072-token context ({sample_bytes} KV bytes), "
                                   "i.e. the whole workload"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.backward_only:
        torch.cuda.set_device(0)
        print(json.dumps(backward_secondary(torch.device("cuda", 0), reps=max(args.steps, 1))))
        return
    if args.varlen_only:
        torch.cuda.set_device(0)
        print(json.dumps(varlen_secondary(torch.device("cuda", 0), reps=max(args.steps, 1))))
        return
    if args.prefill_only:
        torch.cuda.set_device(0)
        print(json.dumps(prefill_secondary(torch.device("cuda", 0), reps=max(args.steps, 1))))
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
