"""Benchmark of the exact-attention hot path on B200.

One step = one call of each of the four hot-path workloads, through the C
ABI on inputs already resident in HBM:
  - causal MHA prefill, B=4, Hq=Hkv=16, L=2048, d=128, bf16, O + LSE
    (``parts.prefill``; its TFLOP/s is the line's ``value``);
  - paged decode, 64 requests, Hq=32, Hkv=8, d=128, contexts
    U[1024, 32768] in 16-token pages, split-KV + LSE combine
    (``parts.decode``);
  - varlen GQA causal prefill, 8 sequences U[512, 8192], Hq=32, Hkv=8
    (``parts.varlen_gqa_prefill``);
  - long-context split-KV decode, 2 x 131072 tokens in 64-token pages
    (``parts.long_decode``).
Each call is timed with CUDA events on the stream it is launched on.  Before
every call a 256 MB buffer is written, so no call finds its inputs in L2
(the prefill inputs, 100 and 213 MB, are smaller than L2 or close to it; the
decode caches exceed it anyway), and then another 256 MB buffer is read, so
the dirty lines of that write are written back before the timed call starts
instead of during it.  Per-call times are averaged over the
--steps timed steps (after --warmup >= 3 untimed ones); the median and the
minimum are reported beside the mean.

Printed (rank 0, one JSON line): ``value`` = causal MHA prefill TFLOP/s
(causal pairs only, 4*d*Hq*L(L+1)/2 per sequence); every part carries its
own value and roofline; ``e2e`` repeats the step through the public API
with pinned host buffers and the host<->device copies inside the timed
region; ``cpu_baseline`` times the fp64 CPU oracle on a bounded sample of
each part.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload step|...]
    python bench.py --impl reference ...   # the CPU oracle as the reference arm

Multi-GPU: one process per GPU.  Under torch.distributed.run (WORLD_SIZE
set) each rank runs the same per-GPU workload (weak scaling, no data-path
collective: the parts are independent problems); the timed region is
bracketed by barriers and the max over ranks is reported.  Without a
WORLD_SIZE in the environment, --gpus N > 1 re-launches this script under
torch.distributed.run with N ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from exact_io_aware_86_b200 import api, inputs  # noqa: E402

METRIC = "prefill attn TFLOP/s (bf16) & paged-decode KV GB/s, % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, value: float, device=None) -> float:
    """Max of a float over all ranks (identity on one rank)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------
# workload accounting
# --------------------------------------------------------------------------
def visible_pairs(L: int, causal: bool, window=(-1, -1)) -> int:
    """(query, key) pairs of one sequence that the mask leaves visible: key j
    for query i when j <= i (causal) and i - left <= j <= i + right (window;
    negative = unlimited).  Only these count as work."""
    left, right = int(window[0]), int(window[1])
    if left < 0 and (right < 0 or causal):
        return L * (L + 1) // 2 if causal else L * L
    import numpy as np
    i = np.arange(L, dtype=np.int64)
    lo = np.maximum(0, i - left) if left >= 0 else np.zeros_like(i)
    r = 0 if causal else right
    hi = np.minimum(L - 1, i + r) if r >= 0 else np.full_like(i, L - 1)
    return int(np.maximum(0, hi - lo + 1).sum())


def prefill_flops(lengths, Hq, d, causal=True, window=(-1, -1)) -> float:
    pairs = sum(visible_pairs(L, causal, window) for L in lengths)
    return 4.0 * d * Hq * pairs


def variant_of(pin) -> dict:
    """Mask-variant arguments of a prefill workload (window, softcap, ALiBi)."""
    return dict(pin.meta.get("variant", {})) if pin is not None else {}


def is_fp8(pin) -> bool:
    return pin is not None and pin.q.dtype == torch.float8_e4m3fn


def is_append(inp) -> bool:
    return isinstance(inp, inputs.AppendInputs)


def decode_bytes(inp) -> float:
    """Algorithmic bytes of one decode call: K and V of every context token,
    q and o, the used block-table entries and seq_lens.  With an append, the
    context includes the new token, and the call also reads k_new, v_new and
    the two rotary table rows and writes the new key and value."""
    if is_append(inp):
        ctx = [int(x) + 1 for x in inp.cache_seqlens]
    else:
        ctx = [int(x) for x in inp.seq_lens]
    kv = sum(ctx) * inp.Hkv * inp.d * 2 * 2
    qo = 2 * inp.B * inp.Hq * inp.d * 2
    pages = sum((c + inp.page_size - 1) // inp.page_size for c in ctx)
    extra = 0
    if is_append(inp):
        extra = 2 * (2 * inp.B * inp.Hkv * inp.d * 2)          # k_new, v_new read; k, v written
        if inp.cos is not None:
            extra += inp.B * 2 * (inp.rotary_dim // 2) * 4      # one cos and one sin row each
    return float(kv + qo + 4 * pages + 4 * inp.B + extra)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kind: str) -> str:
    """Hash of the code a kernel is built from: its source files with line
    comments, trailing blanks and empty lines dropped, so an edit to the
    comments alone keeps the recorded counters."""
    files = {"prefill": ["prefill_sm100.cuh", "ptx.cuh"], "decode": ["decode_sm100.cuh", "ptx.cuh"]}[kind]
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "exact_io_aware_86_b200", "csrc", f)) as fh:
            for line in fh:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def dram_traffic(kind: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None if the
    kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(f"{kind}:{workload}")
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_hash") != kernel_source_hash(kind):
        return None
    return rec.get("bytes_per_launch")


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first(self, timeout: float = 10.0):
        """Blocks until the sampler has produced a line (nvidia-smi takes a
        moment to start), so the timed region is sampled from its start."""
        self.wait_samples(1, timeout)

    def wait_samples(self, n: int, timeout: float = 10.0):
        if self.proc is None:
            return
        base = len(self.lines) if n > 1 else 0
        t0 = time.time()
        while len(self.lines) < base + n and time.time() - t0 < timeout:
            time.sleep(0.02)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self._t is not None:
                self._t.join(timeout=2)
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# --------------------------------------------------------------------------
# the oracle on a bounded sample (CPU baseline and reference arm)
# --------------------------------------------------------------------------
def oracle_prefill_sample(pin, n_pairs: int):
    """Times the fp64 oracle on all rows of the first n_pairs (sequence, head)
    pairs.  Returns (flops, seconds)."""
    import numpy as np

    import oracle
    var = variant_of(pin)
    rt, rh, flops = [], [], 0.0
    pairs = [(b, h) for b in range(pin.B) for h in range(pin.Hq)][:n_pairs]
    for b, h in pairs:
        start, L = int(pin.cu_seqlens[b]), pin.lengths[b]
        rt.extend(range(start, start + L))
        rh.extend([h] * L)
        flops += prefill_flops([L], 1, pin.d, pin.causal, var.get("window", (-1, -1)))
    q, k, v = pin.q, pin.k, pin.v
    if q.dtype == torch.float8_e4m3fn:
        # the oracle's e4m3 path is decode-then-fp64; decode once, outside the timing
        qs, ks, vs = pin.meta["descale"]
        q, k, v = q.double() * qs, k.double() * ks, v.double() * vs
    t0 = time.perf_counter()
    oracle.prefill_rows(q, k, v, pin.cu_seqlens, pin.causal, pin.scale,
                        np.array(rt), np.array(rh), **var)
    return flops, time.perf_counter() - t0


def oracle_decode_sample(din, n_req: int):
    """Times the fp64 oracle on the first n_req requests (all heads).
    Returns (algorithmic bytes of those requests, seconds)."""
    import oracle
    if is_append(din):
        sub = inputs.AppendInputs(**{**din.__dict__, "q": din.q[:n_req], "k_new": din.k_new[:n_req],
                                     "v_new": din.v_new[:n_req],
                                     "block_table": din.block_table[:n_req],
                                     "cache_seqlens": din.cache_seqlens[:n_req]})
        t0 = time.perf_counter()
        oracle.decode_paged_append(sub.q, sub.k_new, sub.v_new, sub.k_pages, sub.v_pages,
                                   sub.block_table, sub.cache_seqlens, sub.scale, sub.cos, sub.sin,
                                   sub.rotary_dim or None, sub.interleaved)
        return decode_bytes(sub), time.perf_counter() - t0
    sub = inputs.DecodeInputs("sample", din.q[:n_req], din.k_pages, din.v_pages,
                              din.block_table[:n_req], din.seq_lens[:n_req], din.page_size,
                              din.scale)
    t0 = time.perf_counter()
    oracle.decode_paged(sub.q, sub.k_pages, sub.v_pages, sub.block_table, sub.seq_lens, sub.scale)
    return decode_bytes(sub), time.perf_counter() - t0


def oracle_sample(inp, n):
    """Times the oracle on n whole (sequence, head) pairs of a prefill or n
    whole requests of a decode.  Returns (algorithmic work of the sample:
    FLOPs or bytes, seconds)."""
    if isinstance(inp, inputs.PrefillInputs):
        return oracle_prefill_sample(inp, n)
    return oracle_decode_sample(inp, n)


def cpu_baseline(parts, budget_s: float = 20.0):
    """The fp64 oracle on a bounded sample of every part of the step (about
    budget_s seconds in all): whole (sequence, head) pairs of a prefill, whole
    requests of a decode.  Each part's rate is sample work / sample time;
    `full_s` is the time the oracle would take on the whole call at that
    rate (rows and requests are independent, so the rate carries over)."""
    import oracle
    cores = oracle.num_threads()
    share = budget_s / max(len(parts), 1)
    out = {"kind": "oracle", "cores": cores}
    per = {}
    for p in parts:
        inp = p.pin if p.is_prefill else p.din
        total = inp.B * inp.Hq if p.is_prefill else inp.B
        w, sec = oracle_sample(inp, 1)
        n = max(1, min(total, int(share / max(sec, 1e-3))))
        if n > 1:
            w, sec = oracle_sample(inp, n)
        rate = w / sec / (1e12 if p.is_prefill else 1e9)
        what = (f"all rows of {n} of {total} (sequence, head) pairs" if p.is_prefill
                else f"{n} of {total} requests (all heads)")
        per[p.key] = {"value": rate, "unit": p.unit, "sample": f"{what} of {inp.name}",
                      "full_s": round(p.work / (w / sec), 2)}
    first = per[parts[0].key]
    out.update(value=first["value"], unit=first["unit"], sample=first["sample"], parts=per)
    return out


# --------------------------------------------------------------------------
# GPU measurement
# --------------------------------------------------------------------------
# The default step, in launch order: (workload, key of its entry in "parts")
STEP = [("mha_prefill", "prefill"), ("paged_decode", "decode"),
        ("varlen_gqa_prefill", "varlen_gqa_prefill"), ("long_decode", "long_decode")]

WORKLOAD_NAMES = {
    "step": "causal MHA prefill B=4 Hq=Hkv=16 L=2048 d=128 + paged decode 64 req Hq=32 Hkv=8 "
            "d=128 ctx U[1024,32768] page 16 + varlen GQA causal prefill 8 seqs U[512,8192] "
            "Hq=32 Hkv=8 + split-KV decode 2 x 131072 page 64",
    "mha_prefill": inputs.WORKLOADS["mha_prefill"],
    "varlen_gqa_prefill": inputs.WORKLOADS["varlen_gqa_prefill"],
    "paged_decode": inputs.WORKLOADS["paged_decode"],
    "long_decode": inputs.WORKLOADS["long_decode"],
    "window_prefill": inputs.WORKLOADS["window_prefill"],
    "softcap_prefill": inputs.WORKLOADS["softcap_prefill"],
    "alibi_prefill": inputs.WORKLOADS["alibi_prefill"],
    "append_decode": inputs.WORKLOADS["append_decode"],
    "fp8_prefill": inputs.WORKLOADS["fp8_prefill"],
}

PREFILL_WORKLOADS = ("mha_prefill", "varlen_gqa_prefill", "window_prefill", "softcap_prefill",
                     "alibi_prefill", "fp8_prefill")


def step_parts(name):
    """(workload, part key) of each call of a step of `name`."""
    if name == "step":
        return list(STEP)
    return [(name, "prefill" if name in PREFILL_WORKLOADS else "decode")]


def make_inputs(name):
    return getattr(inputs, name)()


def decode_launches(din, splits: int) -> int:
    """Kernels one decode call launches: the split kernel, then the LSE
    combine when a request can have more than one range, the one-CTA plan
    kernel before them when the batch is too large for the in-kernel plan,
    and the append + RoPE kernel first for a decode with append."""
    n = 1
    if splits > 1:
        n += 1 + (1 if din.B > api.DECODE_PLAN_MAX_B else 0)
    return n + (1 if is_append(din) else 0)


class Part:
    """One call of the step: its inputs resident on the device, its outputs
    and scratch, and its algorithmic work."""

    def __init__(self, workload, key, dev):
        self.workload, self.key = workload, key
        inp = make_inputs(workload)
        self.is_prefill = isinstance(inp, inputs.PrefillInputs)
        if self.is_prefill:
            self.pin, self.din = inp, None
            self.q, self.k, self.v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
            self.cu = inp.cu_seqlens.to(dev)
            self.o = torch.empty(self.q.shape, dtype=torch.bfloat16, device=dev)
            self.lse = torch.empty(inp.Hq, inp.T, dtype=torch.float32, device=dev)
            self.max_len = max(inp.lengths)
            self.variant = variant_of(inp)
            if self.variant.get("alibi_slopes") is not None:
                self.variant["alibi_slopes"] = self.variant["alibi_slopes"].to(dev)
            self.work = prefill_flops(inp.lengths, inp.Hq, inp.d, inp.causal,
                                      self.variant.get("window", (-1, -1)))
            self.unit = "TFLOP/s"
            self.launches = 1
        else:
            self.pin, self.din = None, inp
            din = inp
            self.dq, self.kp, self.vp = (t.to(dev) for t in (din.q, din.k_pages, din.v_pages))
            self.bt = din.block_table.to(dev)
            self.sl = (din.cache_seqlens if is_append(din) else din.seq_lens).to(dev)
            # automatic page ranges (num_splits = 0); splits = the most ranges a
            # request can get, which sizes the workspace
            self.splits = api.decode_auto_splits(din.B, din.Hq, din.Hkv,
                                                 din.block_table.shape[1], din.page_size)
            if is_append(din):
                self.kn, self.vn = din.k_new.to(dev), din.v_new.to(dev)
                self.cos = din.cos.to(dev) if din.cos is not None else None
                self.sin = din.sin.to(dev) if din.sin is not None else None
                nbytes = api.decode_append_workspace_size(din.B, din.Hq, din.d, self.splits)
            else:
                nbytes = api.decode_workspace_size(din.B, din.Hq, din.d, self.splits)
            self.ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev) if nbytes else None
            self.do = torch.empty_like(self.dq)
            self.dlse = torch.empty(din.B, din.Hq, dtype=torch.float32, device=dev)
            self.work = decode_bytes(din)
            self.unit = "GB/s"
            self.launches = decode_launches(din, self.splits)

    @property
    def name(self):
        return (self.pin or self.din).name

    def call(self):
        if self.is_prefill:
            pin = self.pin
            if pin.q.dtype == torch.float8_e4m3fn:
                qs, ks, vs = pin.meta["descale"]
                api.fa_prefill_fp8(self.q, self.k, self.v, self.o, self.lse, self.cu, pin.causal,
                                   pin.scale, qs, ks, vs, self.max_len)
                return
            api.fa_prefill(self.q, self.k, self.v, self.o, self.lse, self.cu, pin.causal,
                           pin.scale, self.max_len, **self.variant)
            return
        din = self.din
        if is_append(din):
            # the same slot is rewritten with the same values every call
            api.fa_decode_paged_append(self.dq, self.kn, self.vn, self.kp, self.vp, self.bt,
                                       self.sl, 0, self.do, self.dlse, din.scale, self.cos,
                                       self.sin, din.rotary_dim or None, din.interleaved, self.ws)
            return
        api.fa_decode_paged(self.dq, self.kp, self.vp, self.bt, self.sl, 0, self.do, self.dlse,
                            din.scale, self.ws)

    def host_io(self):
        """(device tensor, pinned host copy) pairs of the inputs the call
        reads, and of the outputs it writes."""
        if self.is_prefill:
            pin = self.pin
            ins = [(self.q, pin.q), (self.k, pin.k), (self.v, pin.v), (self.cu, pin.cu_seqlens)]
            outs = [self.o, self.lse]
        else:
            din = self.din
            ins = [(self.dq, din.q), (self.kp, din.k_pages), (self.vp, din.v_pages),
                   (self.bt, din.block_table),
                   (self.sl, din.cache_seqlens if is_append(din) else din.seq_lens)]
            if is_append(din):
                ins += [(self.kn, din.k_new), (self.vn, din.v_new)]
                if din.cos is not None:
                    ins += [(self.cos, din.cos), (self.sin, din.sin)]
            outs = [self.do, self.dlse]
        return ([(d, h.pin_memory()) for d, h in ins],
                [(d, torch.empty(d.shape, dtype=d.dtype, pin_memory=True)) for d in outs])

    def rate(self, ms):
        """Throughput of one call that took `ms` milliseconds, in self.unit."""
        return self.work / (ms * 1e-3) / (1e12 if self.is_prefill else 1e9)


class L2Flush:
    """Writes a buffer larger than L2 (evicting every input), then reads a
    second one (writing the dirty lines of the first back to memory), so
    the next call starts with a cold and clean L2."""

    def __init__(self, dev, nbytes: int = L2_FLUSH_BYTES):
        self.w = torch.empty(nbytes // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(nbytes // 4, dtype=torch.float32, device=dev)
        self.acc = torch.zeros((), dtype=torch.float32, device=dev)

    def __call__(self, value: float):
        self.w.fill_(value)
        torch.sum(self.r, dim=0, out=self.acc)


def time_device(parts, steps: int, warmup: int, dist, gpu_index: int):
    """Per-part CUDA-event times (ms lists) over `steps` timed steps, the
    whole timed region (ms) and the clocks sampled during it."""
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = L2Flush(dev)
    for _ in range(warmup):
        for p in parts:
            flush(1.0)
            p.call()
    torch.cuda.synchronize()
    if api.device_error() != api.FA_OK:
        raise RuntimeError("device error during warm-up")
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in parts] for _ in range(steps)]
    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier(dist)
    torch.cuda.synchronize()
    with ClockSampler(gpu_index) as clocks:
        clocks.wait_first()
        outer[0].record()
        for i in range(steps):
            for j, p in enumerate(parts):
                flush(float(i))
                ev[i][j][0].record()
                p.call()
                ev[i][j][1].record()
        outer[1].record()
        torch.cuda.synchronize()
        # keep sampling a little so short regions still get samples
        clocks.wait_samples(3)
    barrier(dist)
    times = [[ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(steps)]
             for j in range(len(parts))]
    region = outer[0].elapsed_time(outer[1])
    if api.device_error() != api.FA_OK:
        raise RuntimeError("device error during the timed loop")
    return times, region, clocks.summary()


def time_e2e(parts, steps: int):
    """The step through the public API with pinned host buffers: per call,
    H2D of its inputs, the call, D2H of its results, all inside the timed
    region.  Returns (per-part ms lists, h2d bytes per step, d2h bytes per
    step)."""
    io = [p.host_io() for p in parts]
    h2d = sum(h.numel() * h.element_size() for ins, _ in io for _, h in ins)
    d2h = sum(h.numel() * h.element_size() for _, outs in io for _, h in outs)
    times = [[] for _ in parts]
    for i in range(steps + 1):  # the first iteration is a warm-up
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in parts]
        for j, p in enumerate(parts):
            ins, outs = io[j]
            ev[j][0].record()
            for d, h in ins:
                d.copy_(h, non_blocking=True)
            p.call()
            for d, h in outs:
                h.copy_(d, non_blocking=True)
            ev[j][1].record()
        torch.cuda.synchronize()
        if i > 0:
            for j in range(len(parts)):
                times[j].append(ev[j][0].elapsed_time(ev[j][1]))
    return times, h2d, d2h


def roofline(is_prefill, achieved, peak, unit, traffic):
    return {"bound": "tensor" if is_prefill else "hbm", "achieved": round(achieved, 2),
            "peak": peak, "unit": unit, "frac": round(achieved / peak, 4), "traffic": traffic}


def run_gpu(args, world, rank, local):
    torch.cuda.set_device(local)
    dist = init_dist(world, "nccl")
    threads = max(1, (os.cpu_count() or 8) // max(world, 1))
    torch.set_num_threads(threads)
    dev = torch.device("cuda", local)
    parts = [Part(w, k, dev) for w, k in step_parts(args.workload)]
    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(parts, budget_s=args.cpu_budget)
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES", "").replace(",", "").isdigit() else local
    times, region, clocks = time_device(parts, args.steps, args.warmup, dist, gpu_index)
    e2e_steps = max(2, min(args.steps, args.e2e_steps))
    etimes, h2d, d2h = time_e2e(parts, e2e_steps)

    peaks, peak_src = load_peaks()
    ms = [max_over_ranks(dist, statistics.mean(t), "cuda") for t in times]
    ems = [max_over_ranks(dist, statistics.mean(t), "cuda") for t in etimes]
    reg_ms = max_over_ranks(dist, region, "cuda")
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    out_parts = {}
    for p, t, m in zip(parts, times, ms):
        rate = world * p.rate(m)
        if p.is_prefill:
            # an e4m3 contraction takes the fp8 peak: the measured bf16 peak times
            # the nominal fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s dense)
            peak = peaks["bf16_tflops"] * (2.0 if is_fp8(p.pin) else 1.0)
            entry = {"workload": p.name, "value": round(rate, 2), "unit": p.unit,
                     "ms": round(m, 4), "ms_median": round(statistics.median(t), 4),
                     "ms_min": round(min(t), 4), "flops": p.work,
                     "roofline": roofline(True, rate / world, peak, "TFLOP/s",
                                          dram_traffic("prefill", p.name)),
                     "launches_per_call": p.launches}
        else:
            entry = {"workload": p.name, "value": round(rate, 1), "unit": p.unit,
                     "ms": round(m, 4), "ms_median": round(statistics.median(t), 4),
                     "ms_min": round(min(t), 4), "bytes": p.work,
                     "max_ranges_per_request": p.splits,
                     "workspace_bytes": api.decode_workspace_size(p.din.B, p.din.Hq, p.din.d,
                                                                  p.splits),
                     "roofline": roofline(False, rate / world, peaks["hbm_gbs"], "GB/s",
                                          dram_traffic("decode", p.name)),
                     "launches_per_call": p.launches}
        out_parts[p.key] = entry
    head_part = parts[0]
    head = out_parts[head_part.key]
    dom = max(range(len(parts)), key=lambda j: ms[j])
    e2e = {"value": round(world * head_part.rate(ems[0]), 3), "unit": head_part.unit,
           "ms": round(ems[0], 3), "workload": head_part.name,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "parts": {p.key: {"value": round(world * p.rate(m), 3), "unit": p.unit,
                             "ms": round(m, 3)} for p, m in zip(parts, ems)}}
    fp8 = any(p.is_prefill and is_fp8(p.pin) for p in parts)
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": head["unit"],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(sum(ms), 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3" if fp8 else "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_NAMES[args.workload],
                   "l2": "before every timed call: 256 MB written, then another 256 MB read "
                         "(cold, clean L2)",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "parts": out_parts,
        "roofline": dict(out_parts[parts[dom].key]["roofline"], kernel=parts[dom].name),
        "peaks_source": peak_src,
        "region_ms": round(reg_ms, 3),
        "e2e": e2e,
        "gpu_launches": sum(p.launches for p in parts) * args.steps,
        "clocks": clocks,
    }
    if base is not None:
        line["cpu_baseline"] = base
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle, timed on the host cores on a
    bounded sample of each call of the same step; same metric, unit and
    config.  Under torchrun only rank 0 works."""
    if rank != 0:
        return
    import oracle
    workloads = step_parts(args.workload)
    ins = [(make_inputs(w), k) for w, k in workloads]
    pairs, reqs = 1, 2
    if args.warmup > 0:  # one warm-up pass is enough for a CPU code path
        for inp, _ in ins:
            oracle_sample(inp, pairs if isinstance(inp, inputs.PrefillInputs) else reqs)
    acc = {k: [0.0, 0.0] for _, k in ins}
    for _ in range(args.steps):
        for inp, k in ins:
            n = pairs if isinstance(inp, inputs.PrefillInputs) else reqs
            w, sec = oracle_sample(inp, n)
            acc[k][0] += w
            acc[k][1] += sec
    parts, sample = {}, []
    for inp, k in ins:
        pre = isinstance(inp, inputs.PrefillInputs)
        w, sec = acc[k]
        parts[k] = {"workload": inp.name, "value": w / sec / (1e12 if pre else 1e9),
                    "unit": "TFLOP/s" if pre else "GB/s", "ms": 1e3 * sec / args.steps}
        sample.append(f"{inp.name}: all rows of {pairs} of {inp.B * inp.Hq} (sequence, head) pairs"
                      if pre else f"{inp.name}: {reqs} of {inp.B} requests, all heads")
    head = parts[ins[0][1]]
    line = {
        "metric": METRIC, "value": head["value"], "unit": head["unit"], "impl": "reference",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sum(p["ms"] for p in parts.values()), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAMES[args.workload],
                   "l2": "n/a (CPU)", "parallelism": "host cores"},
        "parts": parts,
        "cpu_baseline": {"kind": "oracle", "cores": oracle.num_threads(), "value": head["value"],
                         "unit": head["unit"], "sample": "; ".join(sample)},
        "e2e": {"value": head["value"], "unit": head["unit"], "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def relaunch(args, argv):
    """--gpus N > 1 outside torch.distributed.run: start N ranks of this
    script under it (127.0.0.1 rendezvous) and return their exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           f"--master-port={port}", os.path.abspath(__file__), *argv]
    return subprocess.run(cmd).returncode


def run_plumbing(args, world, rank):
    """--plumbing: the rank and timing plumbing alone on the CPU (gloo), no
    kernels -- one "step" is a barrier.  Prints the JSON line's rank fields
    so a CPU test can check a --gpus N launch end to end."""
    dist = init_dist(world, "gloo")
    t0 = time.perf_counter()
    for _ in range(args.steps):
        barrier(dist)
    ms = max_over_ranks(dist, 1e3 * (time.perf_counter() - t0) / max(args.steps, 1), "cpu")
    if rank == 0:
        print(json.dumps({"plumbing": True, "n_gpus": world, "steps": args.steps,
                          "warmup": args.warmup, "ms_per_step": ms}), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_NAMES), default="step")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-budget", type=float, default=20.0,
                    help="seconds of oracle work for the CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--plumbing", action="store_true",
                    help="rank and timing plumbing only, on the CPU (gloo), no kernels")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(relaunch(args, argv))
    world, rank, local = dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.plumbing:
        run_plumbing(args, world, rank)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_gpu(args, world, rank, local)


if __name__ == "__main__":
    main()
