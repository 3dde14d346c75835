"""Benchmark of the GQA forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one gqa_forward call over the decode workload of a Mistral-7B-shaped
layer (B=16, Hq=32, Hkv=8, Sq=1, Sk=4096 KV cache, D=128, bf16, q/k/v i.i.d.
N(0,1) from the seeded generator, no mask, scale 1/sqrt(128)).  The metric is
decode KV-read GB/s: the algorithmic bytes of q, k, v and out per call
(268,697,600 B) over the device time.  Inputs are resident in HBM before the
timed region; the timed launches rotate over enough copies of K/V that no
launch finds its K/V in the 126 MB L2.

Extra measurements on the same line (N=1 only): the long-context decode of a
Llama-2-70B-shaped layer (GB/s), the causal prefill (TFLOP/s) and the padded
masked prefill (TFLOP/s), each with its roofline fraction.

N > 1 (one process per GPU under torchrun): every rank runs its own copy of the
workload (weak scaling, no data-path collective); the timed region is bracketed
by a barrier and a device synchronise, and the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the correctness reference, not a
tuned baseline) on bounded samples of the same workload on rank 0.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402  (seeded inputs; no attention arithmetic)

DECODE = dict(name="decode_mistral7b_layer", B=16, Hq=32, Hkv=8, Sq=1, Sk=4096, D=128,
              causal=False, mask=False, seed=2)
DECODE_LONG = dict(name="decode_llama2_70b_layer", B=16, Hq=64, Hkv=8, Sq=1, Sk=32768, D=128,
                   causal=False, mask=False, seed=3)
PREFILL_CAUSAL = dict(name="prefill_causal", B=4, Hq=32, Hkv=8, Sq=4096, Sk=4096, D=128,
                      causal=True, mask=False, seed=4)
PREFILL_MASKED = dict(name="prefill_padded_mask", B=8, Hq=12, Hkv=2, Sq=2048, Sk=2048, D=64,
                      causal=False, mask=True, seed=5)
# Ragged KV cache: 4096-key capacity, entry b holds len_b ~ U[256, 4096] keys.
DECODE_RAGGED = dict(name="decode_ragged_cache", B=16, Hq=32, Hkv=8, Sq=1, Sk=4096, D=128,
                     causal=False, mask=False, seed=6, lens=(256, 4096), append=0)
# One generation step: append one token per sequence, then attend over the
# grown cache (bottom-right causal); capacity leaves room for the appends.
DECODE_STEP = dict(name="decode_step_append", B=16, Hq=32, Hkv=8, Sq=1, Sk=4096 + 512, D=128,
                   causal=True, mask=False, seed=7, lens=(256, 4096), append=1)
# The ragged cache held in 64-key pages of a shuffled pool (block table per sequence).
DECODE_PAGED = dict(name="decode_paged_cache", B=16, Hq=32, Hkv=8, Sq=1, Sk=4096, D=128,
                    causal=False, mask=False, seed=6, lens=(256, 4096), append=0, page=64)
# Chunked prefill on a paged cache: 1024 new queries at the end of each
# sequence (bottom-right causal) over lengths U[2048, 8192] in 64-key pages.
PREFILL_CHUNK_PAGED = dict(name="prefill_chunk_paged_cache", B=4, Hq=32, Hkv=8, Sq=1024, Sk=8192,
                           D=128, causal=True, mask=False, seed=10, lens=(2048, 8192), append=0,
                           page=64)
# The Mistral-7B-shaped decode with fp16 operands, and with head dim 96.
DECODE_F16 = dict(DECODE, name="decode_mistral7b_layer_fp16", dtype="f16", seed=8)
DECODE_D96 = dict(DECODE, name="decode_head_dim_96", D=96, seed=9)

L2_BYTES = 126 * 1024 * 1024


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return (float(pk["hbm_gbs"]), float(pk["bf16_tflops"]),
                float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])), "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


TRAFFIC_SOURCES = ("kernels.h", "ptx.cuh", "epilogue.cuh")
# Headers a prefill kernel also includes.
PREFILL_SOURCES = ("prefill_common.cuh",)


def kernel_source_sha256(kernel_file: str) -> str:
    """Hash of a kernel's source and the headers it includes."""
    h = hashlib.sha256()
    extra = PREFILL_SOURCES if kernel_file.startswith("prefill") else ()
    for name in (kernel_file,) + TRAFFIC_SOURCES + extra:
        with open(os.path.join(ROOT, "grouped_query_attention_fwd_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _traffic_for(kernel_file: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel
    source is unchanged since it was captured; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        ent = rec[workload]
        if ent.get("source_sha256") != kernel_source_sha256(kernel_file):
            return None
        return float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.rows = []
        self.proc = None
        self.gpu_id = gpu_id

    def start(self):
        cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
               "-lms", "50"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self, t0=None, t1=None):
        rows = [r for (t, r) in self.rows if (t0 is None or t >= t0) and (t1 is None or t <= t1)]
        if not rows:
            rows = [r for (_, r) in self.rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = [n for i, n in enumerate(names)
                   if any(len(r) > 4 + i and r[4 + i].lower().startswith("active") for r in rows)]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------ inputs

def _host_inputs(cfg, torch, pin=False):
    """Seeded q, k, v (bf16, or fp16 when cfg["dtype"] says so) and mask as
    host tensors."""
    B, Hq, Hkv, Sq, Sk, D = (cfg[x] for x in ("B", "Hq", "Hkv", "Sq", "Sk", "D"))
    seed = cfg["seed"]
    f16 = cfg.get("dtype") == "f16"

    def gen(stream, shape):
        if f16:
            n = 1
            for x in shape:
                n *= x
            t = torch.from_numpy(synth.normal_f32(seed, stream, n).reshape(shape)).half()
            return t.pin_memory() if pin else t
        t = torch.empty(shape, dtype=torch.bfloat16, pin_memory=pin)
        synth.normal_bf16_into(seed, stream, t.data_ptr(), t.numel())
        return t

    q = gen(synth.STREAM_Q, (B, Hq, Sq, D))
    k = gen(synth.STREAM_K, (B, Hkv, Sk, D))
    v = gen(synth.STREAM_V, (B, Hkv, Sk, D))
    mask = None
    if cfg["mask"]:
        lens = synth.uniform_int(seed, synth.STREAM_MASK, B, 256, Sk)
        mask = torch.from_numpy(synth.mask_from_lengths(lens, Sq, Sk))
        if pin:
            mask = mask.pin_memory()
    return q, k, v, mask


def _visible_pairs(cfg, mask_host):
    if mask_host is not None:
        return float(mask_host.sum().item()) * cfg["Hq"]
    if cfg["causal"]:
        S = cfg["Sq"]
        return cfg["B"] * cfg["Hq"] * S * (S + 1) / 2.0
    return float(cfg["B"] * cfg["Hq"] * cfg["Sq"] * cfg["Sk"])


# ------------------------------------------------------------- multi-rank

def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest `value` over all ranks (the job is as slow as its slowest
    rank); `dist` is torch.distributed or None for a single process."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_gbs(bytes_per_step: int, steps: int, world: int, elapsed_ms: float) -> float:
    """Whole-job GB/s when every rank runs its own copy of the workload."""
    return bytes_per_step * steps * world / (elapsed_ms / 1e3) / 1e9


# ------------------------------------------------------------------ GPU arm

def _graph_timed(torch, calls, steps, warmup, stream, repeats=1, per_launch_samples=100,
                 before_each=None):
    """Time exactly `steps` launches, launch i being calls[i % len(calls)],
    `repeats` times over.

    The launches are captured into CUDA graphs (one graph of up to ~64
    launches, a whole number of rounds over the calls, replayed, plus one for
    the remainder), so the host never paces the GPU.  Each repetition of the
    `steps` launches is bracketed by a device synchronise (after
    `before_each()`, e.g. a barrier over ranks) and two events on `stream`.
    A separate pass replays one-launch graphs with an event pair around each.
    Returns (ms of each repetition, per-launch ms list, host seconds per
    launch spent enqueuing a repetition)."""
    for i in range(warmup):
        calls[i % len(calls)]()
    torch.cuda.synchronize()
    n = len(calls)
    chunk = n * max(1, min(64, steps) // n) if steps >= n else steps

    def capture(count, start):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for j in range(count):
                calls[(start + j) % n]()
        return g

    chain = capture(chunk, 0)
    tail = capture(steps % chunk, 0) if steps % chunk else None
    singles = [capture(1, i) for i in range(n)]
    chain.replay()
    if tail is not None:
        tail.replay()
    for g in singles:
        g.replay()
    torch.cuda.synchronize()

    times, host = [], []
    for _ in range(repeats):
        if before_each is not None:
            before_each()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0 = time.perf_counter()
        e0.record(stream)
        for _ in range(steps // chunk):
            chain.replay()
        if tail is not None:
            tail.replay()
        e1.record(stream)
        host.append(time.perf_counter() - h0)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))

    k = min(steps, per_launch_samples)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(k)]
    for i in range(k):
        ev[i][0].record(stream)
        singles[i % n].replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) for a, b in ev]
    del chain, tail, singles
    return times, per, statistics.median(host) / steps


def timing_repeats(steps: int) -> int:
    """Repetitions of the `steps`-launch timed region: about 2000 launches in
    all, at least 3 and at most 50 repetitions."""
    return max(3, min(50, -(-2000 // max(1, steps))))


def _time_config(gqa, torch, cfg, steps, warmup, dev, rotate_to_bytes=3 * L2_BYTES):
    """Device-resident timing of one workload.  Returns a dict of numbers."""
    q, k, v, mask = _host_inputs(cfg, torch)
    qd = q.to(dev)
    kv_bytes = 2 * k.numel() * 2
    copies = max(1, math.ceil(rotate_to_bytes / kv_bytes)) if kv_bytes < rotate_to_bytes else 1
    ks = [k.to(dev) for _ in range(copies)]
    vs = [v.to(dev) for _ in range(copies)]
    md = mask.to(dev) if mask is not None else None
    out = torch.empty(qd.shape, dtype=qd.dtype, device=dev)
    plan = gqa.query(qd, ks[0], vs[0], mask=md, causal=cfg["causal"])
    ws = gqa.workspace_for(dev, plan["workspace_bytes"])
    stream = torch.cuda.current_stream(dev)
    calls = [(lambda i=i: gqa.forward(qd, ks[i], vs[i], mask=md, causal=cfg["causal"], out=out,
                                      workspace=ws)) for i in range(copies)]
    times, per, _ = _graph_timed(torch, calls, steps, warmup, stream, repeats=5)
    total_ms = statistics.median(times)
    st = gqa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status after timing: %s" % gqa.status_string(st))
    res = dict(total_ms=total_ms, per_launch_ms=total_ms / steps,
               single_launch_median_ms=statistics.median(per), plan=plan, copies=copies,
               visible_pairs=_visible_pairs(cfg, mask))
    del ks, vs, qd, md, out
    torch.cuda.empty_cache()
    return res


def visible_pairs(Sq, lens, causal):
    """(query, key) pairs a query head sees over entries with cache lengths
    `lens`: every key, or, bottom-right causal, query i of the block of Sq
    sees keys j <= i + len - Sq (and j >= 0)."""
    total = 0
    for n in lens:
        n = int(n)
        if not causal:
            total += Sq * n
            continue
        # min(max(i + n - Sq + 1, 0), n) summed over i = 0 .. Sq - 1
        lo = max(0, Sq - n)  # first query that sees a key
        total += sum(min(i + n - Sq + 1, n) for i in range(lo, Sq))
    return total


def _time_ragged(gqa, torch, cfg, steps, warmup, dev, rotate_to_bytes=3 * L2_BYTES):
    """Device-resident timing of a ragged-cache workload: per step an optional
    gqa_kv_append of one token per sequence, then gqa_forward with kv_lens."""
    import numpy as np
    B, Hkv, Sk, D = cfg["B"], cfg["Hkv"], cfg["Sk"], cfg["D"]
    q, k, v, _ = _host_inputs(cfg, torch)
    lo, hi = cfg["lens"]
    lens0 = synth.uniform_int(cfg["seed"], synth.STREAM_MASK, B, lo, hi).astype(np.int32)
    valid_bytes = int(lens0.sum()) * Hkv * D * 2 * 2
    copies = max(3, math.ceil(rotate_to_bytes / valid_bytes))
    qd = q.to(dev)
    ks = [k.to(dev) for _ in range(copies)]
    vs = [v.to(dev) for _ in range(copies)]
    lens = [torch.from_numpy(lens0.copy()).to(dev) for _ in range(copies)]
    n_new = cfg["append"]
    kn = vn = None
    if n_new:
        kn = ks[0][:, :, :n_new].clone()
        vn = vs[0][:, :, :n_new].clone()
    tables = [None] * copies
    ps = cfg.get("page")
    if ps:
        # Every (sequence, page) of the cache goes to a random slot of a pool.
        per_seq = Sk // ps
        gen = torch.Generator().manual_seed(cfg["seed"])
        for i in range(copies):
            perm = torch.randperm(B * per_seq, generator=gen)
            inv = torch.empty_like(perm)
            inv[perm] = torch.arange(B * per_seq)
            def pool(x):
                return x.view(B, Hkv, per_seq, ps, D).permute(0, 2, 1, 3, 4).reshape(
                    B * per_seq, Hkv, ps, D)[perm.to(dev)].contiguous()
            ks[i], vs[i] = pool(ks[i]), pool(vs[i])
            tables[i] = inv.view(B, per_seq).to(torch.int32).to(dev)
    out = torch.empty(qd.shape, dtype=qd.dtype, device=dev)
    off = "bottom_right" if cfg["causal"] else None
    plan = gqa.query(qd, ks[0], vs[0], causal=cfg["causal"], causal_offset=off, kv_lens=lens[0],
                     block_table=tables[0])
    ws = gqa.workspace_for(dev, plan["workspace_bytes"])
    stream = torch.cuda.current_stream(dev)

    def call(i):
        if n_new:
            gqa.kv_append(ks[i], vs[i], kn, vn, lens[i], workspace=ws)
        gqa.forward(qd, ks[i], vs[i], out=out, workspace=ws, causal=cfg["causal"],
                    causal_offset=off, kv_lens=lens[i], block_table=tables[i])

    calls = [(lambda i=i: call(i)) for i in range(copies)]
    if n_new:  # every call of a copy appends n_new tokens: they must fit the capacity
        chunk = copies * max(1, min(64, steps) // copies)  # warm replay of the graphs
        executed = warmup + chunk + steps % chunk + copies + 5 * steps + min(steps, 100)
        calls_per_copy = math.ceil(executed / copies)
        if hi + calls_per_copy * n_new > Sk:
            raise ValueError("%d steps overflow the %d-key cache; use fewer" % (steps, Sk))
    times, per, _ = _graph_timed(torch, calls, steps, warmup, stream, repeats=5)
    total_ms = statistics.median(times)
    st = gqa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status after timing: %s" % gqa.status_string(st))
    # Keys read per step: the lengths grow by n_new per call of a copy, so the
    # mean of each copy's first and last lengths is the mean over its calls.
    final = [int(x.sum().item()) for x in lens]
    mean_keys = statistics.mean((int(lens0.sum()) + f) / 2.0 for f in final)
    if n_new:
        mean_keys += n_new * B  # the appended token is read too
    step_bytes = (mean_keys * Hkv * D * 2 * 2 + 2 * qd.numel() * 2 +
                  (4 * B * Hkv * n_new * D * 2 if n_new else 0))
    pairs = None if n_new else visible_pairs(cfg["Sq"], lens0, cfg["causal"])
    res = dict(total_ms=total_ms, per_launch_ms=total_ms / steps,
               single_launch_median_ms=statistics.median(per), plan=plan, copies=copies,
               step_bytes=step_bytes, launches=plan["launches"] + (1 if n_new else 0),
               mean_len=mean_keys / B, visible_pairs_per_head=pairs)
    del ks, vs, qd, out, lens
    torch.cuda.empty_cache()
    return res


def _e2e(gqa, torch, cfg, steps, dev):
    """Through the public call with host buffers: pinned host -> device copy
    of the step's inputs, the forward, and a device -> host read of out."""
    q, k, v, mask = _host_inputs(cfg, torch, pin=True)
    qd, kd, vd = (torch.empty_like(x, device=dev) for x in (q, k, v))
    md = torch.empty_like(mask, device=dev) if mask is not None else None
    out_h = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    out_d = torch.empty(q.shape, dtype=q.dtype, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        qd.copy_(q, non_blocking=True)
        kd.copy_(k, non_blocking=True)
        vd.copy_(v, non_blocking=True)
        if md is not None:
            md.copy_(mask, non_blocking=True)
        gqa.forward(qd, kd, vd, mask=md, causal=cfg["causal"], out=out_d)
        out_h.copy_(out_d, non_blocking=True)

    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    h2d = q.numel() * 2 + k.numel() * 2 + v.numel() * 2 + (mask.numel() if mask is not None else 0)
    return ms, h2d, out_h.numel() * 2


def _time_oracle(fn, budget_s, max_calls=100000):
    """Call fn() until about budget_s of wall time; returns (calls, seconds)."""
    calls, used = 0, 0.0
    while used < budget_s and calls < max_calls:
        t0 = time.perf_counter()
        fn(calls)
        used += time.perf_counter() - t0
        calls += 1
    return calls, used


def _cpu_baseline(budget_s=16.0):
    """The fp64 oracle as it stands (single-threaded C++, unchanged), timed on
    bounded samples of all five workloads, about budget_s of CPU time in all.
    The headline value is the Mistral-7B-shaped decode's; `per_config` holds
    every workload's rate in its own unit with the sample it was taken on."""
    import oracle
    per = {}

    # Page-1 toy, fp32: the whole problem, repeatedly.
    q, k, v = synth.qkv_f32(1, 1, 4, 2, 5, 5, 4)
    n, t = _time_oracle(lambda i: oracle.forward(q, k, v, scale=0.5), 0.05 * budget_s, 20000)
    per["page1_toy_f32"] = {"value": round(t / n * 1e6, 2), "unit": "us per forward",
                            "sample": "the whole (1,4,5,4) problem, %d calls" % n}

    def decode_groups(cfg, share, distinct):
        B, Hq, Hkv, Sk, D = (cfg[x] for x in ("B", "Hq", "Hkv", "Sk", "D"))
        g = Hq // Hkv
        qb = synth.normal_bf16_bits(cfg["seed"], synth.STREAM_Q, B * Hq * D).reshape(B, Hq, 1, D)
        # Cycle over the first `distinct` groups (generating their inputs is
        # not timed, and takes longer than the oracle on the long cache).
        order = [(b, kv) for b in range(B) for kv in range(Hkv)][:distinct]
        cache = {}

        def one(i):
            b, kv = order[i % len(order)]
            if (b, kv) not in cache:
                ks = synth.bf16_bits_to_f64(synth.kv_slice_bf16_bits(
                    cfg["seed"], synth.STREAM_K, B, Hkv, Sk, D, b, kv))[None, None]
                vs = synth.bf16_bits_to_f64(synth.kv_slice_bf16_bits(
                    cfg["seed"], synth.STREAM_V, B, Hkv, Sk, D, b, kv))[None, None]
                cache.clear()
                cache[(b, kv)] = (synth.bf16_bits_to_f64(qb[b:b + 1, kv * g:(kv + 1) * g]), ks, vs)
            oracle.forward(*cache[(b, kv)], causal=cfg["causal"])

        # Input generation is not timed: only the oracle calls.
        calls, used = 0, 0.0
        slices = {}
        while used < share * budget_s and calls < 1000 * len(order):
            b, kv = order[calls % len(order)]
            if (b, kv) not in slices:
                cache.clear()
                one(calls)  # builds the slice (untimed) and runs once (untimed)
                slices[(b, kv)] = cache[(b, kv)]
            cache[(b, kv)] = slices[(b, kv)]
            t0 = time.perf_counter()
            oracle.forward(*cache[(b, kv)], causal=cfg["causal"])
            used += time.perf_counter() - t0
            calls += 1
        nbytes = calls * (2 * g * D * 2 + 2 * Sk * D * 2)
        return {"value": round(nbytes / used / 1e9, 4), "unit": "GB/s",
                "sample": "%d calls over %d (batch, kv-head) groups of %d query heads x %d keys "
                          "(of %d groups), %.1f s" % (calls, len(order), g, Sk, B * Hkv, used)}

    def prefill_rows(cfg, share, causal_flops):
        B, Hq, Hkv, S, D = (cfg[x] for x in ("B", "Hq", "Hkv", "Sq", "D"))
        g = Hq // Hkv
        b, kv = B - 1, Hkv - 1
        qs = np.stack([synth.bf16_bits_to_f64(synth.kv_slice_bf16_bits(
            cfg["seed"], synth.STREAM_Q, B, Hq, S, D, b, kv * g + h)) for h in range(g)])[None]
        ks = synth.bf16_bits_to_f64(synth.kv_slice_bf16_bits(
            cfg["seed"], synth.STREAM_K, B, Hkv, S, D, b, kv))[None, None]
        vs = synth.bf16_bits_to_f64(synth.kv_slice_bf16_bits(
            cfg["seed"], synth.STREAM_V, B, Hkv, S, D, b, kv))[None, None]
        mask = None
        if cfg["mask"]:
            lens = synth.uniform_int(cfg["seed"], synth.STREAM_MASK, B, 256, S)
            mask = synth.mask_from_lengths(lens, S, S)[b:b + 1]
        rows = [(0, h, i) for i in range(0, S, 61) for h in range(g)]
        flops, n, used = 0.0, 0, 0.0
        while used < share * budget_s and n < 50 * len(rows):
            at = n % len(rows)
            chunk = rows[at:at + 64]
            t0 = time.perf_counter()
            oracle.forward_rows(qs, ks, vs, chunk, mask=mask, causal=cfg["causal"])
            used += time.perf_counter() - t0
            n += len(chunk)
            flops += sum(4.0 * D * ((i + 1) if causal_flops else S) for (_, _, i) in chunk)
        return {"value": round(flops / used / 1e9, 3), "unit": "GFLOP/s",
                "sample": "%d rows (cycling over query positions 0, 61, 122, ... of every head "
                          "of batch entry %d, kv head %d), %.1f s; FLOPs counted %s" % (
                              n, b, kv, used, "4*D per visible (causal) key" if causal_flops
                              else "4*D*Sk per row (the dense formula)")}

    per["decode_mistral7b_layer"] = decode_groups(DECODE, 0.35, 16)
    per["decode_llama2_70b_layer"] = decode_groups(DECODE_LONG, 0.2, 2)
    per["prefill_causal"] = prefill_rows(PREFILL_CAUSAL, 0.2, True)
    per["prefill_padded_mask"] = prefill_rows(PREFILL_MASKED, 0.2, False)
    head = per["decode_mistral7b_layer"]
    return dict(value=head["value"], unit="GB/s", cores=1, threads_used=1,
                host_cores=os.cpu_count(), kind="oracle",
                sample="decode workload: " + head["sample"] + "; every workload in per_config",
                per_config=per)


def _roofline_decode(res, hbm, peak_kind, workload, kernel_file="decode.cu"):
    per_s = res["per_launch_ms"] / 1e3
    ab = res["plan"]["algorithmic_bytes"]
    achieved = ab / per_s / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_source": peak_kind,
            "traffic": _traffic_for(kernel_file, workload),
            "algorithmic_bytes_per_launch": ab,
            "launch_ms": round(res["per_launch_ms"], 5)}


def _roofline_prefill(res, tflops, peak_kind, workload, kernel_file="prefill_pp.cu"):
    """Contiguous caches without lengths run on the two-tile kernel."""
    per_s = res["per_launch_ms"] / 1e3
    fl = res["plan"]["algorithmic_flops"]
    achieved = fl / per_s / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": tflops, "unit": "TFLOP/s",
            "frac": round(achieved / tflops, 4), "peak_source": peak_kind,
            "traffic": _traffic_for(kernel_file, workload),
            "algorithmic_flops_per_launch": fl, "launch_ms": round(res["per_launch_ms"], 5)}


def _roofline_ragged(res, hbm, peak_kind, workload):
    achieved = res["step_bytes"] / (res["per_launch_ms"] / 1e3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_source": peak_kind,
            "traffic": _traffic_for("decode.cu", workload),
            "algorithmic_bytes_per_step": int(res["step_bytes"]),
            "mean_len": round(res["mean_len"], 1), "kernels_per_step": res["launches"],
            "step_ms": round(res["per_launch_ms"], 5)}


def _roofline_ragged_prefill(res, cfg, tf_peak, peak_kind):
    """Tensor roofline of a prefill over per-sequence lengths: 4 * D FLOPs per
    visible (query, key) pair and query head."""
    flops = 4.0 * cfg["D"] * cfg["Hq"] * res["visible_pairs_per_head"]
    achieved = flops / (res["per_launch_ms"] / 1e3) / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": tf_peak, "unit": "TFLOP/s",
            "frac": round(achieved / tf_peak, 4), "peak_source": peak_kind,
            "traffic": _traffic_for("prefill_pp.cu", cfg["name"]),
            "algorithmic_flops_per_launch": flops, "mean_len": round(res["mean_len"], 1),
            "launch_ms": round(res["per_launch_ms"], 5)}


WORKLOADS = {c["name"]: c for c in (DECODE, DECODE_LONG, PREFILL_CAUSAL, PREFILL_MASKED,
                                    DECODE_RAGGED, DECODE_STEP, DECODE_PAGED, DECODE_F16,
                                    DECODE_D96, PREFILL_CHUNK_PAGED)}


def run_profile_case(args):
    """One workload alone, for profiler captures: warm-up, `steps` timed
    launches, one JSON line with the launch time."""
    import torch
    import grouped_query_attention_fwd_b200 as gqa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = WORKLOADS[args.profile]
    timer = _time_ragged if "lens" in cfg else _time_config
    res = timer(gqa, torch, cfg, steps=args.steps, warmup=args.warmup, dev=dev)
    print(json.dumps({"profile_case": cfg["name"], "launch_ms": res["per_launch_ms"],
                      "copies": res["copies"], "plan": res["plan"]}), flush=True)


def trace_summary(words, grid, launches, kv_bytes_per_unit):
    """Phase summary of `launches` consecutive decode launches from the
    per-CTA trace records (see gqa_debug_decode_trace); times in microseconds
    relative to each launch's first CTA entry."""
    import numpy as np
    W = 16
    t = np.asarray(words, dtype=np.int64).reshape(launches, grid, W)
    entry, ready, fissue, land, last = (t[:, :, i] for i in (1, 2, 3, 5, 6))
    merged, done, exit_, units = (t[:, :, i] for i in (7, 8, 9, 10))
    flushes, midns, kind = t[:, :, 11], t[:, :, 12], t[:, :, 13]
    t0 = entry.min(axis=1, keepdims=True)
    us = lambda x: (x - t0) / 1e3  # noqa: E731

    def stat(x):
        x = np.asarray(x, dtype=np.float64).ravel()
        return {"min": round(float(x.min()), 2), "median": round(float(np.median(x)), 2),
                "max": round(float(x.max()), 2)}

    span = (exit_.max(axis=1) - t0[:, 0]) / 1e3
    period = np.diff(t0[:, 0]) / 1e3
    gap = (entry.min(axis=1)[1:] - exit_.max(axis=1)[:-1]) / 1e3
    stream_us = (last - land) / 1e3
    rate = units * kv_bytes_per_unit / np.maximum(last - land, 1)  # bytes per ns = GB/s
    slowest = np.argmax(exit_, axis=1)
    return {
        "launches": int(launches), "grid": int(grid),
        "launch_period_us": stat(period),
        "gap_prev_exit_to_entry_us": stat(gap),
        "span_entry_to_last_exit_us": stat(span),
        "entry_us": stat(us(entry)),
        "ready_us": stat(us(ready)),
        "first_issue_us": stat(us(fissue)),
        "first_land_us": stat(us(land)),
        "last_tile_us": stat(us(last)),
        "final_merged_us": stat(us(merged)),
        "final_done_us": stat(us(done)),
        "exit_us": stat(us(exit_)),
        "stream_us_per_cta": stat(stream_us),
        "stream_gbs_per_cta": stat(rate),
        "stream_gbs_all_ctas": round(float(np.median(units.sum(axis=1) * kv_bytes_per_unit /
                                                     (last.max(axis=1) - land.min(axis=1)))), 1),
        "units_per_cta": stat(units),
        "mid_flush_us_per_cta": stat(midns / 1e3),
        "flushes_per_cta": stat(flushes),
        "final_kind_counts": {str(k): int((kind == k).sum()) for k in (0, 1, 2)},
        "final_merge_us": stat((merged - last) / 1e3),
        "final_write_us": stat((done - merged) / 1e3),
        "slowest_cta_units": stat(units[np.arange(launches), slowest]),
    }


def run_trace(args):
    """Per-CTA phase trace of one decode workload: one CUDA graph of
    consecutive launches with the trace buffer set, replayed a few times; the
    summary of the last replay is printed as one JSON line.  Ragged and paged
    caches are traced without the append step (the lengths stay fixed)."""
    import torch
    import numpy as np
    import grouped_query_attention_fwd_b200 as gqa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = WORKLOADS[args.trace]
    if cfg["Sq"] != 1 or cfg.get("append"):
        raise SystemExit("--trace takes a single-query decode workload without an append")
    q, k, v, _ = _host_inputs(cfg, torch)
    qd = q.to(dev)
    B, Hkv, Sk, D = cfg["B"], cfg["Hkv"], cfg["Sk"], cfg["D"]
    lens = table = None
    if "lens" in cfg:
        lo, hi = cfg["lens"]
        lens0 = synth.uniform_int(cfg["seed"], synth.STREAM_MASK, B, lo, hi).astype(np.int32)
        lens = torch.from_numpy(lens0).to(dev)
        kv_bytes = int(lens0.sum()) * Hkv * D * 2 * 2
    else:
        kv_bytes = 2 * k.numel() * 2
    copies = max(3, math.ceil(3 * L2_BYTES / kv_bytes))
    ks = [k.to(dev) for _ in range(copies)]
    vs = [v.to(dev) for _ in range(copies)]
    tables = [None] * copies
    ps = cfg.get("page")
    if ps:  # every (sequence, page) of the cache at a random slot of a pool
        per_seq = Sk // ps
        gen = torch.Generator().manual_seed(cfg["seed"])
        for i in range(copies):
            perm = torch.randperm(B * per_seq, generator=gen)
            inv = torch.empty_like(perm)
            inv[perm] = torch.arange(B * per_seq)

            def pool(x):
                return x.view(B, Hkv, per_seq, ps, D).permute(0, 2, 1, 3, 4).reshape(
                    B * per_seq, Hkv, ps, D)[perm.to(dev)].contiguous()
            ks[i], vs[i] = pool(ks[i]), pool(vs[i])
            tables[i] = inv.view(B, per_seq).to(torch.int32).to(dev)
    out = torch.empty(qd.shape, dtype=qd.dtype, device=dev)
    plan = gqa.query(qd, ks[0], vs[0], kv_lens=lens, block_table=tables[0])
    ws = gqa.workspace_for(dev, plan["workspace_bytes"])
    stream = torch.cuda.current_stream(dev)
    launches = 32
    grid = plan["grid"]

    def call(i):
        gqa.forward(qd, ks[i % copies], vs[i % copies], out=out, workspace=ws, kv_lens=lens,
                    block_table=tables[i % copies])
    buf = torch.zeros(launches * grid * 16, dtype=torch.int64, device=dev)
    for i in range(6):
        call(i)
    torch.cuda.synchronize()
    gqa.debug_decode_trace(buf)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(launches):
            call(i)
    gqa.debug_decode_trace(None)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    st = gqa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status after tracing: %s" % gqa.status_string(st))
    unit_bytes = 2 * 128 * D * 2
    raw = buf.cpu().numpy()
    if getattr(args, "trace_out", None):
        np.save(args.trace_out, raw.reshape(launches, grid, 16))
    summ = trace_summary(raw, grid, launches, unit_bytes)
    ms = e0.elapsed_time(e1) / launches
    summ.update({"trace_workload": cfg["name"], "launch_ms_graph": round(ms, 5),
                 "gbs_algorithmic": round(plan["algorithmic_bytes"] / (ms / 1e3) / 1e9, 1)
                 if lens is None else round((kv_bytes + 2 * qd.numel() * 2) / (ms / 1e3) / 1e9, 1)})
    print(json.dumps(summ), flush=True)
    del g


def run_gpu(args):
    import torch
    import grouped_query_attention_fwd_b200 as gqa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    hbm, tf_burst, tf_sus, peak_kind = _peaks()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(props.uuid)
    except Exception:
        gpu_id = None

    cfg = DECODE
    q, k, v, _ = _host_inputs(cfg, torch)
    qd = q.to(dev)
    kv_bytes = 2 * k.numel() * 2
    copies = max(3, math.ceil(3 * L2_BYTES / kv_bytes))
    ks = [k.to(dev) for _ in range(copies)]
    vs = [v.to(dev) for _ in range(copies)]
    del q, k, v
    out = torch.empty(qd.shape, dtype=qd.dtype, device=dev)
    plan = gqa.query(qd, ks[0], vs[0])
    ws = gqa.workspace_for(dev, plan["workspace_bytes"])
    stream = torch.cuda.current_stream(dev)

    calls = [(lambda i=i: gqa.forward(qd, ks[i], vs[i], out=out, workspace=ws))
             for i in range(copies)]
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    # The timed region (exactly --steps launches, a barrier and a device
    # synchronise before it) is repeated; every repetition is timed on the
    # device and reduced to its maximum over ranks, and the median
    # repetition gives the reported value.
    repeats = timing_repeats(args.steps)
    times, per, host_s = _graph_timed(torch, calls, args.steps, args.warmup, stream,
                                      repeats=repeats,
                                      before_each=(dist.barrier if dist is not None else None))
    t_wall1 = time.time()
    if dist is not None:
        dist.barrier()
    sampler.stop()
    single_launch = statistics.median(per)
    st = gqa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status after timing: %s" % gqa.status_string(st))
    times = [max_over_ranks(t, dist, dev) for t in times]
    elapsed_ms = statistics.median(times)
    # Average launch duration over the median timed region (graphs of many
    # launches); the one-launch-graph pass adds the graph launch to every launch.
    per_launch = elapsed_ms / args.steps
    del ks, vs
    torch.cuda.empty_cache()

    value = weak_scaling_gbs(plan["algorithmic_bytes"], args.steps, world, elapsed_ms)
    clocks = sampler.summary(t_wall0 - 0.2, t_wall1 + 0.2)

    line = {
        "metric": "GQA decode KV-read GB/s (% HBM peak); prefill TFLOP/s (% bf16 TC peak)",
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 5),
        "timing": {"repeats": repeats, "statistic": "median repetition (max over ranks)",
                   "ms_per_step_min": round(min(times) / args.steps, 5),
                   "ms_per_step_max": round(max(times) / args.steps, 5)},
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: q/k/v i.i.d. N(0,1) from a seeded SplitMix64/Box-Muller generator, rounded to bf16",
        "config": {
            "workload": "decode, Mistral-7B-shaped layer: B=16 Hq=32 Hkv=8 (g=4) Sq=1 Sk=4096 "
                        "D=128 bf16, no mask, scale=1/sqrt(128)",
            "B": 16, "Hq": 32, "Hkv": 8, "Sq": 1, "Sk": 4096, "D": 128,
            "parallelism": "replicas" if world == 1 else "dp%d (independent problems per rank)" % world,
            "l2": "K/V rotated over %d device copies (%.0f MB) so no launch finds its K/V in L2"
                  % (copies, copies * kv_bytes / 1e6),
            "launch": "one gqa_forward per step; each repetition of the %d steps is replayed "
                      "from CUDA graphs of up to %d launches (host enqueue %.2f us per step); "
                      "per-launch times from a separate pass of one-launch graphs"
                      % (args.steps, copies * max(1, min(64, args.steps) // copies)
                         if args.steps >= copies else args.steps, host_s * 1e6),
        },
        "gpu_launches": args.steps * plan["launches"],
        "clocks": {k_: v_ for k_, v_ in clocks.items()},
        "roofline": {
            "bound": "hbm",
            "achieved": round(plan["algorithmic_bytes"] / (per_launch / 1e3) / 1e9, 1),
            "peak": hbm,
            "unit": "GB/s",
            "frac": round(plan["algorithmic_bytes"] / (per_launch / 1e3) / 1e9 / hbm, 4),
            "traffic": _traffic_for("decode.cu", DECODE["name"]),
            "peak_source": peak_kind,
            "kernel": "gqa_decode_kernel (split merge fused; the counter memset is in the same graph)",
            "algorithmic_bytes_per_launch": plan["algorithmic_bytes"],
            "launch_ms": round(per_launch, 5),
            "launch_ms_basis": "median timed region / steps (CUDA events around the graphs of "
                               "launches)",
            "single_launch_graph_median_ms": round(single_launch, 5),
        },
    }

    if rank == 0 and world == 1 and not args.skip_extra:
        extra = {}
        for c in (DECODE_LONG, PREFILL_CAUSAL, PREFILL_MASKED, DECODE_RAGGED, DECODE_STEP,
                  DECODE_PAGED, DECODE_F16, DECODE_D96, PREFILL_CHUNK_PAGED):
            timer = _time_ragged if "lens" in c else _time_config
            try:
                res = timer(gqa, torch, c, steps=max(3, min(args.steps, 50)),
                            warmup=max(3, min(args.warmup, 10)), dev=dev)
            except Exception as e:  # report, keep the primary line
                extra[c["name"]] = {"unavailable": "%s: %s" % (type(e).__name__, e)}
                continue
            if "lens" in c and c["Sq"] > 1:
                rf = _roofline_ragged_prefill(res, c, tf_burst, peak_kind)
                extra[c["name"]] = {"value": rf["achieved"], "unit": "TFLOP/s", "roofline": rf,
                                    "frac_of_sustained_peak": round(rf["achieved"] / tf_sus, 4)}
            elif "lens" in c:
                rf = _roofline_ragged(res, hbm, peak_kind, c["name"])
                extra[c["name"]] = {"value": rf["achieved"], "unit": "GB/s", "roofline": rf}
            elif c["Sq"] == 1:
                rf = _roofline_decode(res, hbm, peak_kind, c["name"])
                extra[c["name"]] = {"value": rf["achieved"], "unit": "GB/s", "roofline": rf}
            else:
                rf = _roofline_prefill(res, tf_burst, peak_kind, c["name"])
                vis = res["visible_pairs"] * 4 * c["D"] / (res["per_launch_ms"] / 1e3) / 1e12
                extra[c["name"]] = {"value": rf["achieved"], "unit": "TFLOP/s", "roofline": rf,
                                    "visible_pairs_tflops": round(vis, 1),
                                    "frac_of_sustained_peak": round(rf["achieved"] / tf_sus, 4)}
        line["extra"] = extra

    if rank == 0 and not args.skip_e2e:
        e2e_steps = max(3, min(args.steps, 20))
        ms, h2d, d2h = _e2e(gqa, torch, DECODE, e2e_steps, dev)
        line["e2e"] = {"value": round(plan["algorithmic_bytes"] / (ms / 1e3) / 1e9, 2),
                       "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": round(ms, 4),
                       "note": "pinned host q/k/v copied to the device, gqa_forward, out copied back, every step"}
    if rank == 0 and world == 1 and not args.skip_cpu:
        line["cpu_baseline"] = _cpu_baseline()

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------ reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    cfg = DECODE
    B, Hq, Hkv, Sk, D = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["Sk"], cfg["D"]
    g = Hq // Hkv
    qb = synth.normal_bf16_bits(cfg["seed"], synth.STREAM_Q, B * Hq * D).reshape(B, Hq, 1, D)
    order = [(b, kv) for b in range(B) for kv in range(Hkv)]
    cache = {}

    def group(i):
        b, kv = order[i % len(order)]
        if (b, kv) not in cache:
            ks = synth.bf16_bits_to_f64(synth.kv_slice_bf16_bits(cfg["seed"], synth.STREAM_K, B, Hkv, Sk, D, b, kv))
            vs = synth.bf16_bits_to_f64(synth.kv_slice_bf16_bits(cfg["seed"], synth.STREAM_V, B, Hkv, Sk, D, b, kv))
            cache[(b, kv)] = (synth.bf16_bits_to_f64(qb[b:b + 1, kv * g:(kv + 1) * g]),
                              ks[None, None], vs[None, None])
        return cache[(b, kv)]

    # Calibrate one group, then size each step so that the run stays bounded.
    t0 = time.perf_counter()
    oracle.forward(*group(0))
    t_group = max(time.perf_counter() - t0, 1e-4)
    budget = 60.0
    per_step = int(max(1, min(len(order), budget / ((args.steps + args.warmup) * t_group))))
    group_bytes = 2 * g * D * 2 + 2 * Sk * D * 2
    idx = 0
    for _ in range(args.warmup):
        for _ in range(per_step):
            oracle.forward(*group(idx))
            idx += 1
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for _ in range(per_step):
            oracle.forward(*group(idx))
            idx += 1
    el = time.perf_counter() - t0
    value = group_bytes * per_step * args.steps / el / 1e9
    sample = ("%d of %d (batch, kv-head) groups per step (g=%d query heads x %d keys each), "
              "fp64 oracle, single thread" % (per_step, len(order), g, Sk))
    line = {
        "metric": "GQA decode KV-read GB/s (% HBM peak); prefill TFLOP/s (% bf16 TC peak)",
        "impl": "reference",
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: same seeded inputs as the GPU arm",
        "config": {"workload": "decode, Mistral-7B-shaped layer: B=16 Hq=32 Hkv=8 Sq=1 Sk=4096 "
                               "D=128, bounded sample per step (see cpu_baseline.sample)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "threads_used": 1,
                         "host_cores": os.cpu_count(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-extra", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--profile", default=None, choices=sorted(WORKLOADS),
                    help="time one workload alone (for ncu captures) and exit")
    ap.add_argument("--trace", default=None, choices=sorted(WORKLOADS),
                    help="per-CTA phase trace of one decode workload, then exit")
    ap.add_argument("--trace-out", default=None,
                    help="with --trace: also save the raw records (.npy, [launch, CTA, word])")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.profile:
        run_profile_case(args)
    elif args.trace:
        run_trace(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
