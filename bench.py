"""Benchmark of the mLSTM hot path on B200: chunkwise prefill + decode step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0.  Headline (value): chunkwise-prefill tokens/s of the
large-head workload (B1 NH8 S8192 DHQK256 DHV512 chunk64, bf16 in / fp32 state),
with its dominant kernel's TFLOP/s against the measured bf16 tensor peak.  The
decode workload (B128 NH8 256x512, fp32 state updated in place) is measured in
the same run and reported under "decode" with its state GB/s against the
measured HBM bandwidth.  The path does not shard: with N GPUs every rank runs
its own replica (weak scaling) and value sums the tokens of all ranks over the
slowest rank's time.  --impl reference times the fp64 CPU oracle on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import contextlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mLSTM chunkwise-fwd tokens/s (% bf16 TC peak); decode-step state GB/s (% HBM)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch, from one ncu
# capture, with the sha256 of the files the kernel's device code is compiled from at capture
# time (kernels.h holds host-side declarations only and is left out).  Reported only while
# those files still hash the same; otherwise the counters are stale and traffic is null.
CSRC = os.path.join(ROOT, "linear_recurrent_token_b200", "csrc")
RECORDED_TRAFFIC = {
    ("tc_walk", "large_head"): {
        "bytes": 147_710_464 + 40_030_720,
        "sources": ("chunkwise_tc.cu", "sm100.cuh", "common.cuh", "tma_host.h", "bounds.cuh"),
        "sha256": "fa7f51da28ffcdb68077c88edc89294d57efe21d37fa4c4f1db2478596444c72",
    },
    ("step", "decode"): {
        "bytes": 540_096_256 + 480_655_616,
        "sources": ("step.cu", "common.cuh"),
        "sha256": "6a2af416eaaca085e74fcec66ede057e8949d55ec30f6f0672f423cdc0dcc707",
    },
}


def sources_sha256(names) -> str:
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(CSRC, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: str):
    r = RECORDED_TRAFFIC.get((kernel, workload))
    if r is None or sources_sha256(r["sources"]) != r["sha256"]:
        return None
    return r["bytes"]


# ------------------------------------------------------------------ work accounting
def chunkwise_flops(B, NH, S, dk, dv, L, nb=1, retention=False):
    """Algorithmic flops of a chunkwise prefill: causal intra-chunk pairs (L+1)(dk+dv) per
    token, inter-chunk read-out 2 dk dv and update 2 dk dv per token, normaliser 4 dk
    (not in retention); per (head, block), dk and dv of one block."""
    per_tok = (L + 1) * (dk + dv) + 4 * dk * dv + (0 if retention else 4 * dk)
    return B * NH * nb * S * per_tok


def chunkwise_min_bytes(B, NH, S, DHQK, DHV, esize, nb=1, retention=False):
    """Each input read once, h written once, final state written once."""
    tok = B * NH * S
    b = tok * (2 * DHQK + 2 * DHV) * esize  # q, k, v in; h out
    if not retention:
        b += tok * 2 * 4  # gates
    b += B * NH * (DHV * DHQK // nb + (0 if retention else DHQK + 1)) * 4
    return b


def decode_step_bytes(B, NH, DHQK, DHV, esize, nb=1):
    """Bytes one decode step must move: C and n read + written (fp32), m read + written,
    q, k, v read, h written, two gates read."""
    state = B * NH * (DHV * DHQK // nb + DHQK) * 4 * 2 + B * NH * 4 * 2
    io = B * NH * (2 * DHQK + 2 * DHV) * esize + B * NH * 2 * 4
    return state + io


def decode_step_flops(B, NH, DHQK, DHV, nb=1):
    """Update (f'C + i' v k^T: 3 flops/element) plus read-out (2 per element) plus n."""
    return B * NH * (5 * DHV * DHQK // nb + 6 * DHQK)


def backward_flops(B, NH, S, dk, dv, nb=1):
    """Algorithmic flops of the backward as the sequential reverse-mode evaluation does them:
    per token and block six dk x dv products or rank-1 updates (state update, read-out, dq,
    update of dL/dC, dv, dk), 2 flops per element; vector terms omitted."""
    return B * NH * S * nb * 12 * dk * dv


def fp32_simt_peak_tflops(sm_mhz):
    """B200 fp32 FMA throughput from unit counts: 148 SMs x 128 fp32 lanes x 2 flops x clock."""
    return 148 * 128 * 2 * (sm_mhz or 1965.0) * 1e6 / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ distributed helpers
def dist_setup(gpus: int):
    """Returns (rank, world, local_rank); initialises NCCL when launched under torchrun."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def dist_max(x: float, world: int) -> float:
    """Maximum of a float over ranks (the slowest rank's time)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ NVTX
@contextlib.contextmanager
def nvtx(name):
    """An NVTX range around a bench region (named in a timeline profiler's view)."""
    import torch

    torch.cuda.nvtx.range_push(name)
    try:
        yield
    finally:
        torch.cuda.nvtx.range_pop()


# ------------------------------------------------------------------ L2 flush
class L2Flush:
    """Evicts the previous step's data from the 126 MB L2 between timed steps: a write of a
    buffer larger than L2, then a read of a second one, so that the L2 holds only clean lines of
    the second buffer when the next step starts (the write-back of the first buffer's dirty lines
    would otherwise land inside the next timed step and be charged to its kernels)."""

    def __init__(self, nbytes):
        import torch

        self.w = torch.empty(nbytes // 4, dtype=torch.float32, device="cuda")
        self.r = torch.zeros(nbytes // 4, dtype=torch.float32, device="cuda")
        self.acc = torch.zeros((), dtype=torch.float32, device="cuda")

    def __call__(self, value=1.0):
        import torch

        self.w.fill_(value)
        torch.sum(self.r, dim=0, out=self.acc)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the GPU is busy."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None
        self.active = False

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append((self.active, parts))

    def mark(self, active: bool):
        self.active = active

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        rows = [p for a, p in self.rows if a] or [p for _, p in self.rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle
def oracle_chunkwise_sample(w, tokens: int):
    """The fp64 oracle over the first `tokens` positions of every (batch, head) of the
    workload; returns (seconds, tokens_processed, threads)."""
    import oracle
    from linear_recurrent_token_b200 import inputs
    inp = inputs.forward_inputs(w, S=tokens)
    threads = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    oracle.sequential(inp["q"], inp["k"], inp["v"], inp["igate"], inp["fgate"], num_blocks=w.num_blocks,
                      retention=w.retention, threads=threads)
    return time.perf_counter() - t0, w.B * tokens, min(threads, w.B * w.NH * w.num_blocks)


def cpu_baseline(w, budget_s: float = 12.0, steps: int = 1):
    """Oracle tokens/s on a bounded sample: the sampled prefix is sized so that `steps`
    repetitions take about budget_s seconds in total (capped at the whole sequence)."""
    tokens = min(w.S, 128)
    secs, _, _ = oracle_chunkwise_sample(w, tokens)
    per_step = budget_s / max(1, steps)
    if secs < per_step and tokens < w.S:
        tokens = int(min(w.S, max(tokens, tokens * per_step / max(secs, 1e-3))))
    total_s, total_tok, threads, times = 0.0, 0, 1, []
    for _ in range(max(1, steps)):
        secs, done, threads = oracle_chunkwise_sample(w, tokens)
        total_s += secs
        total_tok += done
        times.append(secs)
    sample = (f"first {tokens} of {w.S} positions of all {w.B * w.NH} (batch, head) sequences of "
              f"{w.describe()}, fp64 sequential recurrence, {len(times)} repetition(s)")
    return {"value": total_tok / total_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": sample, "ms_per_step": 1e3 * total_s / len(times)}


# ------------------------------------------------------------------ GPU legs
def run_chunkwise(w, steps, warmup, flush_bytes, clocks):
    import torch

    from linear_recurrent_token_b200 import inputs, mlstm
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    inp = inputs.forward_inputs(w)
    dev = lambda x, dt: torch.from_numpy(np.ascontiguousarray(x)).to("cuda", dt)
    q, k, v = dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td)
    ig, fg = dev(inp["igate"], torch.float32), dev(inp["fgate"], torch.float32)
    h = torch.empty((w.B, w.NH, w.S, w.DHV), dtype=td, device="cuda")
    C = torch.empty((w.B, w.NH, w.num_blocks, w.dv, w.dk), dtype=torch.float32, device="cuda")
    n = torch.empty((w.B, w.NH, w.num_blocks, w.dk), dtype=torch.float32, device="cuda")
    m = torch.empty((w.B, w.NH), dtype=torch.float32, device="cuda")
    p = mlstm.fwd_params(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.num_blocks, td, w.retention)
    plan = mlstm.plan(p)
    ws = torch.empty(max(1, plan["workspace_bytes"]), dtype=torch.uint8, device="cuda")
    flush = L2Flush(flush_bytes)
    stream = torch.cuda.current_stream()
    gi = (None, None) if w.retention else (ig, fg)

    def one(ev=None):
        mlstm.fwd_chunkwise(q, k, v, *gi, chunk=w.chunk, num_blocks=w.num_blocks, retention=w.retention,
                            h=h, C_out=C, n_out=None if w.retention else n, m_out=None if w.retention else m,
                            workspace=ws, stream=stream, events=ev)

    for _ in range(warmup):
        flush(1.0)
        one()
    torch.cuda.synchronize()
    # steps: events around the whole call only (an event recorded between the call's kernels would
    # stop the next one from starting early, as the walk's first segment does, and serialise them)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    clocks.mark(True)
    t_wall = time.perf_counter()
    with nvtx(f"prefill steps: {w.name}"):
        for e in ev:
            flush(float(len(ev)))
            e[0].record(stream)
            one()
            e[1].record(stream)
        torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    # the dominant kernel alone: the same calls with events recorded by the library around it
    evk = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(max(3, steps // 2))]
    with nvtx(f"prefill, walk timed alone: {w.name}"):
        for e in evk:
            flush(2.0)
            one((e[0], e[1]))
        torch.cuda.synchronize()
    clocks.mark(False)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    main_ms = [c.elapsed_time(d) for c, d in evk]
    return dict(step_ms=step_ms, main_ms=main_ms, wall_s=t_wall, plan=plan,
                tensors=(q, k, v, ig, fg, h, C, n, m, ws))


def run_chunkwise_e2e(w, steps, tensors):
    """Same prefill through the public API with HOST buffers: every step copies its pinned
    host inputs in, runs the call and copies h and the final state back, all inside the timed
    region.  Steps are pipelined the way a serving loop would run them: step i+1's inputs
    upload on one stream while step i computes on another and step i-1's outputs download on
    a third (device inputs and outputs double-buffered); per step time = total / steps."""
    import torch

    from linear_recurrent_token_b200 import mlstm
    q, k, v, ig, fg, h, C, n, m, ws = tensors
    pin = lambda t: t.cpu().pin_memory()
    hq, hk, hv, hig, hfg = pin(q), pin(k), pin(v), pin(ig), pin(fg)
    oh, oC, on_, om = (torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (h, C, n, m))
    # second device copies of the per-step tensors
    dev_in = [(q, k, v, ig, fg), tuple(torch.empty_like(t) for t in (q, k, v, ig, fg))]
    dev_out = [(h, C, n, m), tuple(torch.empty_like(t) for t in (h, C, n, m))]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    in_free = [torch.cuda.Event() for _ in range(2)]
    out_ready = [torch.cuda.Event() for _ in range(2)]
    out_free = [torch.cuda.Event() for _ in range(2)]

    def upload(i):
        b = i % 2
        s_in.wait_event(in_free[b])
        with torch.cuda.stream(s_in):
            for d, hsrc in zip(dev_in[b], (hq, hk, hv, hig, hfg)):
                if w.retention and d.dtype == torch.float32 and d.dim() == 3:
                    continue
                d.copy_(hsrc, non_blocking=True)
        in_ready[b].record(s_in)

    def run(i):
        b = i % 2
        qq, kk, vv, gi_, gf_ = dev_in[b]
        hh, CC, nn, mm = dev_out[b]
        s_run.wait_event(in_ready[b])
        s_run.wait_event(out_free[b])
        gates = (None, None) if w.retention else (gi_, gf_)
        mlstm.fwd_chunkwise(qq, kk, vv, *gates, chunk=w.chunk, num_blocks=w.num_blocks, retention=w.retention,
                            h=hh, C_out=CC, n_out=None if w.retention else nn, m_out=None if w.retention else mm,
                            workspace=ws, stream=s_run)
        in_free[b].record(s_run)
        out_ready[b].record(s_run)

    def download(i):
        b = i % 2
        s_out.wait_event(out_ready[b])
        with torch.cuda.stream(s_out):
            outs = (oh, oC) + (() if w.retention else (on_, om))
            for dst, src in zip(outs, dev_out[b]):
                dst.copy_(src, non_blocking=True)
        out_free[b].record(s_out)

    def pipeline(nsteps):
        upload(0)
        for i in range(nsteps):
            if i + 1 < nsteps:
                upload(i + 1)
            run(i)
            download(i)

    for b in range(2):  # events start signalled
        in_free[b].record(s_run)
        out_free[b].record(s_out)
    pipeline(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with nvtx(f"prefill end to end, host buffers: {w.name}"):
        e0.record(s_in)
        pipeline(steps)
        s_in.wait_stream(s_out)
        e1.record(s_in)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = sum(t.numel() * t.element_size() for t in ((hq, hk, hv) + (() if w.retention else (hig, hfg))))
    d2h = sum(t.numel() * t.element_size() for t in ((oh, oC) + (() if w.retention else (on_, om))))
    return ms, h2d, d2h


def run_decode(w, steps, warmup, clocks):
    import torch

    from linear_recurrent_token_b200 import inputs, mlstm
    td = torch.bfloat16
    T = min(w.steps, steps + warmup)
    C0, n0, m0 = inputs.decode_initial_state(w)
    C = torch.from_numpy(C0).cuda()
    n = torch.from_numpy(n0).cuda()
    m = torch.from_numpy(m0).cuda()
    per = [inputs.decode_step_inputs(w, t) for t in range(T)]
    stack = lambda key, dt: torch.from_numpy(np.stack([p[key] for p in per])).to("cuda", dt)
    q, k, v = stack("q", td), stack("k", td), stack("v", td)
    ig, fg = stack("igate", torch.float32), stack("fgate", torch.float32)
    h = torch.empty((T, w.B, w.NH, w.DHV), dtype=td, device="cuda")
    stream = torch.cuda.current_stream()
    for t in range(warmup):
        mlstm.step(q[t % T], k[t % T], v[t % T], ig[t % T], fg[t % T], C, n, m, h=h[t % T], stream=stream)
    torch.cuda.synchronize()
    # the K steps back to back between one pair of events, as a decode loop runs them (the
    # state exceeds L2, so no flush is needed between steps)
    e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.mark(True)
    with nvtx(f"decode steps: {w.name}"):
        e_a.record(stream)
        for i in range(steps):
            t = (warmup + i) % T
            mlstm.step(q[t], k[t], v[t], ig[t], fg[t], C, n, m, h=h[t], stream=stream)
        e_b.record(stream)
        torch.cuda.synchronize()
    clocks.mark(False)
    step_ms = [e_a.elapsed_time(e_b) / steps] * steps

    # end to end: per step, pinned host q/k/v/gates in, the step, h out; pipelined as in a
    # serving loop (step t+1's inputs upload while step t runs and step t-1's h downloads)
    hq, hk, hv = (x[:1].cpu().pin_memory() for x in (q, k, v))
    hig, hfg = (x[:1].cpu().pin_memory() for x in (ig, fg))
    oh = torch.empty(h[0].shape, dtype=td).pin_memory()
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_ran = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b_ in range(2):
        ev_ran[b_].record(s_run)
        ev_out[b_].record(s_out)

    def upload(i):
        b_ = i % 2
        s_in.wait_event(ev_ran[b_])  # step i-2 is done with slot b_
        with torch.cuda.stream(s_in):
            for d, src in zip((q, k, v, ig, fg), (hq, hk, hv, hig, hfg)):
                d[b_].copy_(src[0], non_blocking=True)
        ev_in[b_].record(s_in)

    def run(i):
        b_ = i % 2
        s_run.wait_event(ev_in[b_])
        s_run.wait_event(ev_out[b_])  # h slot b_ has been downloaded
        mlstm.step(q[b_], k[b_], v[b_], ig[b_], fg[b_], C, n, m, h=h[b_], stream=s_run)
        ev_ran[b_].record(s_run)

    def download(i):
        b_ = i % 2
        s_out.wait_event(ev_ran[b_])
        with torch.cuda.stream(s_out):
            oh.copy_(h[b_], non_blocking=True)
        ev_out[b_].record(s_out)

    def pipeline(nsteps):
        upload(0)
        for i in range(nsteps):
            if i + 1 < nsteps:
                upload(i + 1)
            run(i)
            download(i)

    pipeline(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with nvtx(f"decode end to end, host buffers: {w.name}"):
        e0.record(s_in)
        pipeline(steps)
        s_in.wait_stream(s_out)
        e1.record(s_in)
        torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / steps
    h2d = sum(x[0].numel() * x.element_size() for x in (hq, hk, hv, hig, hfg))
    d2h = oh.numel() * oh.element_size()
    return dict(step_ms=step_ms, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h)


def oracle_backward_sample(w, tokens: int, heads: int):
    """The fp64 backward oracle on the first `tokens` positions of `heads` (batch, head)
    sequences of the workload; returns (seconds, tokens processed)."""
    import oracle
    from linear_recurrent_token_b200 import inputs
    inp = inputs.forward_inputs(w, S=tokens)
    rng = np.random.default_rng(3000)
    sel = lambda x: None if x is None else x[:1, :heads]
    dh = rng.standard_normal((1, heads, tokens, w.DHV))
    t0 = time.perf_counter()
    oracle.sequential_backward(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), dh, sel(inp.get("igate")),
                               sel(inp.get("fgate")), num_blocks=w.num_blocks, retention=w.retention)
    return time.perf_counter() - t0, tokens * heads


def run_backward(w, steps, warmup, flush_bytes, clocks):
    """The backward (mlstm_bwd) on the workload's shapes, inputs resident, L2 flushed
    between steps; returns per-step milliseconds."""
    import torch

    from linear_recurrent_token_b200 import inputs, mlstm
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    inp = inputs.forward_inputs(w)
    rng = np.random.default_rng(3001)
    d = lambda x, dt=torch.float32: None if x is None else torch.from_numpy(np.ascontiguousarray(x)).to("cuda", dt)
    q, k, v = d(inp["q"], td), d(inp["k"], td), d(inp["v"], td)
    ig, fg = d(inp.get("igate")), d(inp.get("fgate"))
    dh = d(rng.standard_normal((w.B, w.NH, w.S, w.DHV)), td)
    p = mlstm.fwd_params(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.num_blocks, td, w.retention)
    ws = torch.empty(max(mlstm.bwd_workspace_size(p), 16), dtype=torch.uint8, device="cuda")
    flush = L2Flush(flush_bytes)
    for _ in range(warmup):
        mlstm.bwd(q, k, v, dh, ig, fg, num_blocks=w.num_blocks, retention=w.retention, workspace=ws)
    torch.cuda.synchronize()
    ms = []
    clocks.mark(True)
    for _ in range(steps):
        flush(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with nvtx(f"backward step: {w.name}"):
            a.record()
            mlstm.bwd(q, k, v, dh, ig, fg, num_blocks=w.num_blocks, retention=w.retention, workspace=ws)
            b.record()
            torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    clocks.mark(False)
    return ms


def run_reversed(w, steps, warmup, flush_bytes):
    """The reversed-sequence prefill (mlstm_fwd_chunkwise_reversed) on the workload, inputs
    resident, L2 flushed between steps; returns per-step milliseconds."""
    import torch

    from linear_recurrent_token_b200 import inputs, mlstm
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    inp = inputs.forward_inputs(w)
    d = lambda x, dt=torch.float32: None if x is None else torch.from_numpy(np.ascontiguousarray(x)).to("cuda", dt)
    q, k, v = d(inp["q"], td), d(inp["k"], td), d(inp["v"], td)
    ig, fg = d(inp.get("igate")), d(inp.get("fgate"))
    p = mlstm.fwd_params(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.num_blocks, td, w.retention)
    ws = torch.empty(mlstm.reversed_workspace_size(p), dtype=torch.uint8, device="cuda")
    h = torch.empty((w.B, w.NH, w.S, w.DHV), dtype=td, device="cuda")
    flush = L2Flush(flush_bytes)
    call = lambda: mlstm.fwd_chunkwise(q, k, v, ig, fg, chunk=w.chunk, num_blocks=w.num_blocks,
                                       retention=w.retention, h=h, workspace=ws, reverse=True)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with nvtx(f"reversed step: {w.name}"):
            a.record()
            call()
            b.record()
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    return ms


def run_scalar_normaliser(w, steps, warmup, flush_bytes):
    """The scalar-normaliser prefill (mlstm_fwd_chunkwise_scalar_normaliser, one n per head
    and a per-head bias) on the workload, inputs resident, L2 flushed between steps; returns
    per-step milliseconds."""
    import torch

    from linear_recurrent_token_b200 import inputs, mlstm
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    inp = inputs.forward_inputs(w)
    d = lambda x, dt=torch.float32: None if x is None else torch.from_numpy(np.ascontiguousarray(x)).to("cuda", dt)
    q, k, v = d(inp["q"], td), d(inp["k"], td), d(inp["v"], td)
    ig, fg = d(inp["igate"]), d(inp["fgate"])
    bias = torch.full((w.NH,), 0.5, dtype=torch.float32, device="cuda")
    p = mlstm.fwd_params(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.num_blocks, td, False)
    ws = torch.empty(max(1, mlstm.scalar_normaliser_workspace_size(p)), dtype=torch.uint8, device="cuda")
    flush = L2Flush(flush_bytes)
    call = lambda: mlstm.fwd_chunkwise_scalar_normaliser(q, k, v, ig, fg, bias, chunk=w.chunk,
                                                         num_blocks=w.num_blocks, workspace=ws)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with nvtx(f"scalar-normaliser step: {w.name}"):
            a.record()
            call()
            b.record()
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    return ms


def run_msr(w, steps, warmup, flush_bytes, hbm_peak):
    """The multi-scale retention block (mlstm_fwd_chunkwise_msr: rotation of q and k, the
    recurrence, GroupNorm + SiLU gate) on the workload, inputs resident, L2 flushed between
    steps; also the plain forward, and the rotation and GroupNorm kernels alone with their
    bytes against the HBM peak.  Returns a dict for the JSON line."""
    import torch

    from linear_recurrent_token_b200 import inputs, mlstm
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    esz = 2 if w.dtype == "bf16" else 4
    inp = inputs.forward_inputs(w)
    d = lambda x, dt=torch.float32: None if x is None else torch.from_numpy(np.ascontiguousarray(x)).to("cuda", dt)
    q, k, v = d(inp["q"], td), d(inp["k"], td), d(inp["v"], td)
    ig = None if w.retention else d(inp["igate"])
    fg = None if w.retention else d(inp["fgate"])
    rng = np.random.default_rng(7)
    g = torch.from_numpy(rng.standard_normal((w.B, w.NH, w.S, w.DHV)).astype(np.float32)).to("cuda", td)
    gw = torch.ones(w.NH * w.DHV, dtype=torch.float32, device="cuda")
    gb = torch.zeros(w.NH * w.DHV, dtype=torch.float32, device="cuda")
    pos0 = torch.zeros(w.B, dtype=torch.int64, device="cuda")
    p = mlstm.fwd_params(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.num_blocks, td, w.retention)
    ws = torch.empty(max(1, mlstm.msr_workspace_size(p)), dtype=torch.uint8, device="cuda")
    wsf = torch.empty(max(1, mlstm.workspace_size(p)), dtype=torch.uint8, device="cuda")
    y = torch.empty((w.B, w.NH, w.S, w.DHV), dtype=td, device="cuda")
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    flush = L2Flush(flush_bytes)
    calls = {
        "block": lambda: mlstm.fwd_chunkwise_msr(q, k, v, ig, fg, g, gw, gb, pos0=pos0, chunk=w.chunk,
                                                 num_blocks=w.num_blocks, retention=w.retention, y=y, workspace=ws),
        "forward": lambda: mlstm.fwd_chunkwise(q, k, v, ig, fg, chunk=w.chunk, num_blocks=w.num_blocks,
                                               retention=w.retention, h=y, workspace=wsf, return_state=False),
        "rotate": lambda: mlstm.theta_rotate(q, k, pos0, q_out=qo, k_out=ko),
        "gn_gate": lambda: mlstm.group_norm_gate(v, g, gw, gb, 1e-5, y=y),
    }
    out = {}
    for name, call in calls.items():
        for _ in range(warmup):
            call()
        torch.cuda.synchronize()
        ms = []
        for _ in range(steps):
            flush(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with nvtx(f"retention block, {name}: {w.name}"):
                a.record()
                call()
                b.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        out[name] = statistics.median(ms)
    tok = w.B * w.NH * w.S
    rot_bytes = 4 * tok * w.DHQK * esz
    gn_bytes = 3 * tok * w.DHV * esz + 2 * w.NH * w.DHV * 4
    return {"block_ms": out["block"], "forward_ms": out["forward"], "steps": steps,
            "rotate": {"ms": out["rotate"], "bytes_per_launch": rot_bytes,
                       "roofline": {"bound": "hbm", "achieved": rot_bytes / (out["rotate"] * 1e-3) / 1e9,
                                    "peak": hbm_peak, "unit": "GB/s",
                                    "frac": rot_bytes / (out["rotate"] * 1e-3) / 1e9 / hbm_peak, "traffic": None,
                                    "kernel": "theta_rotate_kernel"}},
            "gn_gate": {"ms": out["gn_gate"], "bytes_per_launch": gn_bytes,
                        "roofline": {"bound": "hbm", "achieved": gn_bytes / (out["gn_gate"] * 1e-3) / 1e9,
                                     "peak": hbm_peak, "unit": "GB/s",
                                     "frac": gn_bytes / (out["gn_gate"] * 1e-3) / 1e9 / hbm_peak, "traffic": None,
                                     "kernel": "gn_gate_kernel (standalone; v as h)"}}}


def gdn2_flops(B, H, T, K, V):
    """Algorithmic flops of the GDN-2 recurrence: per token and head the decay (K V), the
    read-out r = S'^T k (2 K V), the erase and write (4 K V) and o = S^T q (2 K V)."""
    return B * H * T * 9 * K * V


def gdn2_chunk_on_tensor_cores(wl):
    """Whether mlstm_gdn2_fwd runs the chunk mode on the tensor-core kernels for this workload
    (the library's rule: bf16, chunk 64, K 128, V 64 or 128)."""
    return wl.dtype == "bf16" and wl.chunk == 64 and wl.K == 128 and wl.V in (64, 128) and wl.T > 0


def gdn2_min_bytes(wl):
    """Bytes a GDN-2 prefill must move: q, k, v (dtype), g, b, w (fp32) read once, o written,
    the fp32 state read and written."""
    esz = 2 if wl.dtype == "bf16" else 4
    tok = wl.B * wl.H * wl.T
    return tok * (2 * wl.K * esz + wl.V * esz + 2 * wl.K * 4 + wl.V * 4 + wl.V * esz) + 2 * wl.B * wl.H * wl.K * wl.V * 4


def run_gdn2(steps, warmup, flush_bytes, peaks, sm_mhz):
    """Gated DeltaNet-2: the prefill workload in both modes (fused recurrent, chunk) and the
    decode workload (one token per sequence, state in place), inputs resident, L2 flushed
    between steps.  Returns the dict for the JSON line."""
    import torch

    from linear_recurrent_token_b200 import inputs, mlstm
    out = {}
    flush = L2Flush(flush_bytes)

    def timed(call):
        for _ in range(warmup):
            call()
        torch.cuda.synchronize()
        ms = []
        for _ in range(steps):
            flush(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with nvtx("GDN-2 step"):
                a.record()
                call()
                b.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        return statistics.median(ms)

    for wl in inputs.GDN2_WORKLOADS:
        td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        inp = inputs.gdn2_inputs(wl.B, wl.H, wl.T, wl.K, wl.V, wl.dtype, seed=7)
        d = lambda x, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(x)).to("cuda", dt)
        q, k, v = d(inp["q"], td), d(inp["k"], td), d(inp["v"], td)
        g, b, w, S0 = d(inp["g"]), d(inp["b"]), d(inp["w"]), d(inp["S0"])
        o = torch.empty((wl.B, wl.H, wl.T, wl.V), dtype=td, device="cuda")
        esz = 2 if wl.dtype == "bf16" else 4
        flops = gdn2_flops(wl.B, wl.H, wl.T, wl.K, wl.V)
        fp32_peak = fp32_simt_peak_tflops(sm_mhz)
        if wl.T > 1:
            S_out = torch.empty_like(S0)
            modes = {}
            for mode in ("recurrent", "chunk"):
                ms = timed(lambda: mlstm.gdn2_fwd(q, k, v, g, b, w, S0, mode=mode, chunk=wl.chunk, o=o, S_out=S_out))
                tf = flops / (ms * 1e-3) / 1e12
                if mode == "chunk" and gdn2_chunk_on_tensor_cores(wl):
                    # the whole call against HBM: every input read once, o written, the state
                    # read and written (the per-chunk slots between the two kernels are not
                    # algorithmic bytes); its flops against the bf16 tensor peak beside it
                    nbytes = gdn2_min_bytes(wl)
                    gbs = nbytes / (ms * 1e-3) / 1e9
                    roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": gbs / peaks["hbm_gbs"], "traffic": None, "bytes_per_launch": nbytes,
                            "tensor_frac": tf / peaks["bf16_tflops"], "flops_per_launch": flops,
                            "kernel": "gdn2_tc_prep_kernel (warp-level bf16 MMAs) + gdn2_tc_scan_kernel (tcgen05)"}
                else:
                    roof = {"bound": "alu", "achieved": tf, "peak": fp32_peak, "unit": "TFLOP/s",
                            "frac": tf / fp32_peak, "traffic": None,
                            "kernel": "gdn2_%s_kernel (fp32 SIMT)" % mode, "flops_per_launch": flops,
                            "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 x median SM clock"}
                modes[mode] = {"value": wl.B * wl.T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
                               "roofline": roof}
            out[wl.name] = {"workload": wl.describe(), **modes}
        else:
            S = S0.clone()
            ms = timed(lambda: mlstm.gdn2_fwd(q, k, v, g, b, w, S, o=o, S_out=S))
            nbytes = 2 * wl.B * wl.H * wl.K * wl.V * 4 + wl.B * wl.H * (2 * wl.K * esz + 2 * wl.K * 4 + wl.V * (2 * esz + 4))
            gbs = nbytes / (ms * 1e-3) / 1e9
            out[wl.name] = {"workload": wl.describe(), "value": gbs, "unit": "GB/s", "ms_per_step": ms,
                            "tokens_per_s": wl.B / (ms * 1e-3),
                            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                         "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                                         "kernel": "gdn2_step_kernel (T = 1, state in place)",
                                         "bytes_per_launch": nbytes}}
    out["steps"] = steps
    return out


def gdn2_over_ranks(gdn2, world, sm_mhz):
    """The GDN-2 leg's numbers as the job's: each time is the slowest rank's (every rank runs
    the same leg, so the all-reduces line up), throughputs summed over ranks, and the fp32
    peak taken at the clock seen during the run."""
    out = dict(gdn2)
    for name, val in gdn2.items():
        if not isinstance(val, dict):
            continue
        val = dict(val)
        entries = [(mode, dict(val[mode])) for mode in ("recurrent", "chunk") if mode in val]
        if not entries:  # decode: one entry at the top level
            entries = [(None, val)]
        for mode, e in entries:
            ms_max = dist_max(e["ms_per_step"], world)
            scale = e["ms_per_step"] / ms_max
            e["ms_per_step"] = ms_max
            e["value"] = e["value"] * scale * world
            if "tokens_per_s" in e:
                e["tokens_per_s"] = e["tokens_per_s"] * scale * world
            r = dict(e["roofline"])
            if r["bound"] == "alu":
                r["peak"] = fp32_simt_peak_tflops(sm_mhz)
            r["achieved"] = r["achieved"] * scale
            r["frac"] = r["achieved"] / r["peak"]
            if "tensor_frac" in r:
                r["tensor_frac"] = r["tensor_frac"] * scale
            e["roofline"] = r
            if mode is None:
                val = e
            else:
                val[mode] = e
        out[name] = val
    return out


def backward_uses_cluster(dtype, dk, dv):
    """Whether mlstm_bwd runs the cluster kernel (warp-level bf16 MMAs) for these block widths
    (the library's rule): bf16; key width 64 / 128 / 256 or narrower (a multiple of 8, padded);
    value width a multiple of 64 up to 512, or narrower (a multiple of 8) with keys at most 64."""
    if dtype != "bf16":
        return False
    if dk not in (64, 128, 256) and not (dk < 64 and dk % 8 == 0):
        return False
    if dv < 64:
        return dv % 8 == 0 and dk <= 64
    return dv % 64 == 0 and dv <= 512


def backward_line(w, ms, sm_mhz, cpu: bool, peaks=None):
    step_ms = statistics.median(ms)
    flops = backward_flops(w.B, w.NH, w.S, w.dk, w.dv, w.num_blocks)
    tf = flops / (step_ms * 1e-3) / 1e12
    if backward_uses_cluster(w.dtype, w.dk, w.dv):
        peak = (peaks or FALLBACK_PEAKS)["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                "traffic": None, "kernel": "bwd_cluster_kernel (warp-level bf16 MMAs, a cluster of dv/64 CTAs per head)",
                "flops_per_launch": flops, "peak_source": "bf16 tensor peak (burst)"}
    else:
        peak = fp32_simt_peak_tflops(sm_mhz)
        roof = {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                "traffic": None, "kernel": "bwd_kernel (SIMT, one CTA per head)", "flops_per_launch": flops,
                "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 x median SM clock"}
    out = {"workload": w.describe(), "value": w.B * w.S / (step_ms * 1e-3), "unit": "tokens/s",
           "ms_per_step": step_ms, "steps": len(ms), "dtype": "f32 (inputs " + w.dtype + ")", "roofline": roof}
    if cpu:
        tokens = min(w.S, 64)
        heads = min(w.NH, 2)
        secs, done = oracle_backward_sample(w, tokens, heads)
        out["cpu_baseline"] = {"value": done / secs, "unit": "tokens/s (one sequence)", "cores": 1,
                               "kind": "oracle",
                               "sample": f"first {tokens} positions of {heads} (batch, head) sequences of "
                                         f"{w.describe()}, fp64 reverse-mode sequential recurrence"}
    return out


def forward_leg(w, steps, warmup, clocks, peaks, world, cpu: bool):
    """The chunkwise prefill on one of the smaller workloads (block-diagonal, retention): step
    time (every kernel of the call) with L2 flushed between steps, the roofline of the whole
    step against HBM (these workloads are HBM-bound: their intensity is far below the ridge)
    with the tensor fraction beside it, e2e through the API with host buffers, and the oracle
    on a bounded sample."""
    cw = run_chunkwise(w, steps, warmup, 256 << 20, clocks)
    step_ms = dist_max(statistics.mean(cw["step_ms"]), world)
    main_ms = statistics.mean(cw["main_ms"])
    esz = 2 if w.dtype == "bf16" else 4
    flops = chunkwise_flops(w.B, w.NH, w.S, w.dk, w.dv, w.chunk, w.num_blocks, w.retention)
    mbytes = chunkwise_min_bytes(w.B, w.NH, w.S, w.DHQK, w.DHV, esz, w.num_blocks, w.retention)
    e2e_ms, h2d, d2h = run_chunkwise_e2e(w, max(8, steps // 2), cw["tensors"])
    e2e_ms = dist_max(e2e_ms, world)
    del cw["tensors"]
    gbs = mbytes / (step_ms * 1e-3) / 1e9
    tf = flops / (step_ms * 1e-3) / 1e12
    tc = cw["plan"]["tensor_core"]
    out = {"workload": w.describe(), "value": w.B * w.S * world / (step_ms * 1e-3), "unit": "tokens/s",
           "ms_per_step": step_ms, "steps": steps, "plan": cw["plan"],
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                        "kernel": "whole prefill call (" + ("gate prep, segment summaries, tcgen05 walk"
                                                            if tc else "gate prep, SIMT walk") + ")",
                        "min_bytes_per_launch": mbytes, "walk_ms": main_ms,
                        "tc_achieved_tflops": tf, "tc_frac": tf / peaks["bf16_tflops"], "flops_per_launch": flops},
           "e2e": {"value": w.B * w.S * world / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h}}
    if cpu:
        cb = cpu_baseline(w, budget_s=6.0)
        out["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
    return out


def _r(x, digits=3):
    """x rounded to `digits` significant digits (for the compact summary)."""
    if x is None or not isinstance(x, (int, float)) or x == 0:
        return x
    import math
    return round(x, -int(math.floor(math.log10(abs(x)))) + digits - 1)


def compact_legs(line):
    """Key figures of every leg, short: the headline line ends with them, so that a log that
    keeps only the end of the output still shows each leg's number and roofline fraction."""
    legs = {}
    if "decode" in line:
        d = line["decode"]
        legs["decode"] = {"GB/s": _r(d["value"]), "hbm": _r(d["roofline"]["frac"]), "ms": _r(d["ms_per_step"])}
    for key, name in (("fwd_blockdiag", "fwd_blockdiag"), ("fwd_retention", "fwd_retention")):
        if key in line:
            e = line[key]
            legs[name] = {"tok/s": _r(e["value"]), "ms": _r(e["ms_per_step"]), "hbm": _r(e["roofline"]["frac"]),
                          "tc": _r(e["roofline"]["tc_frac"])}
    if "reversed" in line:
        legs["reversed"] = {"tok/s": _r(line["reversed"]["value"]), "ms": _r(line["reversed"]["ms_per_step"])}
    for e in line.get("backward", []):
        legs["bwd_" + e["workload"].split(":")[0]] = {"tok/s": _r(e["value"]), "ms": _r(e["ms_per_step"]),
                                                       e["roofline"]["bound"]: _r(e["roofline"]["frac"])}
    for e in line.get("scalar_normaliser", []):
        legs["scalar_norm_" + e["workload"].split(":")[0]] = {"tok/s": _r(e["value"]), "ms": _r(e["ms_per_step"]),
                                                              e["roofline"]["bound"]: _r(e["roofline"]["frac"])}
    if "msr_block" in line:
        e = line["msr_block"]
        legs["msr_block"] = {"tok/s": _r(e["value"]), "ms": _r(e["ms_per_step"]), "fwd_ms": _r(e["forward_ms"])}
    g = line.get("gdn2", {})
    for name, val in g.items():
        if not isinstance(val, dict):
            continue
        for mode in ("recurrent", "chunk"):
            if mode in val:
                r = val[mode]["roofline"]
                legs[f"gdn2_{mode}"] = {"tok/s": _r(val[mode]["value"]), "ms": _r(val[mode]["ms_per_step"]),
                                        r["bound"]: _r(r["frac"])}
        if "recurrent" not in val and "roofline" in val:
            legs["gdn2_decode"] = {"GB/s": _r(val["value"]), "hbm": _r(val["roofline"]["frac"])}
    return legs


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=3, help="chunkwise workload index (default 3)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--legs", choices=["both", "chunkwise", "decode", "backward", "msr", "gdn2", "forward"],
                    default="both", help="run only one leg (for profiling); the default runs all of them")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.legs == "chunkwise":
        args.no_decode = True

    from linear_recurrent_token_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    wd = inputs.WORKLOADS[4]
    if args.impl == "reference":
        rank, world, local = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), 0
    else:
        rank, world, local = dist_setup(args.gpus)
    config = {"workload": w.describe(), "decode_workload": wd.describe(), "global_batch": w.B * world,
              "seq_len": w.S, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
              "l2": "flushed between chunkwise steps (256 MiB write, then a 256 MiB read); decode state (512 MiB) exceeds L2"}

    if args.impl == "reference":
        if rank != 0:
            return
        cb = cpu_baseline(w, budget_s=min(120.0, 6.0 * args.steps), steps=args.steps)
        line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": cb["ms_per_step"],
                "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    assert torch.cuda.is_available(), "bench.py --impl ours needs a CUDA device"
    torch.cuda.set_device(local)
    from linear_recurrent_token_b200 import mlstm
    mlstm.lib()
    peaks, peak_src = load_peaks()
    clocks = ClockSampler(local)
    clocks.start()
    try:
        dist_barrier(world)
        torch.cuda.synchronize()
        if args.legs == "backward":
            for idx in (1, 2, 3):
                wb = inputs.WORKLOADS[idx]
                ms = run_backward(wb, args.steps, args.warmup, 256 << 20, clocks)
                if rank == 0:
                    print(json.dumps({"leg": "backward", "workload": wb.describe(), "ms_per_step": statistics.median(ms)}))
            return
        if args.legs == "gdn2":
            r = run_gdn2(args.steps, args.warmup, 256 << 20, peaks, clocks.summary().get("sm_mhz"))
            if rank == 0:
                print(json.dumps({"leg": "gdn2", **r}))
            return
        if args.legs == "msr":
            r = run_msr(inputs.WORKLOADS[2], args.steps, args.warmup, 256 << 20, peaks["hbm_gbs"])
            if rank == 0:
                print(json.dumps({"leg": "msr", "workload": inputs.WORKLOADS[2].describe(), **r}))
            return
        if args.legs == "forward":
            for idx in (1, 2):
                r = forward_leg(inputs.WORKLOADS[idx], args.steps, args.warmup, clocks, peaks, world, False)
                if rank == 0:
                    print(json.dumps({"leg": "forward", **r}))
            return
        if args.legs == "decode":
            dec = run_decode(wd, args.steps, args.warmup, clocks)
            ms = dist_max(statistics.mean(dec["step_ms"]), world)
            dbytes = decode_step_bytes(wd.B, wd.NH, wd.DHQK, wd.DHV, 2, wd.num_blocks)
            if rank == 0:
                print(json.dumps({"leg": "decode", "ms_per_step": ms, "GB/s": dbytes / (ms * 1e-3) / 1e9}))
            return
        cw = run_chunkwise(w, args.steps, args.warmup, 256 << 20, clocks)
        dist_barrier(world)
        torch.cuda.synchronize()
        step_ms = statistics.mean(cw["step_ms"])
        main_ms = statistics.mean(cw["main_ms"])
        slow_ms = dist_max(step_ms, world)
        tokens = w.B * w.S * world
        value = tokens / (slow_ms * 1e-3)
        flops = chunkwise_flops(w.B, w.NH, w.S, w.dk, w.dv, w.chunk, w.num_blocks, w.retention)
        mbytes = chunkwise_min_bytes(w.B, w.NH, w.S, w.DHQK, w.DHV, 2 if w.dtype == "bf16" else 4,
                                     w.num_blocks, w.retention)
        achieved_tf = flops / (main_ms * 1e-3) / 1e12
        e2e_ms, h2d, d2h = run_chunkwise_e2e(w, max(8, args.steps // 2), cw["tensors"])
        e2e_ms = dist_max(e2e_ms, world)
        del cw["tensors"]
        torch.cuda.empty_cache()
        dec = None
        if not args.no_decode:
            dist_barrier(world)
            dec = run_decode(wd, args.steps * 5, args.warmup, clocks)
            dist_barrier(world)
        fwd_small = {}
        if args.legs == "both":
            for key, idx in (("fwd_blockdiag", 1), ("fwd_retention", 2)):
                dist_barrier(world)
                fwd_small[key] = forward_leg(inputs.WORKLOADS[idx], args.steps, args.warmup, clocks, peaks, world,
                                             rank == 0 and world == 1 and not args.no_cpu_baseline)
        rev_ms = None
        if args.legs == "both":
            rev_ms = run_reversed(w, max(3, args.steps // 4), args.warmup, 256 << 20)
        gdn2 = None
        if args.legs == "both":
            gdn2 = run_gdn2(max(3, args.steps // 4), args.warmup, 256 << 20, peaks, None)
        msr = None
        if args.legs in ("both", "msr"):
            msr = (inputs.WORKLOADS[2], run_msr(inputs.WORKLOADS[2], max(3, args.steps // 2), args.warmup, 256 << 20,
                                                 peaks["hbm_gbs"]))
        sn = []
        if args.legs == "both":
            for idx in (1, 3):
                wn = inputs.WORKLOADS[idx]
                sn.append((wn, run_scalar_normaliser(wn, max(3, args.steps // 4), args.warmup, 256 << 20)))
        bwd = []
        if not args.no_backward and args.legs == "both":
            for idx in (1, 2, 3):
                wb = inputs.WORKLOADS[idx]
                bwd.append((wb, run_backward(wb, max(3, args.steps // 4), args.warmup, 256 << 20, clocks)))
            dist_barrier(world)
    finally:
        clocks.stop()
    launches = cw["plan"]["kernels"] * args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": slow_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": config,
        "roofline": {"bound": "tensor", "achieved": achieved_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved_tf / peaks["bf16_tflops"],
                     "step_frac": flops / (slow_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                     "traffic": recorded_traffic("tc_walk", w.name) if cw["plan"]["tensor_core"] else None,
                     "kernel": "chunkwise walk" + (" (tcgen05)" if cw["plan"]["tensor_core"] else " (SIMT)")
                               + ", timed alone (events around it keep it from overlapping the segment summaries)",
                     "kernel_ms": main_ms, "flops_per_launch": flops, "peak_source": f"{peak_src} bf16 burst",
                     "hbm_frac": mbytes / (main_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "min_bytes_per_launch": mbytes},
        "e2e": {"value": w.B * w.S * world / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "plan": cw["plan"],
        "clocks": clocks.summary(),
    }
    if dec is not None:
        dms = statistics.mean(dec["step_ms"])
        dms_max = dist_max(dms, world)
        dbytes = decode_step_bytes(wd.B, wd.NH, wd.DHQK, wd.DHV, 2, wd.num_blocks)
        gbs = dbytes * world / (dms_max * 1e-3) / 1e9
        per_rank_gbs = dbytes / (dms * 1e-3) / 1e9
        line["decode"] = {
            "value": gbs, "unit": "GB/s", "ms_per_step": dms_max, "steps": len(dec["step_ms"]),
            "tokens_per_s": wd.B * world / (dms_max * 1e-3),
            "roofline": {"bound": "hbm", "achieved": per_rank_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": per_rank_gbs / peaks["hbm_gbs"], "traffic": recorded_traffic("step", wd.name),
                         "kernel": "step_kernel<256>",
                         "bytes_per_launch": dbytes, "peak_source": f"{peak_src} copy bandwidth"},
            "e2e": {"value": wd.B * world / (dec["e2e_ms"] * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": dec["h2d"], "d2h_bytes_per_step": dec["d2h"]},
        }
        line["gpu_launches"] += len(dec["step_ms"])
    for key, r in fwd_small.items():
        line[key] = r
        line["gpu_launches"] += r["steps"] * r["plan"]["kernels"]
    if rev_ms:
        rms = dist_max(statistics.median(rev_ms), world)
        tc = cw["plan"]["tensor_core"]
        esz = 2 if w.dtype == "bf16" else 4
        copy_bytes = 0 if tc else 2 * w.B * w.NH * w.S * ((2 * w.DHQK + 2 * w.DHV) * esz + (0 if w.retention else 8))
        line["reversed"] = {"workload": w.describe(), "value": w.B * w.S * world / (rms * 1e-3), "unit": "tokens/s",
                            "ms_per_step": rms, "steps": len(rev_ms), "forward_ms": slow_ms,
                            "note": ("the tensor-core kernels reading the chunks and their rows backwards in place"
                                     if tc else "the forward kernels on reversed copies of q, k, v and the gates, h "
                                                "reversed back"),
                            "reversal_bytes": copy_bytes}
        line["gpu_launches"] += len(rev_ms) * (cw["plan"]["kernels"] + (0 if tc else (4 if w.retention else 6)))
    if gdn2:
        line["gdn2"] = gdn2_over_ranks(gdn2, world, line["clocks"].get("sm_mhz"))
        line["gpu_launches"] += gdn2["steps"] * 4  # recurrent, chunk prep + scan, decode step
    if msr:
        wm, r = msr
        bms = dist_max(r["block_ms"], world)
        line["msr_block"] = {"workload": wm.describe(), "value": wm.B * wm.S * world / (bms * 1e-3), "unit": "tokens/s",
                             "ms_per_step": bms, **{k: v for k, v in r.items() if k != "block_ms"},
                             "note": "rotation of q and k, the recurrence, GroupNorm + SiLU gate (three kernels "
                                     "in sequence), against the plain forward (forward_ms) on the same inputs"}
        line["gpu_launches"] += r["steps"] * (cw["plan"]["kernels"] + 2) + r["steps"] * (cw["plan"]["kernels"] + 2)
    if sn:
        sm_mhz = line["clocks"].get("sm_mhz")
        line["scalar_normaliser"] = []
        for wn, ms in sn:
            nms = dist_max(statistics.median(ms), world)
            flops = chunkwise_flops(wn.B, wn.NH, wn.S, wn.dk, wn.dv, wn.chunk, wn.num_blocks, False)
            tf = flops / (nms * 1e-3) / 1e12
            import torch

            from linear_recurrent_token_b200 import mlstm
            tdn = torch.bfloat16 if wn.dtype == "bf16" else torch.float32
            tc = mlstm.plan(mlstm.fwd_params(wn.B, wn.NH, wn.S, wn.DHQK, wn.DHV, wn.chunk, wn.num_blocks, tdn,
                                             False))["tensor_core"] == 1
            if tc:  # the scalar-normaliser walk on the tensor cores: flops against the bf16 peak
                peak = peaks["bf16_tflops"]
                roof = {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                        "traffic": None, "kernel": "whole call (gate prep, segment summaries, tcgen05 walk with "
                        "the scalar normaliser)", "flops_per_launch": flops, "peak_source": "measured bf16 burst"}
            else:
                peak = fp32_simt_peak_tflops(sm_mhz)
                roof = {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                        "traffic": None, "kernel": "SIMT chunkwise walk, scalar normaliser",
                        "flops_per_launch": flops,
                        "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 x median SM clock"}
            line["scalar_normaliser"].append({
                "workload": wn.describe(), "value": wn.B * wn.S * world / (nms * 1e-3), "unit": "tokens/s",
                "ms_per_step": nms, "steps": len(ms), "roofline": roof})
            line["gpu_launches"] += len(ms) * 2
    if bwd:
        sm_mhz = line["clocks"].get("sm_mhz")
        line["backward"] = [backward_line(wb, ms, sm_mhz, rank == 0 and world == 1 and not args.no_cpu_baseline, peaks)
                            for wb, ms in bwd]
        line["gpu_launches"] += sum(len(ms) for _, ms in bwd)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(w)
        line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
    if rank == 0:
        # every leg in full on one line, then the headline line, which ends with the key
        # figures of each leg (so that the end of the output carries all of them)
        standard = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                    "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "clocks", "e2e",
                    "gpu_launches")
        print(json.dumps({"detail": {k: v for k, v in line.items() if k not in standard}}))
        head = {k: line[k] for k in standard if k in line}
        head["legs"] = compact_legs(line)
        print(json.dumps(head))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
