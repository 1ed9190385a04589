#!/usr/bin/env python
"""Throughput of the gated delta rule forward pass on B200, through the C ABI.

One bench "step" is one chunked prefill (the whole prefill path: gates, q/k
normalisation, intra-chunk UT transform, inter-chunk state passing, outputs and
final state) over the prefill workload: B=1, T=8192, Hk=Hv=48, dk=dv=128, chunk 32,
bf16 q/k/v/a/b, fp32 state and fp32 outputs.  ``value`` is prefill tokens/s over all
ranks.  The decode path is timed beside it on the decode workload (B=64, Hk=Hv=48,
dk=dv=128, 256 consecutive in-place steps) and reported under ``decode`` as steps/s
and state GB/s, with its own roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 the script runs under torchrun (one process per GPU): every rank runs the
same per-GPU workload on its own seeded data (weak scaling; the units -- sequences
x heads -- are independent, so there is no data-path collective), and the timing is
the max over ranks.  ``--impl reference`` times the fp64 CPU oracle on a bounded
sample of the same workload (rank 0 only) and prints the same JSON line.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDR prefill tokens/s & decode state GB/s (Hv=48, dk=dv=128) vs roofline"
PREFILL = dict(B=1, T=8192, Hk=48, Hv=48, dk=128, dv=128, chunk=32)
DECODE = dict(B=64, Hk=48, Hv=48, dk=128, dv=128, steps=256)
PREFILL_NAME = "chunked prefill B=1 T=8192 Hk=Hv=48 dk=dv=128 chunk=32 (bf16 in, fp32 state/out)"
DECODE_NAME = "decode B=64 Hk=Hv=48 dk=dv=128, 256 in-place steps (bf16 in, fp32 state/out)"


# ----------------------------------------------------------------- algorithmic counts


def prefill_alg_bytes(B, T, Hk, Hv, dk, dv, **_):
    """HBM bytes a prefill must move at least: bf16 q, k, v, a, b in; fp32 o and final
    state out (zero initial state, nothing read for it)."""
    tok = B * T
    return tok * (2 * Hk * dk * 2 + Hv * dv * 2 + 2 * Hv * 2 + Hv * dv * 4) + B * Hv * dk * dv * 4


def prefill_alg_flops(B, T, Hk, Hv, dk, dv, chunk, **_):
    """Flops of the chunked form per token-head: 6 dk dv for W S, Q S and K^T Delta
    (two flops per MAC) plus ~5 C d for the chunk-local triangles (K K^T, Q K^T, the
    solve, U, P Delta), each triangle counted once."""
    d = dk
    return B * T * Hv * (6 * dk * dv + 5 * chunk * d)


def decode_alg_bytes(B, Hk, Hv, dk, dv, **_):
    """Per step: the fp32 state read and written once, bf16 inputs in, fp32 o out."""
    return B * Hv * dk * dv * 4 * 2 + B * (2 * Hk * dk * 2 + Hv * dv * 2 + 2 * Hv * 2 +
                                           Hv * dv * 4)


def decode_state_bytes(B, Hv, dk, dv, **_):
    return B * Hv * dk * dv * 4 * 2


# ----------------------------------------------------------------------- environment


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, source="fallback")


def kernel_source_hash(name, text=None):
    """Hash of a kernel source's code: comments and layout removed, so that the recorded
    traffic stays tied to the code it was measured on, not to its commentary."""
    if text is None:
        with open(os.path.join(ROOT, "gated_delta_rule_145_b200", "csrc", name)) as f:
            text = f.read()
    import re

    code = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)  # block comments
    code = re.sub(r"//[^\n]*", " ", code)                 # line comments
    code = " ".join(code.split())                           # layout
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def recorded_traffic(kernel_file):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current source of that kernel (profiles/dram_traffic.txt: file, hash, bytes)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        want = kernel_source_hash(kernel_file)
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel_file \
                        and parts[1] == want:
                    return float(parts[2])
    except OSError:
        pass
    return None


class ClockSampler:
    """nvidia-smi sampled every 100 ms in the background; summary of the samples taken
    inside the marked timed windows."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id):
        self.samples = []
        self.windows = []
        self.proc = None
        self.gpu_id = gpu_id
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu_id)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        def inside(t):
            return any(a - 0.15 <= t <= b + 0.15 for a, b in self.windows)

        rows = [s for t, s in self.samples if inside(t)] or [s for _, s in self.samples]
        sm, mx, reasons = [], [], set()
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(self.REASONS, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=[], samples=0)
        return dict(sm_mhz=statistics.median(sm), sm_max_mhz=max(mx), reasons=sorted(reasons),
                    samples=len(sm))


def gpu_smi_id(dev):
    import torch

    try:
        p = torch.cuda.get_device_properties(dev)
        return "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[dev] if vis else str(dev)


# ------------------------------------------------------------------ distributed plumbing


class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend):
        if self.world > 1:
            import torch.distributed as dist

            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x, device=None):
        if not self.pg:
            return x
        import torch

        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ------------------------------------------------------------------------ our arm


def _timed(dist, dev, stream, sampler, fn, n):
    """Run fn() n times between a barrier + synchronize on both sides; returns the max
    over ranks of the device time (ms) measured with CUDA events on `stream`."""
    import torch

    r0 = torch.cuda.Event(enable_timing=True)
    r1 = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    r0.record(stream)
    for i in range(n):
        fn(i)
    r1.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    sampler.mark(t_wall0, time.time())
    return dist.max(r0.elapsed_time(r1), dev)


def bench_prefill(args, dist, dev, stream, sampler, P, gdr, synth):
    import torch

    inp = synth.make_inputs(P["B"], P["T"], P["Hk"], P["Hv"], P["dk"], P["dv"], "bf16",
                            seed=1002 + 1000 * dist.rank)

    def dev_bf16(x):
        return torch.from_numpy(x).to(dev).to(torch.bfloat16)

    q, k, v, a, b = (dev_bf16(getattr(inp, n)) for n in ("q", "k", "v", "a", "b"))
    A_log = torch.from_numpy(inp.A_log).to(dev)
    dt_bias = torch.from_numpy(inp.dt_bias).to(dev)
    out = torch.empty((P["B"], P["T"], P["Hv"], P["dv"]), device=dev, dtype=torch.float32)
    fin = torch.empty((P["B"], P["Hv"], P["dk"], P["dv"]), device=dev, dtype=torch.float32)

    def launch(qq, kk, vv, aa, bb):
        gdr.gdr_prefill_chunked(qq, kk, vv, aa, bb, A_log, dt_bias, None, out, fin, None,
                                P["B"], P["T"], P["Hk"], P["Hv"], P["dk"], P["dv"], P["chunk"],
                                stream=stream)

    for _ in range(args.warmup):
        launch(q, k, v, a, b)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]

    def step(i):
        ev[i][0].record(stream)
        launch(q, k, v, a, b)
        ev[i][1].record(stream)

    region_ms = _timed(dist, dev, stream, sampler, step, args.steps)
    # two kernels per call: intra-chunk, then state passing
    res = dict(inp=inp, region_ms=region_ms, launches=2 * args.steps,
               kernel_ms=statistics.mean(s.elapsed_time(e) for s, e in ev),
               kernel_ms_median=statistics.median(s.elapsed_time(e) for s, e in ev))
    # the same call timed with the L2 flushed before each call (a 256 MB write between
    # calls, outside the events): the median per call
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    fl = []
    for i in range(max(5, min(args.steps, 20))):
        flush.fill_(i & 255)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        launch(q, k, v, a, b)
        e1.record(stream)
        fl.append((e0, e1))
    torch.cuda.synchronize(dev)
    res["flushed_median_ms"] = statistics.median(s.elapsed_time(e) for s, e in fl)
    res["launches"] += 2 * len(fl)
    del flush
    # the erase=False form (gated linear attention) on the same inputs and kernels
    def gla(_i):
        gdr.gdr_gla_prefill_chunked(q, k, v, a, b, A_log, dt_bias, None, out, fin, None,
                                    P["B"], P["T"], P["Hk"], P["Hv"], P["dk"], P["dv"],
                                    P["chunk"], stream=stream)

    for i in range(3):
        gla(i)
    gla_steps = max(3, min(args.steps, 10))
    res.update(gla_ms=_timed(dist, dev, stream, sampler, gla, gla_steps), gla_steps=gla_steps,
               launches=res["launches"] + 2 * gla_steps)
    # the steps around the rule at the same sizes: conv + SiLU over the q|k|v channels of
    # every token, gated RMSNorm over every (token, head) row of the rule's output
    C = 2 * P["Hk"] * P["dk"] + P["Hv"] * P["dv"]
    g = torch.Generator(device=dev).manual_seed(7)
    xc = torch.randn((P["B"], P["T"], C), device=dev, generator=g).to(torch.bfloat16)
    yc = torch.empty_like(xc)
    wc = torch.randn((C, 4), device=dev, generator=g) * 0.5
    bc = torch.randn((C,), device=dev, generator=g) * 0.1
    sc = torch.zeros((P["B"], C, 3), device=dev)
    zr = torch.randn(out.shape, device=dev, generator=g).to(torch.bfloat16)
    wr = torch.rand((P["dv"],), device=dev, generator=g) + 0.5
    yr = torch.empty_like(out)
    rows = P["B"] * P["T"] * P["Hv"]

    def conv(_i):
        gdr.gdr_short_conv_silu(xc, wc, bc, sc, sc, yc, P["B"], P["T"], C, stream=stream)

    def norm(_i):
        gdr.gdr_gated_rmsnorm(out, zr, wr, yr, rows, P["dv"], 1e-6, stream=stream)

    io = {}
    for name, fn, nbytes in (("conv_silu", conv, 2 * xc.numel() * 2 + sc.numel() * 8),
                             ("gated_rmsnorm", norm, out.numel() * (4 + 2 + 4))):
        for i in range(3):
            fn(i)
        ms = _timed(dist, dev, stream, sampler, fn, 10) / 10
        io[name] = dict(ms=ms, bytes=nbytes)
    res.update(mixer_io=io, launches=res["launches"] + 20)
    if args.no_e2e:
        return res
    # ---- end to end through the public API: the C-ABI call with pinned HOST buffers
    # (gdr_prefill_chunked_host copies the inputs in and the outputs back in segments,
    # overlapped with the kernels; all of it inside the timed region)
    host = {n: torch.from_numpy(getattr(inp, n)).to(torch.bfloat16).pin_memory()
            for n in ("q", "k", "v", "a", "b")}
    A_h = torch.from_numpy(inp.A_log).pin_memory()
    dt_h = torch.from_numpy(inp.dt_bias).pin_memory()
    out_h = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    fin_h = torch.empty(fin.shape, dtype=torch.float32).pin_memory()
    seg_h = (max(256, -(-P["T"] // 8)) + 31) // 32 * 32  # the call's default segment
    nseg_h = -(-P["T"] // seg_h)
    last = P["T"] - (nseg_h - 1) * seg_h  # the call cuts its last segment in two, twice
    for _ in range(2):
        if nseg_h < 2 or last // 2 // 32 * 32 < 128:
            break
        last -= last // 2 // 32 * 32
        nseg_h += 1

    def e2e(_i):
        gdr.gdr_prefill_chunked_host(host["q"], host["k"], host["v"], host["a"], host["b"], A_h,
                                     dt_h, None, out_h, fin_h, P["B"], P["T"], P["Hk"], P["Hv"],
                                     P["dk"], P["dv"], P["chunk"], 0, stream=stream)

    e2e_steps = max(3, min(args.steps, 20))
    for i in range(min(args.warmup, 3)):
        e2e(i)
    e2e_ms = _timed(dist, dev, stream, sampler, e2e, e2e_steps)
    res.update(e2e_steps=e2e_steps, e2e_ms=e2e_ms,
               launches=res["launches"] + 2 * nseg_h * e2e_steps,
               h2d=sum(t.numel() * t.element_size() for t in host.values()) + 8 * P["Hv"],
               d2h=out_h.numel() * 4 + fin_h.numel() * 4)
    return res


def bench_decode(args, dist, dev, stream, sampler, gdr, synth):
    import torch

    D = DECODE
    dinp = synth.make_inputs(D["B"], D["steps"], D["Hk"], D["Hv"], D["dk"], D["dv"], "bf16",
                             seed=1001 + 1000 * dist.rank, s0_std=0.02)

    def steps_first(x):
        return torch.from_numpy(np.ascontiguousarray(np.swapaxes(x, 0, 1))).to(dev).to(
            torch.bfloat16)

    dq, dk_, dv_, da, db = (steps_first(getattr(dinp, n)) for n in ("q", "k", "v", "a", "b"))
    dA = torch.from_numpy(dinp.A_log).to(dev)
    ddt = torch.from_numpy(dinp.dt_bias).to(dev)
    state = torch.from_numpy(dinp.init_state).to(dev)
    dout = torch.empty((D["B"], D["Hv"], D["dv"]), device=dev, dtype=torch.float32)
    passes = max(1, min(args.steps, 10))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(D["steps"])]

    def one_pass(_pi, record=False):
        for t in range(D["steps"]):
            if record:
                ev[t][0].record(stream)
            gdr.gdr_decode_step(dq[t], dk_[t], dv_[t], da[t], db[t], dA, ddt, state, dout,
                                D["B"], D["Hk"], D["Hv"], D["dk"], D["dv"], stream=stream)
            if record:
                ev[t][1].record(stream)

    for _ in range(max(1, args.warmup // 2)):
        one_pass(0)
    # the timed passes launch the steps back to back (an event pair around every launch
    # would add its own gap to each step); the average launch duration is the timed
    # region over the launches in it
    ms = _timed(dist, dev, stream, sampler, one_pass, passes)
    steps = passes * D["steps"]
    # one more pass, untimed, with an event pair per launch, for the per-launch spread
    one_pass(0, record=True)
    torch.cuda.synchronize(dev)
    per = [s.elapsed_time(e) for s, e in ev]
    return dict(ms=ms, steps=steps, kernel_ms=ms / steps,
                launch_ms_events=statistics.median(per))


def bench_varlen(args, dist, dev, stream, sampler, gdr, synth):
    """The grouped-key varlen prefill: 8 packed sequences with seeded lengths U[256, 4096],
    Hk=16 key heads shared by Hv=48 value heads, d=128, chunk 32 (mean per call)."""
    import torch

    inp = synth.workload(3, seed=1003 + 1000 * dist.rank)
    d = {n: torch.from_numpy(getattr(inp, n)).to(dev).to(torch.bfloat16)
         for n in ("q", "k", "v", "a", "b")}
    A_log = torch.from_numpy(inp.A_log).to(dev)
    dt_bias = torch.from_numpy(inp.dt_bias).to(dev)
    cu = torch.from_numpy(inp.cu_seqlens).to(dev)
    T, nseq = inp.q.shape[1], inp.nseq
    Hk, Hv = inp.q.shape[2], inp.v.shape[2]
    out = torch.empty((1, T, Hv, 128), device=dev)
    fin = torch.empty((nseq, Hv, 128, 128), device=dev)
    n = max(5, min(args.steps, 20))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]

    def call(i):
        ev[i][0].record(stream)
        gdr.gdr_prefill_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], A_log, dt_bias, None, out,
                                fin, cu, nseq, T, Hk, Hv, 128, 128, 32, stream=stream)
        ev[i][1].record(stream)

    for i in range(3):
        call(i)
    ms = _timed(dist, dev, stream, sampler, call, n)
    kms = statistics.mean(s.elapsed_time(e) for s, e in ev)
    alg = T * (2 * Hk * 128 * 2 + Hv * 128 * 2 + 2 * Hv * 2 + Hv * 128 * 4) + \
        nseq * Hv * 128 * 128 * 4
    lens = np.diff(inp.cu_seqlens).tolist()
    return dict(workload=f"varlen B={nseq} seqs (lengths {lens}, seeded U[256,4096]) T={T} "
                         f"Hk={Hk} Hv={Hv} d=128 chunk 32 bf16",
                tokens=T, ms=ms / n, kernel_ms=kms, alg_bytes=alg, launches=2 * (n + 3))


def bench_long(args, dist, dev, stream, sampler, gdr):
    """Long context: the chunked prefill over B=1, T=65536, Hk=Hv=48, d=128, then 512
    decode steps from its final state (seeded device-side draws of the same recipe)."""
    import torch

    g = torch.Generator(device=dev).manual_seed(1004 + 1000 * dist.rank)
    T, H, nd = 65536, 48, 512
    r = lambda *shape: torch.randn(shape, device=dev, generator=g).to(torch.bfloat16)
    x = dict(q=r(1, T + nd, H, 128), k=r(1, T + nd, H, 128), v=r(1, T + nd, H, 128),
             a=r(1, T + nd, H), b=r(1, T + nd, H))
    A_log = torch.rand((H,), device=dev, generator=g) * math.log(16.0)
    dt = torch.exp(torch.rand((H,), device=dev, generator=g) *
                   (math.log(1e-1) - math.log(1e-3)) + math.log(1e-3))
    dt_bias = torch.log(torch.expm1(dt))
    pre = {n: x[n][:, :T] for n in x}
    dec = {n: x[n][0, T:].contiguous() for n in x}  # [512, ...]: one row per step
    out = torch.empty((1, T, H, 128), device=dev)
    S = torch.empty((1, H, 128, 128), device=dev)
    dout = torch.empty((1, H, 128), device=dev)

    def prefill(_i):
        gdr.gdr_prefill_chunked(pre["q"], pre["k"], pre["v"], pre["a"], pre["b"], A_log,
                                dt_bias, None, out, S, None, 1, T, H, H, 128, 128, 32,
                                stream=stream)

    prefill(0)
    n = 3
    pms = _timed(dist, dev, stream, sampler, prefill, n) / n

    def decode(_i):
        for t in range(nd):
            gdr.gdr_decode_step(dec["q"][t], dec["k"][t], dec["v"][t], dec["a"][t], dec["b"][t],
                                A_log, dt_bias, S, dout, 1, H, H, 128, 128, stream=stream)

    dms = _timed(dist, dev, stream, sampler, decode, 1)
    # the same 512 steps captured once in a CUDA graph and replayed (a serving loop's form:
    # no host work per step); the replay continues from the state the first run left
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device=dev)
    cap.wait_stream(stream)
    with torch.cuda.graph(graph, stream=cap):
        for t in range(nd):
            gdr.gdr_decode_step(dec["q"][t], dec["k"][t], dec["v"][t], dec["a"][t],
                                dec["b"][t], A_log, dt_bias, S, dout, 1, H, H, 128, 128,
                                stream=cap)
    stream.wait_stream(cap)

    def replay(_i):
        with torch.cuda.stream(stream):
            graph.replay()

    replay(0)
    gms = _timed(dist, dev, stream, sampler, replay, 1)
    del graph
    alg = prefill_alg_bytes(1, T, H, H, 128, 128)
    return dict(workload=f"long context B=1 T={T} Hk=Hv={H} d=128 chunk 32 bf16, then {nd} "
                         "decode steps from its final state",
                prefill_ms=pms, alg_bytes=alg, decode_us_per_step=dms * 1e3 / nd,
                decode_graph_us_per_step=gms * 1e3 / nd,
                launches=2 * (n + 1) + 2 * nd)


def bench_cp(args, dist, dev, stream, sampler, gdr):
    """Context-parallel prefill (segment maps, composition, prefill from each segment's
    start state), two measurements on this GPU:
      one_gpu   -- long context with few heads (B=1, T=65536, Hk=Hv=8): the plain prefill
                   keeps 24 CTAs busy for 2048 chunk steps; gdr_prefill_chunked_cp runs 6
                   segments side by side;
      per_rank  -- one rank's share of an 8-GPU split of B=1, T=65536, Hk=Hv=48: its 8192
                   tokens' maps, the composition of 8 maps and its prefill (the all-gather
                   of 8 x 2 x 3.1 MB over NVLink is not included)."""
    import torch

    g = torch.Generator(device=dev).manual_seed(11 + dist.rank)

    def draw(T, H):
        r = lambda *shape: torch.randn(shape, device=dev, generator=g).to(torch.bfloat16)
        A_log = torch.rand((H,), device=dev, generator=g) * math.log(16.0)
        dt = torch.exp(torch.rand((H,), device=dev, generator=g) *
                       (math.log(1e-1) - math.log(1e-3)) + math.log(1e-3))
        return dict(q=r(1, T, H, 128), k=r(1, T, H, 128), v=r(1, T, H, 128), a=r(1, T, H),
                    b=r(1, T, H), A_log=A_log, dt_bias=torch.log(torch.expm1(dt)))

    def timed(fn, n=3):
        fn(0)
        return _timed(dist, dev, stream, sampler, fn, n) / n

    res = {}
    T, H, nseg = 65536, 8, 6
    x = draw(T, H)
    out = torch.empty((1, T, H, 128), device=dev)
    fin = torch.empty((1, H, 128, 128), device=dev)
    args_in = (x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"])
    plain = timed(lambda _i: gdr.gdr_prefill_chunked(*args_in, None, out, fin, None, 1, T, H, H,
                                                     128, 128, 32, stream=stream))
    cp = timed(lambda _i: gdr.gdr_prefill_chunked_cp(*args_in, None, out, fin, T, H, H, 128, 128,
                                                     32, nseg, stream=stream))
    res["one_gpu"] = dict(workload=f"B=1 T={T} Hk=Hv={H} d=128 bf16, {nseg} segments",
                          plain_ms=round(plain, 4), cp_ms=round(cp, 4),
                          cp_tokens_per_s=round(T / (cp / 1e3), 1),
                          alg_bytes=prefill_alg_bytes(1, T, H, H, 128, 128))
    del x, out
    G, Tr, H = 8, 8192, 48
    x = draw(Tr, H)
    args_in = (x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"])
    out = torch.empty((1, Tr, H, 128), device=dev)
    phi = torch.empty((1, H, 128, 128), device=dev)
    nmap = torch.empty_like(phi)
    phi_all = torch.empty((G, H, 128, 128), device=dev)
    nmap_all = torch.empty_like(phi_all)
    seg = torch.empty_like(phi_all)

    def rank_work(_i):
        gdr.gdr_prefill_segment_maps(*args_in, phi, nmap, None, 1, Tr, H, H, 128, 128, 32,
                                     stream=stream)
        phi_all.copy_(phi.expand(G, -1, -1, -1))  # stands in for the all-gather
        nmap_all.copy_(nmap.expand(G, -1, -1, -1))
        gdr.gdr_segment_combine(phi_all, nmap_all, None, seg, fin.new_empty((1, H, 128, 128)),
                                G, H, 128, 128, stream=stream)
        gdr.gdr_prefill_chunked(*args_in, seg[3:4], out, None, None, 1, Tr, H, H, 128, 128, 32,
                                stream=stream)

    per = timed(rank_work)
    res["per_rank"] = dict(workload=f"rank 3 of {G}: B=1 T={G * Tr} Hk=Hv={H} d=128 bf16, "
                                    f"{Tr} tokens per rank",
                           ms=round(per, 4),
                           implied_tokens_per_s=round(G * Tr / (per / 1e3), 1),
                           note="one rank's measured work; the exchange is not included")
    res["launches"] = 4 * 2 + 4 * 8 + 4 * 7  # plain, cp, rank work (1 warm-up + 3 each)
    return res


def run_ours(args, dist):
    import torch

    import gated_delta_rule_145_b200 as gdr
    from gated_delta_rule_145_b200 import synth

    torch.cuda.set_device(dist.local)
    dev = torch.device("cuda", dist.local)
    dist.init("nccl")
    pk = peaks()
    sampler = ClockSampler(gpu_smi_id(dist.local))
    sampler.start()
    stream = torch.cuda.current_stream(dev)
    P = dict(PREFILL)
    if args.T:
        P["T"] = args.T
    pre = dec = None
    if args.only in (None, "prefill"):
        pre = bench_prefill(args, dist, dev, stream, sampler, P, gdr, synth)
    if args.only in (None, "decode"):
        dec = bench_decode(args, dist, dev, stream, sampler, gdr, synth)
    cpx = var = lng = None
    if args.only in (None, "cp"):
        cpx = bench_cp(args, dist, dev, stream, sampler, gdr)
    if args.only in (None, "varlen"):
        var = bench_varlen(args, dist, dev, stream, sampler, gdr, synth)
    if args.only in (None, "long"):
        lng = bench_long(args, dist, dev, stream, sampler, gdr)
    sampler.stop()
    clocks = sampler.summary()

    result = None
    if dist.rank == 0:
        result = {"metric": METRIC, "n_gpus": dist.world, "steps": args.steps,
                  "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                  "vs_baseline": None, "dtype": "bf16",
                  "data": "synthetic (seeded N(0,1) bf16 q/k/v/a/b; A_log~U(0,ln16); "
                          "dt~logU(1e-3,1e-1))", "clocks": clocks, "gpu_launches": 0}
        if pre is not None:
            alg_b, alg_f = prefill_alg_bytes(**P), prefill_alg_flops(**P)
            achieved = alg_b / (pre["kernel_ms"] / 1e3) / 1e9
            cpu = None
            if dist.world == 1 and not args.no_cpu_baseline and args.only is None:
                cpu = cpu_baseline_sample(pre["inp"], seconds_hint=args.cpu_seconds)
            result.update({
                "value": round(P["B"] * P["T"] * args.steps * dist.world /
                               (pre["region_ms"] / 1e3), 1),
                "unit": "tokens/s", "ms_per_step": round(pre["region_ms"] / args.steps, 4),
                "config": {
                    "workload": PREFILL_NAME if P["T"] == PREFILL["T"] else
                    PREFILL_NAME.replace("T=8192", f"T={P['T']}"),
                    "global_batch": P["B"] * dist.world, "seq_len": P["T"],
                    "heads": P["Hv"], "head_dim": P["dk"], "chunk": P["chunk"],
                    "parallelism": f"dp{dist.world} (independent sequences x heads, "
                                   "no collective)",
                    "l2": "value and roofline: no flush between calls (inputs 302 MB and "
                          "outputs 201 MB exceed the 126 MB L2); flushed_median_ms: 256 MB "
                          "written before each call",
                },
                "roofline": {
                    "bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                    "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4),
                    "traffic": recorded_traffic("prefill_tc64.cu"), "peak_source": pk["source"],
                    "alg_bytes_per_launch": alg_b, "alg_flops_per_launch": alg_f,
                    "kernel_ms": round(pre["kernel_ms"], 4),
                    "kernel_ms_median": round(pre["kernel_ms_median"], 4),
                    "flushed_median_ms": round(pre["flushed_median_ms"], 4),
                    "frac_flushed_median": round(alg_b / (pre["flushed_median_ms"] / 1e3) /
                                                 1e9 / pk["hbm_gbs"], 4),
                    "tensor_frac": round(alg_f / (pre["kernel_ms"] / 1e3) / 1e12 /
                                         pk["bf16_tflops"], 4),
                },
                "cpu_baseline": cpu,
            })
            result["gpu_launches"] += pre["launches"]
            result["mixer_io"] = {
                name: {"ms": round(v["ms"], 4), "alg_bytes": v["bytes"],
                       "roofline": {"bound": "hbm",
                                    "achieved": round(v["bytes"] / (v["ms"] / 1e3) / 1e9, 1),
                                    "peak": pk["hbm_gbs"], "unit": "GB/s",
                                    "frac": round(v["bytes"] / (v["ms"] / 1e3) / 1e9 /
                                                  pk["hbm_gbs"], 4)}}
                for name, v in pre["mixer_io"].items()}
            result["mixer_io"]["workload"] = (
                "conv_silu: x [1, 8192, 18432] bf16 (q|k|v channels, Hk=Hv=48, d=128), "
                "4 taps, state in place; gated_rmsnorm: o [8192*48, 128] fp32, bf16 gate")
            gla_s = pre["gla_ms"] / pre["gla_steps"] / 1e3
            result["gla"] = {
                "form": "erase=False (gated linear attention), same workload and kernels",
                "value": round(P["B"] * P["T"] * dist.world / gla_s, 1), "unit": "tokens/s",
                "ms_per_step": round(pre["gla_ms"] / pre["gla_steps"], 4),
                "roofline": {"bound": "hbm", "achieved": round(alg_b / gla_s / 1e9, 1),
                             "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": round(alg_b / gla_s / 1e9 / pk["hbm_gbs"], 4)}}
            if "e2e_ms" in pre:
                result["e2e"] = {"value": round(P["B"] * P["T"] * pre["e2e_steps"] * dist.world /
                                                (pre["e2e_ms"] / 1e3), 1),
                                 "unit": "tokens/s", "h2d_bytes_per_step": pre["h2d"],
                                 "d2h_bytes_per_step": pre["d2h"], "steps": pre["e2e_steps"],
                                 "api": "gdr_prefill_chunked_host (pinned host buffers in and "
                                        "out, copies overlapped with the kernels)"}
        if dec is not None:
            D = DECODE
            dalg = decode_alg_bytes(**D)
            dach = dalg / (dec["kernel_ms"] / 1e3) / 1e9
            dtraffic = recorded_traffic("recurrent.cu")
            dcpu = None
            if dist.world == 1 and not args.no_cpu_baseline and args.only is None:
                dcpu = decode_cpu_baseline(synth, seconds_hint=args.cpu_seconds / 3)
            result["decode"] = {
                "workload": DECODE_NAME, "value": round(dec["steps"] / (dec["ms"] / 1e3), 1),
                "cpu_baseline": dcpu,
                "unit": "steps/s",
                "state_gbs": round(decode_state_bytes(**D) * dec["steps"] * dist.world /
                                   (dec["ms"] / 1e3) / 1e9, 1),
                "ms_per_step": round(dec["ms"] / dec["steps"], 5),
                "roofline": {"bound": "hbm", "achieved": round(dach, 1), "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": round(dach / pk["hbm_gbs"], 4),
                             "traffic": dtraffic,
                             "alg_bytes_per_launch": dalg,
                             "kernel_ms": round(dec["kernel_ms"], 5),
                             "kernel_ms_from": "timed region / launches (steps back to back)",
                             "launch_ms_events_median": round(dec["launch_ms_events"], 5)}}
            if dtraffic:
                # part of the updated state is still in L2 when the next step reads it:
                # the DRAM bytes the counters saw per launch, as a fraction of the peak
                result["decode"]["roofline"]["dram_frac"] = round(
                    dtraffic / (dec["kernel_ms"] / 1e3) / 1e9 / pk["hbm_gbs"], 4)
            result["gpu_launches"] += dec["steps"]
        if var is not None:
            result["gpu_launches"] += var.pop("launches")
            ach = var["alg_bytes"] / (var["kernel_ms"] / 1e3) / 1e9
            result["varlen"] = {
                "workload": var["workload"],
                "value": round(var["tokens"] * dist.world / (var["ms"] / 1e3), 1),
                "unit": "tokens/s", "ms_per_step": round(var["ms"], 4),
                "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 4),
                             "alg_bytes_per_launch": var["alg_bytes"],
                             "kernel_ms": round(var["kernel_ms"], 4)}}
        if lng is not None:
            result["gpu_launches"] += lng.pop("launches")
            ach = lng["alg_bytes"] / (lng["prefill_ms"] / 1e3) / 1e9
            result["long"] = {
                "workload": lng["workload"],
                "value": round(65536 * dist.world / (lng["prefill_ms"] / 1e3), 1),
                "unit": "tokens/s", "prefill_ms": round(lng["prefill_ms"], 4),
                "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 4),
                             "alg_bytes_per_launch": lng["alg_bytes"]},
                "decode_us_per_step": round(lng["decode_us_per_step"], 2),
                "decode_graph_us_per_step": round(lng["decode_graph_us_per_step"], 2),
                "decode_note": "B=1: 6.3 MB of state, L2-resident, launch-latency bound; "
                               "per call through the Python binding, and the same steps "
                               "replayed from one CUDA graph"}
        if cpx is not None:
            result["gpu_launches"] += cpx.pop("launches")
            one = cpx["one_gpu"]
            ach = one["alg_bytes"] / (one["cp_ms"] / 1e3) / 1e9
            one["roofline"] = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
                               "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 4)}
            result["context_parallel"] = cpx
    dist.close()
    return result


def cpu_baseline_sample(inp, seconds_hint=15.0):
    """The fp64 oracle, as it stands, on a bounded sample of the prefill workload: all 48
    heads over the first T_s tokens (T_s sized from a short probe to take ~seconds_hint)."""
    from oracle import oracle

    cores = oracle.default_threads()

    def run(Ts):
        sl = slice(0, Ts)
        t0 = time.perf_counter()
        oracle.forward(inp.q[:, sl], inp.k[:, sl], inp.v[:, sl], inp.a[:, sl], inp.b[:, sl],
                       inp.A_log, inp.dt_bias, nthreads=cores)
        return time.perf_counter() - t0

    probe = 64
    t = run(probe)
    Ts = int(min(inp.q.shape[1], max(probe, probe * seconds_hint / max(t, 1e-3))))
    t = run(Ts)
    return {"value": round(Ts / t, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 oracle, all {inp.v.shape[2]} heads, first {Ts} of {inp.q.shape[1]} "
                      f"tokens of the prefill workload, {t:.1f} s wall"}


def decode_cpu_baseline(synth, seconds_hint=5.0):
    """The fp64 oracle, as it stands, on a bounded sample of the decode workload: the first
    n of its 256 steps for all 64 sequences x 48 heads, on all host cores and on one."""
    from oracle import oracle

    D = DECODE
    inp = synth.make_inputs(D["B"], D["steps"], D["Hk"], D["Hv"], D["dk"], D["dv"], "bf16",
                            seed=1001, s0_std=0.02)
    cores = oracle.default_threads()

    def run(n, threads):
        sl = slice(0, n)
        t0 = time.perf_counter()
        oracle.forward(inp.q[:, sl], inp.k[:, sl], inp.v[:, sl], inp.a[:, sl], inp.b[:, sl],
                       inp.A_log, inp.dt_bias, inp.init_state, nthreads=threads)
        return time.perf_counter() - t0

    res = {}
    for label, threads in (("all", cores), ("one", 1)):
        t = run(1, threads)
        n = int(min(D["steps"], max(1, seconds_hint / max(t, 1e-3))))
        t = run(n, threads)
        res[label] = (n / t, n, t)
    v, n, t = res["all"]
    v1, n1, t1 = res["one"]
    return {"value": round(v, 2), "unit": "steps/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 oracle, first {n} of 256 decode steps for all 64 x 48 (sequence, "
                      f"head) states, {t:.1f} s wall",
            "one_thread": {"value": round(v1, 3), "unit": "steps/s", "cores": 1,
                           "sample": f"first {n1} steps, {t1:.1f} s wall"}}


# ----------------------------------------------------------------- reference arm


def run_reference(args, dist):
    """The oracle timed as the reference arm (rank 0 only; other ranks exit at once)."""
    if dist.rank != 0:
        return None
    from gated_delta_rule_145_b200 import synth
    from oracle import oracle

    P = PREFILL
    inp = synth.make_inputs(P["B"], P["T"], P["Hk"], P["Hv"], P["dk"], P["dv"], "bf16", seed=1002)
    cores = oracle.default_threads()
    Ts = args.ref_tokens
    sl = slice(0, Ts)
    sample = [getattr(inp, n)[:, sl] for n in ("q", "k", "v", "a", "b")]

    def step():
        oracle.forward(*sample, inp.A_log, inp.dt_bias, nthreads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = Ts * args.steps / dt
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded recipe)", "impl": "reference",
        "config": {"workload": PREFILL_NAME if Ts == P["T"] else
                   PREFILL_NAME + f" (first {Ts} tokens per step)",
                   "global_batch": P["B"], "seq_len": P["T"], "heads": P["Hv"],
                   "head_dim": P["dk"], "chunk": P["chunk"],
                   "parallelism": "host threads over (sequence, head)"},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"fp64 oracle, all 48 heads, {Ts} of {P['T']} tokens per "
                                   "step"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-tokens", type=int, default=PREFILL["T"],
                    help="tokens per reference-arm step (all 48 heads; default: the whole "
                         "prefill workload, as our arm)")
    ap.add_argument("--only", choices=("prefill", "decode", "cp", "varlen", "long"),
                    default=None,
                    help="time one path only (profiling runs; not the contract line)")
    ap.add_argument("--T", type=int, default=0, help="prefill length override (profiling)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg")
    args = ap.parse_args()
    dist = Dist()
    if dist.world != args.gpus:
        print(f"note: --gpus {args.gpus} but WORLD_SIZE={dist.world}; using WORLD_SIZE",
              file=sys.stderr)
    res = run_reference(args, dist) if args.impl == "reference" else run_ours(args, dist)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
