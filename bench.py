#!/usr/bin/env python
"""Throughput of the BitNet b1.58 BitLinear forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (one JSON line on rank 0): BitLinear decode GB/s of the decode
sweep -- M in {1, 4, 16} tokens on the (K, N) = (4096, 4096) and
(4096, 11008) projections, six bitlinear_forward calls per step -- with the
packed weights resident in HBM and rotated over copies that total more than
three times the L2 so that every step streams them from DRAM.  A step is
captured once as a CUDA graph per weight copy and replayed.

Also on the line:
  roofline      the decode kernel (the whole forward is that one kernel):
                algorithmic bytes per launch / mean launch time over the timed
                graph replays, against the measured HBM copy bandwidth
  prefill       int8 TOPS of the prefill workload (M in {512, 2048, 8192},
                (K, N) = (3200, 8640) and (8640, 3200)), the same way, with
                the tcgen05 GEMM's own roofline against the int8 peak
  e2e           the decode metric with host buffers: the step's six bf16
                inputs copied in from one pinned buffer and its outputs back
                to a pinned buffer, the six calls between, double-buffered on
                three streams so that neighbouring steps' copies run beside a
                step's calls, one wait per step for its outputs on the host;
                beside it the same steps run serially (e2e.serial) and
                bitlinear_forward_host_async copying every call's input in
                and output out (e2e.per_call_host_api)
  dequant_export, stack3b_decode
                the bf16 export kernel's GB/s, and the 3B-class 26-layer
                projection stack at M=1 with and without grouped calls
  stack3b_prefill the same 3B-class stack at M=2048 (prefill engine), with
                int8 TOPS
  ffn100b_stack the 100B-class FFN stack (13 layers, 2.29 GB of packed
                weights) at M in {1, 8, 64, 512}: tokens/s per stack pass
  pack          weight ternarisation and packing timed alone on the GPU
                (28672 x 8192), and both CPU oracles' packing beside it
  cpu_baseline  the numpy CPU oracle on a bounded sample of the decode
                workload, with the plain C++ oracle timed beside it
                (cpu_baseline.cpp_oracle, one thread), and bounded samples of the
                prefill, 3B-stack and 100B-FFN workloads (cpu_baseline.per_workload)
  clocks        nvidia-smi samples taken while the workload ran

With --gpus N > 1 (under torchrun) every rank runs the same workload on its
own GPU (data-parallel replicas: tokens split, weights replicated; the
forward has no exchange step), elapsed time is the max over ranks and the
value is the total over ranks.  --impl reference times the CPU oracle (the
only reference this method has) on the same metric, on rank 0 only.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth                                   # noqa: E402
from synth import workloads as wl               # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_OVER_BF16 = 2.0      # nominal dense ratio (4.5 / 2.25 PFLOP/s)


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def forward_launches(M, K):
    """Kernels one bitlinear_forward launches: the act-quant kernel and the
    GEMM above 16 tokens; the decode kernel alone up to 8 tokens (at 8
    tokens only up to K = 8192), else the act-quant kernel before it."""
    return 2 if (M > 8 or (M == 8 and K > 8192)) else 1


def decode_bytes(M, N, K, bias=True):
    """Algorithmic bytes of one BitLinear forward: 2-bit packed weights,
    bf16 x in, bf16 y out, bf16 bias, fp32 s_w."""
    return N * K // 4 + 2 * M * K + 2 * M * N + (2 * N if bias else 0) + 4


def contraction_bytes(M, N, K, bias=True):
    """Algorithmic bytes of the contraction kernel alone: packed weights,
    int8 x, s_x and row sums, bias, bf16 y."""
    return N * K // 4 + M * K + 8 * M + 2 * M * N + (2 * N if bias else 0) + 4


def kernel_src_hash(name):
    src = os.path.join(ROOT, "bitlinear_fwd_b200", "csrc", name)
    return hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]


def traffic_from_profile(kernel, src_name):
    """DRAM bytes per launch of ``kernel`` from an ncu capture, as recorded in
    profiles/traffic.json (written beside the capture's summary), or None
    when there is no record or the kernel's source changed since the
    capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec or rec.get("source_sha256_16") != kernel_src_hash(src_name):
        return None
    return float(rec["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-lms", "100", "-i", str(device_index)], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                s = float(r[1])
                smax = float(r[2])
            except (ValueError, IndexError):
                continue
            sm.append(s)
            for nm, v in zip(names, r[5:9]):
                if v.strip() == "Active":
                    reasons.add(nm)
        loaded = [s for s in sm if smax and s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist_on():
    return torch.distributed.is_available() and torch.distributed.is_initialized()


def world_size():
    return torch.distributed.get_world_size() if _dist_on() else 1


def _reduce_device():
    # NCCL reduces device tensors; gloo (the CPU test harness) host tensors
    if torch.distributed.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def elapsed_max_over_ranks(ms):
    """The job's time is its slowest rank's: every rank passes its own
    device-timed milliseconds and gets the maximum back."""
    if _dist_on():
        t = torch.tensor([ms], dtype=torch.float64, device=_reduce_device())
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())
    return ms


def whole_job_gbs(bytes_per_rank_step, steps, ms_max, world):
    """Whole-job throughput: the bytes all replicas processed over the
    slowest rank's time (every rank runs the same step)."""
    return world * bytes_per_rank_step * steps / (ms_max * 1e-3) / 1e9


def barrier():
    if _dist_on():
        torch.distributed.barrier()


def sync_all():
    barrier()
    torch.cuda.synchronize()


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

class Problem:
    def __init__(self, M, N, K, x, w_packed, s_w, bias, copies):
        import bitlinear_fwd_b200 as bl
        self.M, self.N, self.K = M, N, K
        self.x = x
        self.bias = bias
        self.s_w = s_w
        self.packed = [w_packed] + [w_packed.clone() for _ in range(copies - 1)]
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        self.ws = bl.workspace(M, N, K, "cuda")
        self.xq, self.s_x, self.rs = bl.bitlinear_quant_act(x)
        self.ws_q8 = torch.zeros(256, dtype=torch.uint8, device="cuda")

    def forward(self, r):
        import bitlinear_fwd_b200 as bl
        bl.bitlinear_forward(self.x, self.packed[r], self.s_w, self.bias, ws=self.ws, out=self.y,
                             flags=bl.WEIGHTS_RESIDENT)

    def contract(self, r):
        import bitlinear_fwd_b200 as bl
        bl.bitlinear_forward_q8(self.xq, self.s_x, self.rs, self.packed[r], self.s_w, self.bias, ws=self.ws_q8,
                                out=self.y)


def make_problems(cases, l2_bytes, rotate_factor=3.0, max_copies=64, force_copies=0):
    import bitlinear_fwd_b200 as bl
    wcache = {}
    per_step = 0
    staged = []
    for c in cases:
        key = (c.N, c.K, c.tags.get("shape"))
        if key not in wcache:
            packed, s_w, _ = bl.bitlinear_pack_weights(c.w().cuda())
            wcache[key] = (packed, s_w)
        b = c.bias()
        staged.append((c, b))
        per_step += c.N * c.K // 4
    copies = int(min(max_copies, max(2, np.ceil(rotate_factor * l2_bytes / max(per_step, 1)))))
    if force_copies:
        copies = force_copies
    probs = []
    for c, b in staged:
        packed, s_w = wcache[(c.N, c.K, c.tags.get("shape"))]
        probs.append(Problem(c.M, c.N, c.K, c.x().cuda(), packed, s_w, None if b is None else b.cuda(), copies))
    torch.cuda.synchronize()
    return probs, copies


class StepGraphs:
    """CUDA graphs of the timed steps: one graph per weight copy (one step
    each) and one graph holding a pass over all copies (``copies`` steps in
    order), so that consecutive steps run back to back on the device with no
    graph launch between them.  Step i always uses weight copy i % copies."""

    def __init__(self, single, multi, copies):
        self.single, self.multi, self.copies = single, multi, copies

    def run(self, first, n):
        """Replays steps first .. first + n - 1."""
        i = first
        end = first + n
        while i < end:
            if i % self.copies == 0 and end - i >= self.copies:
                self.multi.replay()
                i += self.copies
            else:
                self.single[i % self.copies].replay()
                i += 1


def capture_steps(probs, copies, fn_name):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for r in range(copies):
            for p in probs:                       # warm call outside capture
                getattr(p, fn_name)(r)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    single = []
    for r in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for p in probs:
                getattr(p, fn_name)(r)
        single.append(g)
    multi = torch.cuda.CUDAGraph()
    with torch.cuda.graph(multi):
        for r in range(copies):
            for p in probs:
                getattr(p, fn_name)(r)
    torch.cuda.synchronize()
    return StepGraphs(single, multi, copies)


def timed_replays(graphs, steps, warmup, preroll_s=0.0):
    graphs.run(0, warmup)
    torch.cuda.synchronize()
    if preroll_s > 0:
        t0 = time.time()
        while time.time() - t0 < preroll_s:
            graphs.run(0, graphs.copies)
            torch.cuda.synchronize()
    sync_all()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graphs.run(0, steps)
    e1.record()
    e1.synchronize()
    sync_all()
    return elapsed_max_over_ranks(e0.elapsed_time(e1))


def kernel_times(probs, copies, reps=20, fn="contract"):
    """Mean duration (ms) of one isolated launch per problem, between CUDA
    events on the launching stream, launches queued behind a sleep so that
    the host does not pace them."""
    out = []
    for p in probs:
        evs = []
        torch.cuda._sleep(20_000_000)
        for i in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            getattr(p, fn)(i % copies)
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize()
        out.append(statistics.mean(a.elapsed_time(b) for a, b in evs[2:]))
    return out


def run_decode(args, hbm_gbs, l2_bytes, peak_kind):
    """The decode forward is one kernel (quantisation, contraction, epilogue;
    above 8 tokens the act-quant kernel first), so the timed region is a
    back-to-back sequence of dependent forwards: its average launch duration
    is the timed time over the forwards, and its algorithmic bytes are the
    forward's.  Steps are replayed from graphs that hold several steps, so
    that no graph launch sits between consecutive steps."""
    cases = wl.workload2()
    probs, copies = make_problems(cases, l2_bytes, force_copies=args.copies)
    graphs = capture_steps(probs, copies, "forward")
    bytes_step = sum(decode_bytes(p.M, p.N, p.K, p.bias is not None) for p in probs)
    ms = timed_replays(graphs, args.steps, args.warmup, preroll_s=args.preroll)
    world = world_size()
    value = whole_job_gbs(bytes_step, args.steps, ms, world)
    launches = len(probs) * args.steps
    achieved = bytes_step * args.steps / (ms * 1e-3) / 1e9          # this rank's kernel
    kt = kernel_times(probs, copies, fn="forward")
    per_case = [{"M": p.M, "N": p.N, "K": p.K, "isolated_us": round(t * 1e3, 3),
                 "isolated_gbs": round(decode_bytes(p.M, p.N, p.K) / (t * 1e-3) / 1e9, 1)}
                for p, t in zip(probs, kt)]
    traffic = traffic_from_profile("decode_kernel", "gemv_decode.cu")
    roof = {"kernel": "decode_kernel", "bound": "hbm", "achieved": round(achieved, 1),
            "peak": hbm_gbs, "unit": "GB/s", "frac": round(achieved / hbm_gbs, 4),
            "peak_source": f"{peak_kind} HBM copy bandwidth (burst figure)",
            "avg_launch_us": round(ms * 1e3 / launches, 3),
            "algorithmic_bytes_per_launch_avg": round(bytes_step / len(probs)),
            "traffic": traffic, "per_case_isolated_launch": per_case}
    return {"value": value, "ms": ms, "bytes_step": bytes_step, "roofline": roof, "copies": copies,
            "graphs": graphs, "probs": probs,
            # the decode kernel, plus the act-quant kernel above 8 tokens
            "launches_per_step": sum(forward_launches(p.M, p.K) for p in probs)}


def run_e2e(args, probs, steps):
    """The headline metric end to end with host buffers, three ways.

    Step-batched: the step's six inputs sit in one pinned host buffer and
    are copied to the device in one copy, the six bitlinear_forward calls
    run on device views of it, and the six outputs come back in one copy to
    a pinned buffer.  Pipelined (the reported value), the same copies and
    calls double-buffered on three streams, so that the copies of the
    neighbouring steps run beside a step's calls, with one wait per step for
    that step's outputs in host memory; serial (reported beside it), copy
    in, calls and copy out one after the other, one graph launch and one
    synchronisation per step.

    Per call (reported beside it): every bitlinear_forward_host_async call
    copies its own bf16 x in and its bf16 y out (12 copies, 6 kernels per
    step), captured as a graph -- the library's calls are stream-ordered, so
    a graph holds them as they are -- and also issued call by call."""
    import bitlinear_fwd_b200 as bl
    xs = [p.x.cpu().pin_memory() for p in probs]
    ys = [torch.empty((p.M, p.N), dtype=torch.bfloat16).pin_memory() for p in probs]
    wss = [bl.workspace(p.M, p.N, p.K, "cuda", host=True) for p in probs]
    bytes_step = sum(decode_bytes(p.M, p.N, p.K, p.bias is not None) for p in probs)
    copies = len(probs[0].packed)

    def enqueue(r):
        for p, x, y, ws in zip(probs, xs, ys, wss):
            bl.bitlinear_forward_host_async(x, p.packed[r % copies], p.s_w, p.bias, y_host=y, ws=ws,
                                            flags=bl.WEIGHTS_RESIDENT)

    def timed(step_fn):
        for i in range(3):
            step_fn(i)
        sync_all()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(steps):
            step_fn(i)
        e1.record()
        e1.synchronize()
        sync_all()
        return elapsed_max_over_ranks(e0.elapsed_time(e1))

    def plain_step(r):
        enqueue(r)
        torch.cuda.current_stream().synchronize()

    ms_plain = timed(plain_step)
    # one graph per weight copy, captured on a side stream
    graphs = []
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        enqueue(0)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for r in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            enqueue(r)
        graphs.append(g)

    def graph_step(r):
        graphs[r % copies].replay()
        torch.cuda.current_stream().synchronize()

    ms = timed(graph_step)
    del graphs

    # step-batched: one pinned buffer of the six inputs, one of the six outputs
    xsz = [p.M * p.K for p in probs]
    ysz = [p.M * p.N for p in probs]
    xh = torch.cat([x.reshape(-1) for x in xs]).pin_memory()
    yh = torch.empty(sum(ysz), dtype=torch.bfloat16).pin_memory()
    xd = torch.empty(sum(xsz), dtype=torch.bfloat16, device="cuda")
    yd = torch.empty(sum(ysz), dtype=torch.bfloat16, device="cuda")
    xo = np.cumsum([0] + xsz)
    yo = np.cumsum([0] + ysz)
    xv = [xd[xo[i]:xo[i + 1]].view(p.M, p.K) for i, p in enumerate(probs)]
    yv = [yd[yo[i]:yo[i + 1]].view(p.M, p.N) for i, p in enumerate(probs)]
    dws = [bl.workspace(p.M, p.N, p.K, "cuda") for p in probs]

    def enqueue_batched(r):
        xd.copy_(xh, non_blocking=True)
        for p, x, y, ws in zip(probs, xv, yv, dws):
            bl.bitlinear_forward(x, p.packed[r % copies], p.s_w, p.bias, ws=ws, out=y, flags=bl.WEIGHTS_RESIDENT)
        yh.copy_(yd, non_blocking=True)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        enqueue_batched(0)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    bgraphs = []
    for r in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            enqueue_batched(r)
        bgraphs.append(g)

    def batched_step(r):
        bgraphs[r % copies].replay()
        torch.cuda.current_stream().synchronize()

    ms_b = timed(batched_step)
    # the outputs that came back are the device results
    torch.cuda.synchronize()
    ok = bool(torch.equal(yh, yd.cpu()))
    del bgraphs

    # pipelined (the reported value): the same copies and calls, with two
    # device input and output buffers and two pinned output buffers, on three
    # streams -- step i+1's input copy and step i-1's output copy run beside
    # step i's six calls; the host waits for step i-1's outputs to land in
    # host memory before it issues step i+1
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    xd2 = [xd, xd.clone()]                      # both hold the step's inputs before the warm-up call
    yd2 = [yd, torch.empty_like(yd)]
    yh2 = [yh, torch.empty_like(yh).pin_memory()]
    xv2 = [[b[xo[i]:xo[i + 1]].view(p.M, p.K) for i, p in enumerate(probs)] for b in xd2]
    yv2 = [[b[yo[i]:yo[i + 1]].view(p.M, p.N) for i, p in enumerate(probs)] for b in yd2]
    dws2 = [dws, [bl.workspace(p.M, p.N, p.K, "cuda") for p in probs]]

    def calls(b, r):
        for p, x, y, ws in zip(probs, xv2[b], yv2[b], dws2[b]):
            bl.bitlinear_forward(x, p.packed[r % copies], p.s_w, p.bias, ws=ws, out=y, flags=bl.WEIGHTS_RESIDENT)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        calls(1, 0)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    pgraphs = {}
    for b in range(2):
        for r in range(copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                calls(b, r)
            pgraphs[(b, r)] = g

    def pipelined(nsteps):
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        done = [None] * nsteps
        cur = torch.cuda.current_stream()
        for s in (s_in, s_cmp, s_out):
            s.wait_stream(cur)

        def issue(i):
            b = i % 2
            s_in.wait_event(ev_cmp[b])              # step i-2's calls have read xd[b]
            with torch.cuda.stream(s_in):
                xd2[b].copy_(xh, non_blocking=True)
            ev_in[b].record(s_in)
            s_cmp.wait_event(ev_in[b])
            s_cmp.wait_event(ev_out[b])             # step i-2's outputs have left yd[b]
            with torch.cuda.stream(s_cmp):
                pgraphs[(b, i % copies)].replay()
            ev_cmp[b].record(s_cmp)
            s_out.wait_event(ev_cmp[b])
            with torch.cuda.stream(s_out):
                yh2[b].copy_(yd2[b], non_blocking=True)
            ev_out[b].record(s_out)
            done[i] = ev_out[b]

        issue(0)
        for i in range(nsteps):
            if i + 1 < nsteps:
                issue(i + 1)
            done[i].synchronize()                   # step i's outputs are in host memory
        cur.wait_stream(s_out)

    pipelined(4)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    pipelined(steps)
    e1.record()
    e1.synchronize()
    sync_all()
    ms_p = elapsed_max_over_ranks(e0.elapsed_time(e1))
    torch.cuda.synchronize()
    last = (steps - 1) % 2
    ok_p = bool(torch.equal(yh2[last], yd2[last].cpu())) and bool(torch.equal(yh2[last], yh))
    del pgraphs
    world = world_size()
    return {"value": round(whole_job_gbs(bytes_step, steps, ms_p, world), 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(sum(2 * n for n in xsz)),
            "d2h_bytes_per_step": int(sum(2 * n for n in ysz)),
            "us_per_step": round(ms_p * 1e3 / steps, 2),
            "api": "per step: one copy of the six bf16 inputs from one pinned host buffer, six "
                   "bitlinear_forward calls on device views (one CUDA graph), one copy of the six outputs "
                   "to a pinned host buffer; double-buffered on three streams (copy in, calls, copy out) "
                   "so the copies of neighbouring steps run beside a step's calls; the host waits for "
                   "each step's outputs in host memory (one event sync per step, at most one step ahead)",
            "outputs_match_device": ok and ok_p,
            "serial": {
                "value": round(whole_job_gbs(bytes_step, steps, ms_b, world), 2), "unit": "GB/s",
                "us_per_step": round(ms_b * 1e3 / steps, 2),
                "api": "the same copies and calls, copy in, calls and copy out one after the other in one "
                       "CUDA graph per step; one graph launch and one stream sync per step"},
            "per_call_host_api": {
                "value": round(whole_job_gbs(bytes_step, steps, ms, world), 2), "unit": "GB/s",
                "us_per_step": round(ms * 1e3 / steps, 2),
                "api": "bitlinear_forward_host_async (pinned host x in, host y out) x 6 per step, the step "
                       "captured once as a CUDA graph; one graph launch and one stream sync per step",
                "without_graph": {"value": round(whole_job_gbs(bytes_step, steps, ms_plain, world), 2),
                                  "unit": "GB/s", "us_per_step": round(ms_plain * 1e3 / steps, 2),
                                  "api": "the same six calls issued one by one, one stream sync per step"}}}


def measured_i8_peak():
    """The dense int8 tensor-core rate of this GPU from the library's own
    tcgen05 kind::i8 loop (bitlinear_measure_i8_peak), with the SM clock
    sampled while it ran."""
    import bitlinear_fwd_b200 as bl
    sampler = ClockSampler(torch.cuda.current_device())
    r = bl.measure_i8_peak(iters=20000, reps=3)
    clk = sampler.stop()
    mhz = clk.get("sm_mhz") or None
    out = {"tops": round(r["tops"], 1), "ms": round(r["ms"], 3), "clocks": clk,
           "how": "tcgen05.mma.cta_group::1.kind::i8 128x256x32, smem operands, one CTA per SM, "
                  f"{r['iters']} x 4 per CTA, best of 3 launches (CUDA events)"}
    if mhz:
        out["mac_per_clk_per_sm"] = round(r["macs_per_sm"] / (r["ms"] * 1e-3) / (mhz * 1e6), 1)
    return out


def run_prefill(args, bf16_tflops, peak_kind, l2_bytes, i8_peak=None):
    cases = wl.workload3()
    probs, copies = make_problems(cases, l2_bytes, rotate_factor=1.0, max_copies=3, force_copies=args.copies)
    graphs = capture_steps(probs, copies, "forward")
    ops_step = sum(2 * p.M * p.N * p.K for p in probs)
    steps = max(3, args.prefill_steps)
    ms = timed_replays(graphs, steps, max(3, args.warmup))
    tops = world_size() * ops_step * steps / (ms * 1e-3) / 1e12
    kt = kernel_times(probs, copies, reps=8)
    ops = [2 * p.M * p.N * p.K for p in probs]
    achieved = sum(ops) / (sum(kt) * 1e-3) / 1e12
    peak_bf16x2 = bf16_tflops * INT8_OVER_BF16
    peak = i8_peak["tops"] if i8_peak else peak_bf16x2
    per_case = [{"M": p.M, "N": p.N, "K": p.K, "us": round(t * 1e3, 2),
                 "tops": round(o / (t * 1e-3) / 1e12, 1)} for p, t, o in zip(probs, kt, ops)]
    traffic = traffic_from_profile("gemm_prefill_kernel", "gemm_prefill.cu")
    del graphs
    return {"metric": "BitLinear prefill int8 TOPS (bitlinear_forward incl. activation quantisation)",
            "value": round(tops, 1), "unit": "TOPS", "ms_per_step": round(ms / steps, 4), "steps": steps,
            "workload": "prefill: M in {512,2048,8192} x (K,N) in {(3200,8640),(8640,3200)}, x Student-t(4) "
                        "bf16, W N(0,0.02) ternarised; 6 forwards per step",
            "roofline": {"kernel": "gemm_prefill_kernel", "bound": "tensor", "achieved": round(achieved, 1),
                         "peak": round(peak, 1), "unit": "TOPS", "frac": round(achieved / peak, 4),
                         "peak_source": ("measured int8 tensor-core rate (bitlinear_measure_i8_peak, this run)"
                                         if i8_peak else
                                         f"{peak_kind} bf16 dense x {INT8_OVER_BF16:g} (nominal int8/bf16)"),
                         "peak_bf16x2": round(peak_bf16x2, 1), "frac_of_bf16x2": round(achieved / peak_bf16x2, 4),
                         "traffic": traffic, "per_case": per_case}}


# ---------------------------------------------------------------------------
# the CPU oracle (cpu_baseline and the reference arm)
def _random_packed(N, K, gen):
    """Packed ternary rows with valid codes (each 2-bit field in {0, 1, 2})."""
    lut = torch.tensor([a | (b << 2) | (c << 4) | (d << 6) for a in range(3) for b in range(3)
                        for c in range(3) for d in range(3)], dtype=torch.uint8, device="cuda")
    return lut[torch.randint(0, 81, (N, K // 4), device="cuda", generator=gen)]


def run_stack3b(hbm_gbs, M=1, layers=26, reps=20, int8_tops=None):
    """The 3B-class decoder projection stack at M tokens: per layer q/k/v
    (3200 -> 3 x 3200), o (3200 -> 3200), gate/up (3200 -> 2 x 8640), down
    (8640 -> 3200); 26 layers of independent weights (806 MB packed).
    Timed two ways: one bitlinear_forward per projection (7 launches per
    layer) and with the shared-input groups fused (q/k/v and gate/up through
    bitlinear_forward_grouped: 4 launches per layer).  Weights resident,
    replayed as one CUDA graph per pass.  With M > 16 (the prefill engine)
    and ``int8_tops`` given, int8 TOPS against that peak are added."""
    import bitlinear_fwd_b200 as bl
    H, F = 3200, 8640
    gen = torch.Generator(device="cuda").manual_seed(21)
    lay = []
    for _ in range(layers):
        L = {"qkv": _random_packed(3 * H, H, gen), "o": _random_packed(H, H, gen),
             "gu": _random_packed(2 * F, H, gen), "down": _random_packed(H, F, gen)}
        L["s3"] = torch.full((3,), 40.0, device="cuda")              # stacked, for the grouped calls
        L["s2"] = torch.full((2,), 40.0, device="cuda")
        L["s1"] = [torch.full((1,), 40.0, device="cuda") for _ in range(5)]   # one per separate call
        lay.append(L)
    x = (torch.randn((M, H), device="cuda", generator=gen)).to(torch.bfloat16)
    xf = (torch.randn((M, F), device="cuda", generator=gen)).to(torch.bfloat16)
    y3 = torch.empty((M, 3 * H), dtype=torch.bfloat16, device="cuda")
    yo = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty((M, 2 * F), dtype=torch.bfloat16, device="cuda")
    ws = bl.workspace(M, 2 * F, F, "cuda")
    R = bl.WEIGHTS_RESIDENT

    def grouped():
        for L in lay:
            bl.bitlinear_forward_grouped(x, L["qkv"], [H, H, H], L["s3"], ws=ws, out=y3, flags=R)
            bl.bitlinear_forward(x, L["o"], L["s3"][:1], ws=ws, out=yo, flags=R)
            bl.bitlinear_forward_grouped(x, L["gu"], [F, F], L["s2"], ws=ws, out=y2, flags=R)
            bl.bitlinear_forward(xf, L["down"], L["s2"][:1], ws=ws, out=yo, flags=R)

    def separate():
        for L in lay:
            for g in range(3):
                bl.bitlinear_forward(x, L["qkv"][g * H:(g + 1) * H], L["s1"][g], ws=ws,
                                     out=y3[:, g * H:(g + 1) * H] if M == 1 else None, flags=R)
            bl.bitlinear_forward(x, L["o"], L["s3"][:1], ws=ws, out=yo, flags=R)
            for g in range(2):
                bl.bitlinear_forward(x, L["gu"][g * F:(g + 1) * F], L["s1"][3 + g], ws=ws,
                                     out=y2[:, g * F:(g + 1) * F] if M == 1 else None, flags=R)
            bl.bitlinear_forward(xf, L["down"], L["s2"][:1], ws=ws, out=yo, flags=R)

    out = {"workload": f"3B-class projection stack, {layers} layers, M={M}", "layers": layers, "M": M}
    wbytes = layers * (3 * H * H + H * H + 2 * F * H + H * F) // 4
    # per layer: grouped q/k/v, o, grouped gate/up, down; or the 7 projections
    ks = {"grouped": (H, H, H, F), "separate": (H, H, H, H, H, H, F)}
    for name, fn in (("grouped", grouped), ("separate", separate)):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        e1.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / reps
        out[name] = {"us_per_pass": round(us, 1), "tokens_per_s": round(M / (us * 1e-6), 1),
                     "weights_gbs": round(wbytes / (us * 1e-6) / 1e9, 1),
                     "frac_of_hbm": round(wbytes / (us * 1e-6) / 1e9 / hbm_gbs, 4),
                     "launches_per_pass": layers * sum(forward_launches(M, k) for k in ks[name])}
        if M > 16 and int8_tops:
            ops = 2 * M * layers * (3 * H * H + H * H + 2 * F * H + H * F)
            tops = ops / (us * 1e-6) / 1e12
            out[name].update({"tops": round(tops, 1), "frac_of_int8": round(tops / int8_tops, 4)})
        del g
    out["weights_bytes_per_pass"] = wbytes
    return out


def run_dequant(hbm_gbs, reps=20):
    """bf16 export of packed weights at the 100B-class gate/up shape (28672 x
    8192): 0.25 B read + 2 B written per weight, against the HBM copy peak."""
    import bitlinear_fwd_b200 as bl
    N, K = 28672, 8192
    g = torch.Generator(device="cuda").manual_seed(11)
    packed = torch.randint(0, 256, (N, K // 4), dtype=torch.uint8, device="cuda", generator=g)
    s_w = torch.full((1,), 50.0, device="cuda")
    out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    lib, st = bl.lib(), torch.cuda.current_stream().cuda_stream
    call = lambda: lib.bitlinear_dequant_weights(packed.data_ptr(), N, K, s_w.data_ptr(), out.data_ptr(), st)
    for _ in range(3):
        assert call() == 0
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        call()
    e1.record()
    e1.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    nbytes = N * K // 4 + 2 * N * K
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"kernel": "dequant_kernel", "shape": [N, K], "us_per_launch": round(us, 2),
            "bytes_per_launch": nbytes, "achieved": round(gbs, 1), "unit": "GB/s", "peak": hbm_gbs,
            "frac": round(gbs / hbm_gbs, 4), "note": "output 470 MB > L2, each launch streams it to DRAM"}


def run_ffn100b(hbm_gbs, int8_tops, Ms=(1, 8, 64, 512), layers=13, reps=10):
    """The 100B-class FFN stack: hidden 8192, FFN 28672; per layer gate and
    up (8192 -> 28672, the same input) and down (28672 -> 8192); 13 layers
    of independent weights (2.29 GB packed, far above L2).  One
    bitlinear_forward per projection (3 launches per layer), weights
    resident, one CUDA graph per pass of the whole stack.  Reports the
    equivalent tokens/s of the stack, and the weight stream (GB/s, M <= 8:
    the decode engine) or int8 TOPS (M >= 64: the prefill engine) against
    its roofline."""
    import bitlinear_fwd_b200 as bl
    H, F = 8192, 28672
    gen = torch.Generator(device="cuda").manual_seed(31)
    lay = [{"gate": _random_packed(F, H, gen), "up": _random_packed(F, H, gen),
            "down": _random_packed(H, F, gen), "s": torch.full((1,), 80.0, device="cuda")}
           for _ in range(layers)]
    wbytes = layers * 3 * F * H // 4
    R = bl.WEIGHTS_RESIDENT
    out = {"workload": f"100B-class FFN stack: {layers} layers x (gate, up 8192->28672; down 28672->8192), "
                       "random valid 2-bit codes, no bias",
           "layers": layers, "weights_bytes_per_pass": wbytes, "calls_per_pass": 3 * layers,
           "per_M": []}
    for M in Ms:
        x = torch.randn((M, H), device="cuda", generator=gen).to(torch.bfloat16)
        xd = torch.randn((M, F), device="cuda", generator=gen).to(torch.bfloat16)
        yg = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")
        yu = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")
        yd = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
        ws = bl.workspace(M, F, F, "cuda")

        def stack():
            for L in lay:
                bl.bitlinear_forward(x, L["gate"], L["s"], ws=ws, out=yg, flags=R)
                bl.bitlinear_forward(x, L["up"], L["s"], ws=ws, out=yu, flags=R)
                bl.bitlinear_forward(xd, L["down"], L["s"], ws=ws, out=yd, flags=R)

        stack()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            stack()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        e1.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / reps
        ops = layers * 3 * 2 * M * F * H
        row = {"M": M, "us_per_pass": round(us, 1), "tokens_per_s": round(M / (us * 1e-6), 1),
               "launches_per_pass": layers * (2 * forward_launches(M, H) + forward_launches(M, F))}
        if M <= 16:
            gbs = wbytes / (us * 1e-6) / 1e9
            row.update({"bound": "hbm", "weights_gbs": round(gbs, 1), "frac": round(gbs / hbm_gbs, 4)})
        else:
            tops = ops / (us * 1e-6) / 1e12
            row.update({"bound": "tensor", "tops": round(tops, 1), "frac": round(tops / int8_tops, 4)})
        out["per_M"].append(row)
        del g, x, xd, yg, yu, yd, ws
    del lay
    return out


def pack_bytes(N, K):
    """Algorithmic bytes of one weight packing: W read twice (the mean must be
    complete before any weight is ternarised, and these W are larger than
    L2), the 2-bit codes written, the scale and the mean."""
    return 2 * 4 * N * K + N * K // 4 + 8


def run_pack(hbm_gbs, reps=10):
    """Weight ternarisation and packing timed alone (bitlinear_pack_weights:
    absmean bins, finalize, ternarise-and-pack, three kernels) on the
    100B-class gate shape, 28672 x 8192 fp32 (940 MB, larger than L2), CUDA
    events over ``reps`` calls on the current stream."""
    import bitlinear_fwd_b200 as bl
    N, K = 28672, 8192
    g = torch.Generator(device="cuda").manual_seed(12)
    w = torch.randn((N, K), device="cuda", generator=g).mul_(0.01)
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    s_w = torch.empty(1, dtype=torch.float32, device="cuda")
    mean = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(bl.pack_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
    lib, st = bl.lib(), torch.cuda.current_stream().cuda_stream
    call = lambda: lib.bitlinear_pack_weights(w.data_ptr(), N, K, packed.data_ptr(), s_w.data_ptr(),
                                              mean.data_ptr(), ws.data_ptr(), ws.numel(), st)
    for _ in range(3):
        assert call() == 0
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        call()
    e1.record()
    e1.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    nbytes = pack_bytes(N, K)
    gbs = nbytes / (us * 1e-6) / 1e9
    del w, packed, ws
    return {"kernels": "absmean_bins_kernel + absmean_finalize_kernel + ternarise_pack_kernel",
            "shape": [N, K], "us_per_call": round(us, 1), "bytes_per_call": nbytes,
            "achieved": round(gbs, 1), "unit": "GB/s", "peak": hbm_gbs, "frac": round(gbs / hbm_gbs, 4),
            "note": "once per weight matrix, outside the forward; bytes = 8 B/weight (W read twice) "
                    "+ 0.25 B/weight written"}


def oracle_pack_baseline(budget_s=6.0):
    """Both CPU oracles' pack_weights on the decode sweep's 11008 x 4096
    weights, bytes counted as for the GPU."""
    out = {}
    w = None
    for impl in ("numpy", "cpp"):
        try:
            if impl == "cpp":
                from oracle import cpp as orc
            else:
                import oracle as orc
            if w is None:
                c = [c for c in wl.workload2() if c.N == 11008][0]
                w = c.w().numpy()
            N, K = w.shape
            s, n = 0.0, 0
            while s < budget_s / 2 and n < 4:
                t0 = time.perf_counter()
                orc.pack_weights(w)
                s += time.perf_counter() - t0
                n += 1
            out[impl] = {"value": round(pack_bytes(N, K) * n / s / 1e9, 3), "unit": "GB/s",
                         "cores": 1, "sample": f"{n} calls ({s:.1f} s) of pack_weights on [{N}, {K}] fp32"}
        except Exception as e:
            out[impl] = {"unavailable": f"{type(e).__name__}: {e}"}
    return out


# ---------------------------------------------------------------------------

class OracleDecode:
    """A CPU oracle on the decode workload (all six problems, every weight
    row): the numpy oracle, or with ``impl="cpp"`` the plain C++ one.
    Inputs are generated and packed by that oracle once, untimed."""

    def __init__(self, impl="numpy", threads=1):
        self.threads = max(1, int(threads))
        if impl == "cpp":
            from oracle import cpp as oracle
        else:
            import oracle
        self.oracle = oracle
        try:
            from threadpoolctl import threadpool_info
            self.blas = max([i.get("num_threads", 1) for i in threadpool_info()
                             if i.get("user_api") == "blas"] or [1])
        except Exception:
            self.blas = 1
        wcache = {}
        self.items = []
        for c in wl.workload2():
            key = (c.N, c.K)
            if key not in wcache:
                wcache[key] = oracle.pack_weights(c.w().numpy())
            packed, s_w, _ = wcache[key]
            self.items.append((synth.bf16_bits(c.x()), packed, s_w, synth.bf16_bits(c.bias()),
                               decode_bytes(c.M, c.N, c.K)))
        if impl == "cpp":
            self.cores = self.threads
            self.desc = ("the C++ oracle's forward (plain loops: act quant, unpack, int64 contraction, "
                         "epilogue) on the 6 decode problems with every weight row, packing untimed; " +
                         ("one thread" if self.threads == 1 else
                          f"{self.threads} host threads, each calling it on its own block of weight rows "
                          "(the oracle itself unchanged)"))
        else:
            self.cores = self.blas
            self.desc = ("oracle.forward (act quant, unpack, exact contraction, epilogue) on the 6 decode "
                         "problems with every weight row, packing untimed; numpy elementwise steps "
                         f"single-threaded, float64 matmul on {self.blas} BLAS threads")

    def step(self):
        """One pass over the workload; returns (bytes, seconds)."""
        b, s = 0, 0.0
        pool = None
        if self.threads > 1:
            import concurrent.futures as fut
            pool = fut.ThreadPoolExecutor(self.threads)
        try:
            for xb, packed, s_w, bb, nbytes in self.items:
                t0 = time.perf_counter()
                if pool is None:
                    self.oracle.forward(xb, packed, s_w, bb)
                else:
                    # rows are independent: each thread runs the oracle on one block of them
                    N = packed.shape[0]
                    cuts = np.linspace(0, N, self.threads + 1).astype(int)
                    jobs = [pool.submit(self.oracle.forward, xb, np.ascontiguousarray(packed[a:c]), s_w,
                                        None if bb is None else np.ascontiguousarray(bb[a:c]))
                            for a, c in zip(cuts[:-1], cuts[1:]) if c > a]
                    for j in jobs:
                        j.result()
                s += time.perf_counter() - t0
                b += nbytes
        finally:
            if pool is not None:
                pool.shutdown()
        return b, s


def timed_oracle(impl, budget_s, max_passes=8, threads=1):
    """Passes of one CPU oracle over the decode workload until ``budget_s``
    seconds of oracle time; a cpu_baseline-style dict."""
    od = OracleDecode(impl, threads)
    b, s, n = 0, 0.0, 0
    while s < budget_s and n < max_passes:
        bb, ss = od.step()
        b, s, n = b + bb, s + ss, n + 1
    return {"value": round(b / s / 1e9, 4), "unit": "GB/s", "cores": od.cores, "kind": "oracle",
            "sample": f"{n} passes ({s:.1f} s) of " + od.desc}


def oracle_workloads_baseline():
    """The numpy oracle beyond the decode sweep, one bounded sample each:
    workload 3 at M=512 (K=3200, N=8640); one layer of workload 4 at M=1
    (7 projections; the 26-layer figure is extrapolated); the gate
    projection of workload 5 at M=8 (random valid 2-bit codes, since the
    forward's cost does not depend on their values; the 39-projection stack
    figure is extrapolated).  Packing is untimed."""
    import oracle
    out = []

    def timed(fn, reps=1, warm=True):
        if warm:
            fn()
        t0 = time.perf_counter()
        for _ in range(reps):
            fn()
        return (time.perf_counter() - t0) / reps

    try:
        c = [c for c in wl.workload3() if c.M == 512 and c.K == 3200][0]
        packed, s_w, _ = oracle.pack_weights(c.w().numpy())
        xb = synth.bf16_bits(c.x())
        t = timed(lambda: oracle.forward(xb, packed, s_w))
        out.append({"workload": "prefill M=512, K=3200, N=8640 (workload 3)", "s_per_call": round(t, 3),
                    "value": round(2 * c.M * c.N * c.K / t / 1e12, 5), "unit": "TOPS"})
    except Exception as e:
        out.append({"workload": "prefill M=512", "unavailable": f"{type(e).__name__}: {e}"})
    try:
        calls = []
        for c in wl.workload4(1, layers=[0]):
            packed, s_w, _ = oracle.pack_weights(c.w().numpy())
            calls.append((synth.bf16_bits(c.x()), packed, s_w))
        t = timed(lambda: [oracle.forward(xb, p, s) for xb, p, s in calls])
        out.append({"workload": "3B-class stack at M=1 (workload 4): one layer of 7 projections timed, "
                                "26 layers extrapolated", "s_per_layer": round(t, 3),
                    "value": round(1.0 / (26 * t), 4), "unit": "tokens/s (extrapolated)"})
    except Exception as e:
        out.append({"workload": "3B-class stack", "unavailable": f"{type(e).__name__}: {e}"})
    try:
        N, K, M = 28672, 8192, 8
        rng = np.random.default_rng(5)
        lut = np.array([a | (b << 2) | (c << 4) | (d << 6) for a in range(3) for b in range(3)
                        for c in range(3) for d in range(3)], dtype=np.uint8)
        packed = lut[rng.integers(0, 81, (N, K // 4))]
        xb = synth.bf16_bits(synth.normal_bf16(wl.seed_of(5), 10_000, (M, K)))
        t = timed(lambda: oracle.forward(xb, packed, np.float32(80.0)), warm=False)
        out.append({"workload": "100B-class FFN (workload 5): one gate projection at M=8 timed, the "
                                "13-layer stack (39 projections) extrapolated", "s_per_call": round(t, 3),
                    "value": round(M / (39 * t), 5), "unit": "tokens/s (extrapolated)"})
    except Exception as e:
        out.append({"workload": "100B-class FFN", "unavailable": f"{type(e).__name__}: {e}"})
    return out


def cpp_oracle_baseline(budget_s=5.0):
    """The C++ oracle timed beside the numpy one, on one thread and on every
    host core (nproc); never fails the line."""
    try:
        one = timed_oracle("cpp", budget_s)
        nproc = os.cpu_count() or 1
        one["nproc"] = nproc
        if nproc > 1:
            one["all_cores"] = timed_oracle("cpp", budget_s, threads=nproc)
        return one
    except Exception as e:                      # e.g. no C++ compiler on the host
        return {"unavailable": f"{type(e).__name__}: {e}"}


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    od = OracleDecode()
    od.step()                                       # warm-up (page-in, BLAS threads)
    steps = max(1, min(args.steps, 8))
    b, s = 0, 0.0
    for _ in range(steps):
        bb, ss = od.step()
        b += bb
        s += ss
    v = b / s / 1e9
    line = {"impl": "reference", "metric": "BitLinear decode GB/s (% of HBM peak); prefill int8 TOPS (% TC peak)",
            "value": round(v, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": steps, "warmup": 1, "ms_per_step": round(1e3 * s / steps, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/int64 (numpy)",
            "data": "synthetic",
            "config": {"workload": "decode GEMV sweep: M in {1,4,16}, (K,N) in {(4096,4096),(4096,11008)}; "
                                   "the CPU oracle, the only reference implementation of this method",
                       "parallelism": "rank 0 host cores"},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": od.cores, "kind": "oracle",
                             "sample": f"{steps} passes of " + od.desc,
                             "cpp_oracle": cpp_oracle_baseline()},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------

def run_case(name):
    """One small case of one kernel, for ncu captures of a single kernel
    (no timing, no JSON line): seeded inputs at the sizes the profiles in
    profiles/ quote, each call repeated so that a capture can skip the first."""
    import bitlinear_fwd_b200 as bl
    dev = "cuda"
    if name in ("gemm", "gemm8640"):
        M, K, N = (2048, 3200, 8640) if name == "gemm" else (2048, 8640, 3200)
        packed, s_w, _ = bl.bitlinear_pack_weights(synth.normal_f32(1, 1, (N, K), 0.02, device=dev))
        x = synth.normal_bf16(1, 2, (M, K), device=dev)
        for _ in range(3):
            bl.bitlinear_forward(x, packed, s_w)
    elif name == "decode":
        K, N = 4096, 11008
        packed, s_w, _ = bl.bitlinear_pack_weights(synth.normal_f32(1, 1, (N, K), 0.02, device=dev))
        b = synth.normal_bf16(1, 3, (N,), 0.01, device=dev)
        for M in (1, 4, 16):
            bl.bitlinear_forward(synth.normal_bf16(1, 2 + M, (M, K), device=dev), packed, s_w, b,
                                 flags=bl.WEIGHTS_RESIDENT)
    elif name == "decodewide":
        # the 100B-class gate projection (28672 x 8192) at M = 1: the
        # weight stream, two CTAs per SM
        K, N = 8192, 28672
        packed, s_w, _ = bl.bitlinear_pack_weights(synth.normal_f32(1, 1, (N, K), 0.02, device=dev))
        x = synth.normal_bf16(1, 2, (1, K), device=dev)
        for _ in range(3):
            bl.bitlinear_forward(x, packed, s_w, flags=bl.WEIGHTS_RESIDENT)
    elif name == "actq":
        x = synth.normal_bf16(1, 2, (8192, 8640), device=dev)
        for _ in range(2):
            bl.bitlinear_quant_act(x)
    elif name == "pack":
        w = synth.normal_f32(1, 1, (28672, 8192), 0.01, device=dev)
        for _ in range(2):
            bl.bitlinear_pack_weights(w)
    elif name == "dequant":
        packed, s_w, _ = bl.bitlinear_pack_weights(synth.normal_f32(1, 1, (28672, 8192), 0.01, device=dev))
        for _ in range(2):
            bl.bitlinear_dequant_weights(packed, s_w)
    elif name == "ksplit":
        M, K, N = 4, 4096, 8192
        x = synth.normal_bf16(1, 2, (M, K), device=dev)
        packed, s_w, _ = bl.bitlinear_pack_weights(synth.normal_f32(1, 1, (N, K), 0.02, device=dev))
        am = bl.bitlinear_act_absmax(x)
        part = bl.bitlinear_forward_partial(x, am, packed)
        for _ in range(2):
            bl.bitlinear_epilogue_sum([part, part], am, s_w)
    torch.cuda.synchronize()
    print(json.dumps({"case": name, "ok": True}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--preroll", type=float, default=1.0, help="seconds of untimed replays before timing")
    ap.add_argument("--prefill-steps", type=int, default=20)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--only", choices=["decode", "prefill", "dequant", "stack3b"], default=None,
                    help="run one workload only (profiling runs; no JSON contract line)")
    ap.add_argument("--copies", type=int, default=0, help="force the number of rotating weight copies")
    ap.add_argument("--case", choices=["decode", "decodewide", "gemm", "gemm8640", "actq", "pack", "dequant",
                                       "ksplit"],
                    default=None, help="run one small case of one kernel for an ncu capture, then exit")
    args = ap.parse_args()
    if args.case:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        run_case(args.case)
        return 0
    args.warmup = max(3, args.warmup)

    if args.impl == "reference":
        return reference_arm(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    import bitlinear_fwd_b200 as bl
    bl.lib()
    hbm_gbs, bf16_tflops, peak_kind = peaks()
    l2_bytes = torch.cuda.get_device_properties(local).L2_cache_size

    if args.only == "prefill":
        i8 = measured_i8_peak()
        out = run_prefill(args, bf16_tflops, peak_kind, l2_bytes, i8)
        out["i8_peak"] = i8
        print(json.dumps(out), flush=True)
        return 0
    if args.only == "stack3b":
        print(json.dumps(run_stack3b(hbm_gbs)), flush=True)
        return 0
    if args.only == "dequant":
        print(json.dumps(run_dequant(hbm_gbs)), flush=True)
        return 0
    if args.only == "decode":
        d = run_decode(args, hbm_gbs, l2_bytes, peak_kind)
        print(json.dumps({"value": d["value"], "ms": d["ms"], "roofline": d["roofline"]}), flush=True)
        return 0
    sampler = ClockSampler(local)
    dec = run_decode(args, hbm_gbs, l2_bytes, peak_kind)
    clocks = sampler.stop()
    e2e = None if args.no_e2e else run_e2e(args, dec["probs"], max(3, min(200, args.steps // 10)))
    try:
        i8 = measured_i8_peak()
    except Exception as e:
        i8 = None
        i8_err = f"{type(e).__name__}: {e}"
    pre = None if args.no_prefill else run_prefill(args, bf16_tflops, peak_kind, l2_bytes, i8)
    if pre is not None:
        pre["i8_peak"] = i8 if i8 is not None else {"unavailable": i8_err}
    deq = run_dequant(hbm_gbs)
    stack = run_stack3b(hbm_gbs)
    try:
        pack = {"gpu": run_pack(hbm_gbs)}
    except Exception as e:
        pack = {"gpu": {"unavailable": f"{type(e).__name__}: {e}"}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = timed_oracle("numpy", 10.0)
        cpu["cpp_oracle"] = cpp_oracle_baseline()
        cpu["per_workload"] = oracle_workloads_baseline()
        pack["cpu_oracle"] = oracle_pack_baseline()
    try:
        ffn = run_ffn100b(hbm_gbs, i8["tops"] if i8 else bf16_tflops * INT8_OVER_BF16)
    except Exception as e:
        ffn = {"unavailable": f"{type(e).__name__}: {e}"}
    try:
        stack_pre = run_stack3b(hbm_gbs, M=2048, reps=5,
                                int8_tops=i8["tops"] if i8 else bf16_tflops * INT8_OVER_BF16)
    except Exception as e:
        stack_pre = {"unavailable": f"{type(e).__name__}: {e}"}

    line = {
        "metric": "BitLinear decode GB/s (% of HBM peak); prefill int8 TOPS (% TC peak)",
        "value": round(dec["value"], 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dec["ms"] / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic",
        "config": {"workload": "decode GEMV sweep: M in {1,4,16}, (K,N) in {(4096,4096),(4096,11008)}, "
                               "x N(0,1) bf16 with 1% channels x20, W N(0,0.02) ternarised + 2-bit packed, "
                               "bias N(0,0.01); 6 bitlinear_forward calls per step",
                   "global_batch": 21 * world, "parallelism": f"dp{world} replicas (no collective)",
                   "l2": f"inputs larger than L2: {dec['copies']} rotating packed-weight copies, "
                         f"{dec['copies'] * sum(p.N * p.K // 4 for p in dec['probs']) / 1e6:.0f} MB vs "
                         f"{l2_bytes / 1e6:.0f} MB L2",
                   "bytes_per_step": dec["bytes_step"],
                   "graph_replay": f"one CUDA graph per pass over the {dec['copies']} weight copies "
                                   f"({dec['copies']} steps back to back), one-step graphs for a remainder"},
        "roofline": dec["roofline"],
        "gpu_launches": dec["launches_per_step"] * args.steps,
        "e2e": e2e,
        "prefill": pre,
        "dequant_export": deq,
        "stack3b_decode": stack,
        "pack": pack,
        "ffn100b_stack": ffn,
        "stack3b_prefill": stack_pre,
        "cpu_baseline": cpu,
        "clocks": clocks,
    }
    del dec
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
