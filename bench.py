#!/usr/bin/env python
"""Benchmark of the MoE layout -> FP8 dispatch -> BF16 combine path on B200.

One step = cgl_get_layout + cgl_dispatch_fp8 + cgl_combine over one batch of
synthetic routing (batches of at most one token per SM: cgl_layout_dispatch_fp8,
one launch, + cgl_combine) (the 4096-token prefill shape by default: hidden 7168, 256
experts in 8 groups, top-4 groups / top-8 experts, 64 logical ranks) with all
inputs resident in HBM.  The metric is the step's algorithmic HBM bytes per
second; per-kernel microseconds and fractions of the measured HBM peak are in
the same JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill]
  python bench.py --impl reference ...   # the CPU oracle as the reference arm

Multi-GPU (torchrun): every rank runs its own replica of the workload (weak
scaling, no data-path collective); the timing is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from combine_get_layout_02_b200 import workloads as W  # noqa: E402

METRIC = "dispatch+combine µs and HBM GB/s (% of peak) at 4096 tok×7168, top-8/256"
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes per launch read by ncu (dram__bytes_read.sum + dram__bytes_write.sum)
# for the kernels at the 4096-token prefill shape, with the sha256 of the kernel
# source and the shared device header it was taken on; a changed source
# reports traffic null.
NCU_TRAFFIC = {
    "combine": {"bytes": 507279104, "src_sha": "829d3f12a04df5c7"},
    "dispatch_fp8": {"bytes": 243865088, "src_sha": "1e399167ee854d42"},
    "layout+dispatch_fp8": {"bytes": 247476480, "src_sha": "ff4c3e2d259d9d86"},
    "layout": {"bytes": 212736, "src_sha": "ff4c3e2d259d9d86"},
}


def _src_sha(name: str) -> str:
    h = hashlib.sha256()
    for f in (name, "common.cuh"):
        h.update(open(os.path.join(ROOT, "combine_get_layout_02_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, src: str):
    rec = NCU_TRAFFIC.get(kernel)
    if not rec or rec.get("src_sha") != _src_sha(src):
        return None
    return rec["bytes"]


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------- distributed

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_init(backend: str, timeout_s: float = 120.0):
    import datetime

    import torch.distributed as dist

    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity with one rank)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def rank_seed(seed: int, rank: int) -> int:
    """Each replica draws its own batch of the same workload."""
    return seed + 1000 * rank


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- steps

def workload_label(wl: W.Workload, dedup: bool = False, pow2: bool = False) -> str:
    tail = "; per-rank deduplicated dispatch (one copy per token and rank)" if dedup else ""
    tail += "; power-of-two (UE8M0) FP8 scales" if pow2 and wl.fp8 else ""
    return f"{wl.name}: {wl.description}{tail}"


class GpuStep:
    """Device buffers for one workload and the launch sequence of one step."""

    def __init__(self, wl: W.Workload, seed: int, device, dedup: bool = False, full_backward: bool = False,
                 fused_decode: bool = False, split_layout: bool = False, pow2_scales: bool = False,
                 fused_layout: bool = False):
        import torch

        import combine_get_layout_02_b200 as cgl

        self.cgl, self.torch, self.wl, self.dev = cgl, torch, wl, device
        self.dedup = dedup
        self.pow2 = pow2_scales
        self.full_backward = full_backward and wl.with_grad and not dedup
        self.fused_decode = fused_decode and wl.fp8 and not dedup
        # FP8 steps: the library's three calls (cgl_get_layout, cgl_dispatch_fp8
        # handing tokens out from a scratch counter, cgl_combine), measured a
        # little faster at prefill than the fused cgl_layout_dispatch_fp8 kernel;
        # batches of at most one token per SM take cgl_layout_dispatch_fp8 (one
        # launch, one CTA per token).  --fused-layout: cgl_layout_dispatch_fp8
        # at every size; --split-layout: the three calls at every size.
        one_per_sm = wl.num_tokens <= torch.cuda.get_device_properties(device).multi_processor_count
        self.layout_dispatch = (wl.fp8 and not dedup and not self.fused_decode and not split_layout
                                and (fused_layout or one_per_sm))
        inp = W.make_inputs(wl, seed)
        n, h, k = wl.num_tokens, wl.hidden, wl.topk
        self.host = inp
        self.M = n * k
        y_host = W.expert_outputs(self.M, h, seed)
        self.host_y = y_host

        def bf16(a):
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)

        self.x = bf16(inp.x).to(device)
        self.idx = torch.from_numpy(inp.topk_idx).to(device)
        self.w = torch.from_numpy(inp.topk_w).to(device)
        self.y = bf16(y_host).to(device)
        self.grad = bf16(inp.grad).to(device) if inp.grad is not None else None
        self.status = cgl.new_status(device)
        # the standalone dispatch calls hand tokens out from a counter in this scratch (cgl_opts.scratch)
        self.scratch = cgl.new_scratch(device)
        E, R = wl.num_experts, wl.num_ranks
        self.ws = torch.empty(max(cgl.layout_workspace_bytes(n, k, E, R),
                                  cgl.layout_dispatch_workspace_bytes(n, k, E, R)), dtype=torch.uint8, device=device)
        self.cap = 0
        if wl.padded:   # padded receive buffers: size them from a first compact call (host reads max)
            lay = cgl.get_layout(self.idx, E, R, 0, workspace=self.ws, status=self.status)
            self.cap = int(lay.max_count.item())
        self.lay = cgl.get_layout(self.idx, E, R, self.cap, workspace=self.ws, status=self.status)
        rows = self.lay.num_recv_rows
        self.rows = rows
        if wl.fp8:
            self.recv_x = torch.empty((rows, h), dtype=torch.uint8, device=device)
            self.recv_scale = torch.empty((rows, h // 128), dtype=torch.float32, device=device)
            if wl.padded:   # y rows follow the padded layout
                self.y = self.y.new_zeros((rows, h))
                self.y[self.lay.dst_pos.flatten().long()] = bf16(y_host).to(device)
        else:
            self.recv_x = torch.empty((rows, h), dtype=torch.bfloat16, device=device)
            self.grad_recv = torch.empty((rows, h), dtype=torch.bfloat16, device=device)
            self.grad_w = torch.empty((n, k), dtype=torch.float32, device=device)
        self.out = torch.empty((n, h), dtype=torch.bfloat16, device=device)
        self.bytes = W.algorithmic_bytes(wl)
        if dedup:
            # one copy per (token, destination rank); the combine sums each rank's partial row
            rcap = 0
            if wl.padded:
                rcap = int(cgl.get_rank_layout(self.idx, E, R, 0, workspace=self.ws).max_count.item())
            self.rcap = rcap
            self.rlay = cgl.get_rank_layout(self.idx, E, R, rcap, workspace=self.ws, status=self.status)
            self.rrows = self.rlay.num_recv_rows
            self.w_rank = (self.rlay.rank_dst >= 0).float()
            used = int(self.rlay.rank_offset[-1].item())
            self.used_rank_rows = used
            nb = wl.num_tokens
            self.bytes = {
                "layout": 12 * nb * k,
                "dispatch_fp8": 2 * nb * h + 4 * nb * k + used * (h + 4 * (h // 128)),
                "dispatch_bf16": 2 * nb * h + 4 * nb * k + used * 2 * h,
                "combine": 2 * used * h + 8 * nb * k + 2 * nb * h,
            }
            if wl.padded:
                self.y = self.y.new_zeros((self.rrows, h))
                self.y[self.rlay.rank_dst[self.rlay.rank_dst >= 0].long()] = \
                    bf16(y_host[:used]).to(device)
        torch.cuda.synchronize(device)

    def kernels(self):
        """(name, launches per step, algorithmic bytes per launch) of each step phase."""
        b = self.bytes
        wl = self.wl
        if self.fused_decode:   # one launch for layout + dispatch
            ph = [("layout+dispatch_fp8", 1, b["layout"] + b["dispatch_fp8"]),
                  ("combine", 1, b["combine"])]
            return ph
        if self.layout_dispatch:
            nk = self.cgl.layout_dispatch_kernel_count(wl.num_tokens, wl.topk, wl.num_experts, wl.num_ranks,
                                                       wl.hidden)
            return [("layout+dispatch_fp8", nk, b["layout"] + b["dispatch_fp8"]), ("combine", 1, b["combine"])]
        if self.dedup:   # rank keys: the layout of an E = R problem
            nl = self.cgl.layout_kernel_count(wl.num_tokens, wl.topk, wl.num_ranks, wl.num_ranks)
        else:
            nl = self.cgl.layout_kernel_count(wl.num_tokens, wl.topk, wl.num_experts, wl.num_ranks)
        ph = [("layout", nl, b["layout"])]
        if self.wl.fp8:
            ph.append(("dispatch_fp8", 1, b["dispatch_fp8"]))
        else:
            ph.append(("dispatch_bf16", 1, b["dispatch_bf16"]))
        ph.append(("combine", 1, b["combine"]))
        if self.wl.with_grad:
            if self.full_backward:   # g read once, y read and grad_y written per slot, ids/weights/grad_w
                n, h, k = wl.num_tokens, wl.hidden, wl.topk
                ph.append(("combine_backward", 1, 2 * n * h + 4 * n * k * h + 12 * n * k))
            else:
                ph.append(("combine_backward", 1, b["dispatch_bf16"]))
        return ph

    def step_bytes(self):
        return sum(v for _, _, v in self.kernels())

    def run(self, events=None):
        """One step; if `events` is a list, record an event after each phase."""
        cgl, wl = self.cgl, self.wl
        E, R = wl.num_experts, wl.num_ranks
        rec = (lambda: events.append(self._event())) if events is not None else (lambda: None)
        rec()
        if self.fused_decode:
            cgl.decode_dispatch_fp8(self.idx, self.x, E, R, self.cap, out=self.lay, recv_x=self.recv_x,
                                    recv_scale=self.recv_scale, status=self.status, pow2_scales=self.pow2)
            rec()
            cgl.combine(self.y, self.lay.dst_pos, self.w, out=self.out, status=self.status)
            rec()
            return
        if self.layout_dispatch:
            cgl.layout_dispatch_fp8(self.idx, self.x, E, R, self.cap, out=self.lay, recv_x=self.recv_x,
                                    recv_scale=self.recv_scale, workspace=self.ws, status=self.status,
                                    pow2_scales=self.pow2)
            rec()
            cgl.combine(self.y, self.lay.dst_pos, self.w, out=self.out, status=self.status)
            rec()
            return
        if self.dedup:
            cgl.get_rank_layout(self.idx, E, R, self.rcap, workspace=self.ws, out=self.rlay, status=self.status)
            rec()
            if wl.fp8:
                cgl.dispatch_fp8(self.x, self.rlay.rank_dst, self.rrows, recv_x=self.recv_x,
                                 recv_scale=self.recv_scale, status=self.status, pow2_scales=self.pow2,
                                 scratch=self.scratch)
            else:
                cgl.dispatch_bf16(self.x, self.rlay.rank_dst, self.rrows, recv_x=self.recv_x,
                                  status=self.status, scratch=self.scratch)
            rec()
            cgl.combine(self.y, self.rlay.rank_dst, self.w_rank, out=self.out, status=self.status)
            rec()
            if wl.with_grad:
                cgl.dispatch_bf16(self.grad, self.rlay.rank_dst, self.rrows, recv_x=self.grad_recv,
                                  status=self.status, scratch=self.scratch)
                rec()
            return
        cgl.get_layout(self.idx, E, R, self.cap, workspace=self.ws, out=self.lay, status=self.status)
        rec()
        if wl.fp8:
            cgl.dispatch_fp8(self.x, self.lay.dst_pos, self.rows, recv_x=self.recv_x,
                             recv_scale=self.recv_scale, status=self.status, pow2_scales=self.pow2,
                             scratch=self.scratch)
        else:
            cgl.dispatch_bf16(self.x, self.lay.dst_pos, self.rows, recv_x=self.recv_x,
                              status=self.status, scratch=self.scratch)
        rec()
        cgl.combine(self.y, self.lay.dst_pos, self.w, out=self.out, status=self.status)
        rec()
        if wl.with_grad:
            if self.full_backward:
                cgl.combine_backward(self.grad, self.y, self.lay.dst_pos, self.w, grad_y=self.grad_recv,
                                     grad_w=self.grad_w, status=self.status)
            else:
                cgl.dispatch_bf16(self.grad, self.lay.dst_pos, self.rows, recv_x=self.grad_recv,
                                  status=self.status, scratch=self.scratch)
            rec()

    def _event(self):
        e = self.torch.cuda.Event(enable_timing=True)
        e.record()
        return e

    def alone_calls(self):
        """(name, call, algorithmic bytes) of each kernel of the step, to time it alone."""
        cgl, wl, b = self.cgl, self.wl, self.bytes
        E, R = wl.num_experts, wl.num_ranks
        if self.dedup:
            lay_call = lambda: cgl.get_rank_layout(self.idx, E, R, self.rcap, workspace=self.ws, out=self.rlay,
                                                   status=self.status)
            dst, rows, w = self.rlay.rank_dst, self.rrows, self.w_rank
        else:
            lay_call = lambda: cgl.get_layout(self.idx, E, R, self.cap, workspace=self.ws, out=self.lay,
                                              status=self.status)
            dst, rows, w = self.lay.dst_pos, self.rows, self.w
        calls = [("layout", lay_call, b["layout"])]
        if wl.fp8:
            calls.append(("dispatch_fp8", lambda: cgl.dispatch_fp8(self.x, dst, rows, recv_x=self.recv_x,
                                                                   recv_scale=self.recv_scale, status=self.status,
                                                                   pow2_scales=self.pow2, scratch=self.scratch),
                          b["dispatch_fp8"]))
            if self.layout_dispatch:
                calls.append(("layout+dispatch_fp8", lambda: cgl.layout_dispatch_fp8(
                    self.idx, self.x, E, R, self.cap, out=self.lay, recv_x=self.recv_x, recv_scale=self.recv_scale,
                    workspace=self.ws, status=self.status, pow2_scales=self.pow2), b["layout"] + b["dispatch_fp8"]))
        else:
            calls.append(("dispatch_bf16", lambda: cgl.dispatch_bf16(self.x, dst, rows, recv_x=self.recv_x,
                                                                     status=self.status, scratch=self.scratch),
                          b["dispatch_bf16"]))
        calls.append(("combine", lambda: cgl.combine(self.y, dst, w, out=self.out, status=self.status),
                      b["combine"]))
        if wl.with_grad and not self.dedup:
            n, h, k = wl.num_tokens, wl.hidden, wl.topk
            if self.full_backward:
                calls.append(("combine_backward", lambda: cgl.combine_backward(
                    self.grad, self.y, self.lay.dst_pos, self.w, grad_y=self.grad_recv, grad_w=self.grad_w,
                    status=self.status), 2 * n * h + 4 * n * k * h + 12 * n * k))
            else:
                calls.append(("combine_backward", lambda: cgl.dispatch_bf16(
                    self.grad, self.lay.dst_pos, self.rows, recv_x=self.grad_recv, status=self.status,
                    scratch=self.scratch), b["dispatch_bf16"]))
        return calls


def copy_probe(dev, nbytes: int = 1 << 30, reps: int = 10):
    """HBM copy bandwidth of this device, read + write bytes (a device-to-device
    tensor copy of nbytes, timed with CUDA events after two warm-up copies):
    context for the roofline when no measured peak is on file."""
    import torch

    a = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    b = torch.empty_like(a)
    a.fill_(1)
    for _ in range(2):
        b.copy_(a)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record()
    for _ in range(reps):
        b.copy_(a)
    e1.record()
    torch.cuda.synchronize(dev)
    gbs = 2 * nbytes * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del a, b
    torch.cuda.empty_cache()
    return gbs


def time_alone(step: GpuStep, reps: int, peak: float):
    """Each kernel of the step launched back to back: a CUDA graph of 20 launches
    (captured on a side stream after 3 eager warm-up launches) replayed until
    about `reps` launches, between two CUDA events, so host launch overhead
    does not count.  µs per launch, GB/s of algorithmic bytes and the fraction
    of the measured peak.  Inputs exceed L2 at the HBM-bound sizes."""
    import torch

    per_graph = 20
    replays = max(1, reps // per_graph)
    out = {}
    for name, call, nbytes in step.alone_calls():
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(3):
                call()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(per_graph):
                call()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(replays):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        us = e0.elapsed_time(e1) / (replays * per_graph) * 1e3
        gbs = nbytes / (us * 1e-6) / 1e9
        out[name] = {"us": us, "bytes": nbytes, "gbs": gbs, "frac_of_peak": gbs / peak}
    return out


def graph_chunk(steps: int, cap: int = 20) -> int:
    """Steps captured per CUDA graph in the timed passes: the largest divisor
    of `steps` up to `cap`, so that exactly `steps` steps run.  Inside one graph
    consecutive steps follow each other as launches of one stream do (each
    kernel may start while the previous one drains); between two replays every
    replay pays the graph launch, which at the decode shape is as long as a
    kernel."""
    for s in range(min(cap, steps), 0, -1):
        if steps % s == 0:
            return s
    return 1


def capture_step(step: GpuStep, nsteps: int = 1):
    """`nsteps` steps' launches captured into one CUDA graph (on a side stream, after two eager runs)."""
    import torch

    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(2):
            step.run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(nsteps):
            step.run()
    torch.cuda.synchronize()
    return g


def time_phase_graphs(step: GpuStep, steps: int):
    """Per-phase step time without events between kernels.

    The combine phase alone: a CUDA graph holding graph_chunk(steps) of the
    step's combine launches, replayed to `steps` launches between two events
    (its input, the expert outputs, is larger than L2, so back-to-back
    launches read HBM like the step does).  The dispatch phase (layout + dispatch) is the rest of the clean
    step: ms_per_step minus that.  Timing the dispatch phase the same way would
    flatter it, because its input x (56 MiB at the prefill shape) stays in L2
    between back-to-back replays, while in the step the combine evicts it."""
    import torch

    if step.fused_decode or step.layout_dispatch:
        call = lambda: step.cgl.combine(step.y, step.lay.dst_pos, step.w, out=step.out, status=step.status)
    elif step.dedup:
        call = lambda: step.cgl.combine(step.y, step.rlay.rank_dst, step.w_rank, out=step.out, status=step.status)
    else:
        call = lambda: step.cgl.combine(step.y, step.lay.dst_pos, step.w, out=step.out, status=step.status)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            call()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    chunk = graph_chunk(steps)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(chunk):
            call()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps // chunk):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / steps


def _twin(step: GpuStep) -> GpuStep:
    """A second set of device buffers for the same step (inputs, workspace,
    outputs); the host copies fill its inputs, so only derived inputs are cloned."""
    import copy

    import torch

    t = copy.copy(step)
    for name in ("x", "idx", "w", "y", "grad", "ws", "recv_x", "recv_scale", "grad_recv", "grad_w", "out"):
        v = getattr(step, name, None)
        if isinstance(v, torch.Tensor):
            setattr(t, name, torch.empty_like(v))
    t.status = step.cgl.new_status(step.dev)
    t.scratch = step.cgl.new_scratch(step.dev)
    for name in ("lay", "rlay"):
        v = getattr(step, name, None)
        if v is not None:
            setattr(t, name, type(v)(*[torch.empty_like(f) if isinstance(f, torch.Tensor) else f for f in v]))
    if getattr(step, "w_rank", None) is not None:
        t.w_rank = step.w_rank.clone()
    return t


def run_e2e(step: GpuStep, steps: int):
    """Same step through the public API with host buffers: pinned H2D of the
    step's inputs, the kernels, D2H of the combined output and the counts.
    Two sets of device buffers and three streams (copy in, compute, copy out),
    so the output read of step i runs while step i+1's inputs come in; every
    step still moves all of its own inputs and its result."""
    import torch

    pin = lambda t: t.cpu().pin_memory()
    hx, hidx, hw, hy = pin(step.x), pin(step.idx), pin(step.w), pin(step.y)
    hg = pin(step.grad) if step.grad is not None else None
    bufs = [step, _twin(step)]
    hout = [torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory() for _ in range(2)]
    htpe = [torch.empty(step.lay.tokens_per_expert.shape, dtype=torch.int32).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in (hx, hidx, hw, hy) + ((hg,) if hg is not None else ()))
    d2h = hout[0].numel() * hout[0].element_size() + htpe[0].numel() * 4
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        j = i % 2
        b = bufs[j]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[j])      # step i-2 has finished reading these inputs
            b.x.copy_(hx, non_blocking=True)
            b.idx.copy_(hidx, non_blocking=True)
            b.w.copy_(hw, non_blocking=True)
            b.y.copy_(hy, non_blocking=True)
            if hg is not None:
                b.grad.copy_(hg, non_blocking=True)
            ev_in[j].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[j])
            s_cmp.wait_event(ev_out[j])     # step i-2's output has been read
            b.run()
            ev_cmp[j].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[j])
            htpe[j].copy_(b.lay.tokens_per_expert, non_blocking=True)
            hout[j].copy_(b.out, non_blocking=True)
            ev_out[j].record(s_out)

    for i in range(2):
        one(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        one(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    for b in bufs[1:]:
        bits = step.cgl.status_bits(b.status)
        if bits:
            raise RuntimeError(f"device status after the e2e pass: {bits}")
    return ms, h2d, d2h


# ----------------------------------------------------------------- CPU oracle timing

def oracle_step_seconds(inp: W.Inputs, y: np.ndarray, tokens: int, reps_min_s: float, max_reps: int,
                        pow2: bool = False):
    """Time the oracle's layout + dispatch + combine on the first `tokens` tokens."""
    import oracle

    wl = inp.workload
    idx = inp.topk_idx[:tokens]
    x = inp.x[:tokens]
    w = inp.topk_w[:tokens]
    reps, t_total = 0, 0.0
    while reps < max_reps and (reps == 0 or t_total < reps_min_s):
        t0 = time.perf_counter()
        L = oracle.get_layout(idx, wl.num_experts, wl.num_ranks, 0)
        rows = idx.size
        if wl.fp8:
            oracle.dispatch_fp8(x, L.dst_pos, rows, pow2_scales=pow2)
        else:
            oracle.dispatch_bf16(x, L.dst_pos, rows)
        oracle.combine(y[:rows], L.dst_pos, w)
        if wl.with_grad:
            oracle.dispatch_bf16(inp.grad[:tokens], L.dst_pos, rows)
        t_total += time.perf_counter() - t0
        reps += 1
    return t_total, reps


def step_bytes_for(wl: W.Workload, tokens: int) -> int:
    b = W.algorithmic_bytes(wl, tokens)
    tot = b["layout"] + b["combine"] + (b["dispatch_fp8"] if wl.fp8 else b["dispatch_bf16"])
    if wl.with_grad:
        tot += b["dispatch_bf16"]
    return tot


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------- arms

def base_line(args, wl, n_gpus):
    return {
        "metric": METRIC, "unit": "GB/s", "n_gpus": n_gpus, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("f32 arithmetic; bf16 x in, e4m3 + f32 scale rows out, bf16 combine" if wl.fp8
                  else "f32 arithmetic; bf16 rows"), "data": "synthetic",
        "config": {
            "workload": workload_label(wl, getattr(args, "dedup", False), getattr(args, "ue8m0", False)),
            "num_tokens": wl.num_tokens, "hidden": wl.hidden,
            "num_experts": wl.num_experts, "num_groups": wl.num_groups, "topk_group": wl.topk_group,
            "topk": wl.topk, "num_ranks": wl.num_ranks,
            "storage": ("x bf16 -> e4m3 rows + f32 1x128 scales; combine bf16 in, f32 accumulate, bf16 out"
                        if wl.fp8 else "x bf16 rows; combine bf16; combine-backward bf16 rows"),
            "parallelism": f"replicas x{n_gpus} (logical EP ranks inside each GPU)",
            "l2": "no flush: inputs larger than L2 (each step touches "
                  f"{step_bytes_for(wl, wl.num_tokens) / 1e9:.2f} GB)",
            "seed": args.seed,
        },
    }


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle

    wl = W.WORKLOADS[args.workload]
    inp = W.make_inputs(wl, args.seed)
    y = W.expert_outputs(inp.topk_idx.size, wl.hidden, args.seed)
    threads = oracle.set_threads(cpu_threads())
    # size the per-step sample so that warmup + steps end within ~2 minutes
    t_full, _ = oracle_step_seconds(inp, y, wl.num_tokens, 0.0, 1, args.ue8m0)
    budget = 120.0 / max(1, args.steps + args.warmup)
    tokens = wl.num_tokens if t_full <= budget else max(16, int(wl.num_tokens * budget / t_full) // 16 * 16)
    for _ in range(args.warmup):
        oracle_step_seconds(inp, y, tokens, 0.0, 1, args.ue8m0)
    times = []
    for _ in range(args.steps):
        t, _ = oracle_step_seconds(inp, y, tokens, 0.0, 1, args.ue8m0)
        times.append(t)
    sec = sum(times) / len(times)
    gbs = step_bytes_for(wl, tokens) / sec / 1e9
    line = base_line(args, wl, world)
    sample = (f"first {tokens} of {wl.num_tokens} tokens per step (layout + "
              f"{'dispatch_fp8' if wl.fp8 else 'dispatch_bf16'} + combine), C oracle, OpenMP over tokens")
    line.update({
        "impl": "reference", "value": gbs, "ms_per_step": sec * 1e3,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    })
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")
    wl = W.WORKLOADS[args.workload]
    if args.num_tokens:
        import dataclasses

        wl = dataclasses.replace(wl, num_tokens=args.num_tokens)
    step = GpuStep(wl, rank_seed(args.seed, rank), dev, dedup=args.dedup, full_backward=args.full_backward,
                   fused_decode=args.fused_decode, split_layout=args.split_layout, pow2_scales=args.ue8m0,
                   fused_layout=args.fused_layout)
    phases = step.kernels()

    chunk = graph_chunk(args.steps)
    graph = None if args.no_graph else capture_step(step)                  # one step: the warm-up
    graph_k = None if args.no_graph else capture_step(step, chunk)         # `chunk` steps: the timed pass
    for _ in range(args.warmup):
        if graph is not None:
            graph.replay()
        else:
            step.run()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if (rank == 0 and not args.no_clocks) else None
    if sampler:
        sampler.start()
        time.sleep(0.3)   # let nvidia-smi start sampling before the timed region
    # timed region: K steps, one event on each side, nothing between the kernels
    # (an event between two kernels stops the next one from launching early);
    # by default K / chunk replays of a CUDA graph holding `chunk` steps' launches
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record()
    if graph_k is not None:
        for _ in range(args.steps // chunk):
            graph_k.replay()
    else:
        for _ in range(args.steps):
            step.run()
    e_end.record()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    barrier()
    ms = e_start.elapsed_time(e_end) / args.steps

    # per-kernel durations: a second pass of K steps with an event after every
    # kernel; each duration includes the launch gap those events add
    evs = []
    for _ in range(args.steps):
        ev = []
        step.run(ev)
        evs.append(ev)
    torch.cuda.synchronize()
    barrier()
    per_phase = [0.0] * len(phases)
    for ev in evs:
        for i in range(len(phases)):
            per_phase[i] += ev[i].elapsed_time(ev[i + 1])
    per_phase = [v / args.steps for v in per_phase]
    ms_instr = evs[0][0].elapsed_time(evs[-1][-1]) / args.steps
    ms_comb = time_phase_graphs(step, args.steps) if not step.wl.with_grad else None
    red = max_over_ranks([ms, ms_instr, ms_comb or 0.0] + per_phase, device=dev)
    ms, ms_instr, ms_comb, per_phase = red[0], red[1], (red[2] if ms_comb is not None else None), red[3:]
    status_bits = step.cgl.status_bits(step.status)

    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h = run_e2e(step, args.e2e_steps)
        e2e_ms = max_over_ranks([e2e_ms], device=dev)[0]
        e2e = {"value": step.step_bytes() * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "overlap": "two device buffer sets on copy-in / compute / copy-out streams: "
                          "step i's D2H overlaps step i+1's H2D"}

    if rank != 0:
        barrier()
        return 0
    peak, peak_src = hbm_peak()
    alone = time_alone(step, min(args.steps, 200), peak)
    status_bits = sorted(set(status_bits) | set(step.cgl.status_bits(step.status)))
    srcs = {"combine": "combine.cu", "dispatch_fp8": "dispatch.cu", "dispatch_bf16": "dispatch.cu",
            "layout": "layout.cu", "layout+dispatch_fp8": "layout.cu", "combine_backward": "combine_backward.cu"}
    # the traffic records were taken at the prefill shape, expert-keyed path
    at_prefill = (wl.name == "prefill" and wl.num_tokens == W.WORKLOADS["prefill"].num_tokens and not args.dedup)
    kernels = {}
    for (name, launches, nbytes), t in zip(phases, per_phase):
        gbs = nbytes / (t * 1e-3) / 1e9
        kernels[name] = {"us": t * 1e3, "launches_per_step": launches, "bytes": nbytes,
                         "gbs": gbs, "frac_of_peak": gbs / peak,
                         "traffic": traffic_for(name, srcs.get(name, "layout.cu")) if at_prefill else None}
    dom = max(phases, key=lambda p: p[2])[0]
    src = srcs.get(dom, "layout.cu")
    roof = {"kernel": dom, "bound": "hbm", "achieved": kernels[dom]["gbs"], "peak": peak,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, copy read+write)" if peak_src == "measured" else "fallback 6.65 TB/s",
            "unit": "GB/s", "frac": kernels[dom]["gbs"] / peak,
            "traffic": traffic_for(dom, src) if at_prefill else None,
            "bytes_per_launch": kernels[dom]["bytes"],
            "timing": ("in the step: CUDA events on the launching stream around each launch of the kernel over "
                       "the K steps of the instrumented pass (the gap the events add included)")}
    line = base_line(args, wl, world)
    value = step.step_bytes() * world / (ms * 1e-3) / 1e9
    line.update({
        "value": value, "ms_per_step": ms, "roofline": roof, "kernels": kernels,
        "kernels_alone": alone,
        "kernels_alone_timing": ("each kernel of the step alone: a CUDA graph of 20 back-to-back launches replayed "
                                 "to about min(K, 200) launches between two CUDA events, after 3 warm-up launches"),

        "gpu_launches": args.steps * sum(p[1] for p in phases),
        "launch": "eager" if args.no_graph else (f"CUDA graph of {chunk} steps, replayed K/{chunk} times (warm-up: a "
                                                 "one-step graph; e2e and per-kernel passes eager)"),
        "kernel_timing": ("per-kernel us from a second pass of the same K steps with a CUDA event "
                          f"after every kernel ({ms_instr * 1e3:.1f} us/step there vs {ms * 1e3:.1f} clean); "
                          "each includes the launch gap the events add"),
        "clocks": clocks, "device_status": status_bits or "ok",
    })
    if peak_src != "measured":   # no measured peak on file: the same kind of copy, measured here
        probe = copy_probe(dev)
        line["hbm_copy_probe"] = {"gbs": probe, "dominant_frac_of_probe": roof["achieved"] / probe,
                                  "how": "device-to-device copy of 1 GiB, read + write bytes, CUDA events, "
                                         "after the timed passes"}
    if ms_comb is not None:
        nb = {n: b for n, _, b in phases}
        comb_b = nb.get("combine", 0)
        line.update({
            "dispatch_us": (ms - ms_comb) * 1e3, "combine_us": ms_comb * 1e3,
            "dispatch_gbs": (step.step_bytes() - comb_b) / ((ms - ms_comb) * 1e-3) / 1e9,
            "combine_gbs": comb_b / (ms_comb * 1e-3) / 1e9,
            "phase_timing": ("no event between kernels: combine_us = the step's combine launch alone, K launches "
                             "from a CUDA graph of the same chunk of launches as the step's (its expert-output "
                             "input exceeds L2); dispatch_us = "
                             "ms_per_step - combine_us (layout and dispatch, with the transitions of the step); "
                             "the instrumented per-kernel split is under 'kernels'"),
        })
    if e2e:
        line["e2e"] = e2e
    if not args.no_cpu_baseline and world == 1 and not args.dedup:
        import oracle

        threads = oracle.set_threads(cpu_threads())
        t, reps = oracle_step_seconds(step.host, step.host_y, wl.num_tokens, args.cpu_seconds, 1000, args.ue8m0)
        gbs = step_bytes_for(wl, wl.num_tokens) * reps / t / 1e9
        line["cpu_baseline"] = {
            "value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{reps} full {wl.num_tokens}-token steps (same inputs), {t:.1f} s, C oracle with OpenMP over tokens"}
    print(json.dumps(line), flush=True)
    barrier()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=W.WORKLOAD_ORDER, default="prefill")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--num-tokens", type=int, default=0,
                    help="override the workload's token count (e.g. small cases for profiling)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--dedup", action="store_true",
                    help="per-rank deduplicated dispatch: one copy per (token, rank), rank-sum combine")
    ap.add_argument("--full-backward", action="store_true",
                    help="bf16 workload: weighted combine backward with grad_w instead of the plain re-dispatch")
    ap.add_argument("--fused-decode", action="store_true",
                    help="layout and FP8 dispatch in one launch (batches of at most 1024 token-slot pairs)")
    ap.add_argument("--split-layout", action="store_true",
                    help="FP8: cgl_get_layout and cgl_dispatch_fp8 as two calls at every size (the default above "
                         "one token per SM)")
    ap.add_argument("--fused-layout", action="store_true",
                    help="FP8: cgl_layout_dispatch_fp8 at every size (at prefill sizes one fused kernel)")
    ap.add_argument("--no-graph", action="store_true", help="launch each timed step eagerly instead of replaying a CUDA graph")
    ap.add_argument("--ue8m0", action="store_true", help="FP8: power-of-two (UE8M0) scales instead of amax / 448")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    try:
        return run_ours(args)
    finally:
        import torch.distributed as dist

        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
