#!/usr/bin/env python
"""Throughput of the quantised gated Delta-rule decode step on B200.

A *step* is one decode step of one linear-attention layer for a batch of
requests: for every (request, head) read the packed state, reconstruct it,
apply the gated Delta update, emit y = X^T q, refit the scales and write the
state back packed (readout kernel on the main stream, fit + pack kernel on a
second stream).  The metric is head-updates per second (one head-update = one
(request, head) state step), plus the HBM bandwidth this implies.

Default workload (fits one GPU): 64 requests x 32 heads, d_k = d_v = 128,
bf16 q/k/v, scalar gates, per-head 4/6/8-bit plan averaging 6 bits plus one
FP16 pivot head.  Inputs are synthetic and seeded (``workload.py``).

Consecutive steps cycle through several layers' state pools whose total size
is at least twice the 126 MB L2, so every step reads its state from HBM; as
in a model, layer l's fit + pack overlaps layer l+1's readout.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl stepq|reference]
Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
GPU (weak scaling; the step has no cross-GPU exchange) and rank 0 prints one
JSON line with the whole-job throughput, timed on the device as the max over
ranks.
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workload as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FIT_STREAMS = 0             # side streams the layers' fits take in turn (0: one per layer pool)
MAIN_PRIORITY = -5          # readout stream priority (lower is higher; mapped into the device's range)
SMS, FP32_LANES = 148, 128
METRIC = "quantized state-step throughput (head-updates/s) and HBM GB/s vs B200 peak"
UNIT = "head-updates/s"
ALU_OPS_PER_ENTRY = 60     # fp32 ops per quantised state entry in the fit + pack kernel
ALU_OPS_PER_ENTRY_UNIFORM = 13  # the same without the column search (per-row scales only)
PIVOT_OPS_PER_ENTRY = 6


# quantiser variants: (fit mode, uniform width or None for the plan's widths,
# FP16 pivots kept).  "spatial", "temporal" and "nopivot" are the ablations of
# the method: the dual-axis fit alone on uniform widths, the lifetime-aware
# widths alone with per-row scales, and the full method without pivots.
MODES = {
    "stepquant": (W.MODE_STEPQUANT, None, True),
    "uniform8": (W.MODE_UNIFORM, 8, False),
    "uniform6": (W.MODE_UNIFORM, 6, False),
    "spatial": (W.MODE_STEPQUANT, 6, False),
    "temporal": (W.MODE_UNIFORM, None, True),
    "nopivot": (W.MODE_STEPQUANT, None, False),
    # offline calibration (calibrated_plan): estimated row-impact weights,
    # allocated widths, or both
    "impact": (W.MODE_STEPQUANT, None, True),
    "allocated": (W.MODE_STEPQUANT, None, True),
    "calibrated": (W.MODE_STEPQUANT, None, True),
}

CAL_STEPS, CAL_SNAPSHOTS, CAL_REQUESTS = 64, 4, 16
CAL_STEP_BASE = 1 << 24     # calibration inputs: step indices no decode run uses


def calibrated_plan(cfg, what):
    """The workload's plan with calibrated row-impact weights ("impact"),
    widths and pivots from the lifetime-aware allocation ("allocated"), or
    both ("calibrated": the weights first, then the allocation measured with
    them).

    Calibration data: CAL_REQUESTS requests numbered after the workload's own,
    stepped CAL_STEPS times by the fp32 kernel from their seeded S0 with
    seeded inputs of step indices CAL_STEP_BASE + t; the row-impact scores
    from every step's inputs, the distortion from CAL_SNAPSHOTS snapshots of
    the states; lifetimes from the plan's gates; the budget and the pivot
    count of the workload's own recipe."""
    import torch

    import quantized_delta_rule_decode_b200 as S
    from quantized_delta_rule_decode_b200 import calibrate
    pin = W.make_plan(cfg)
    d, H = cfg.d, cfg.heads
    reqs = list(range(cfg.requests, cfg.requests + CAL_REQUESTS))
    Sx = torch.from_numpy(W.initial_state(cfg, reqs)).cuda()
    slots = torch.arange(len(reqs), dtype=torch.int32, device="cuda")
    dt = torch.bfloat16 if cfg.bf16_inputs else torch.float32
    y = torch.empty((len(reqs), H, d), dtype=torch.float32, device="cuda")
    states, inputs = [], []
    every = CAL_STEPS // CAL_SNAPSHOTS
    for t in range(CAL_STEPS):
        si = W.step_inputs(cfg, CAL_STEP_BASE + t, pin, reqs)
        q, k, v = (torch.from_numpy(a).to(dt).cuda() for a in (si.q, si.k, si.v))
        beta, gate = torch.from_numpy(si.beta).cuda(), torch.from_numpy(si.gate).cuda()
        inputs.append((q, k, beta, gate))
        S.stepq_fp32_step(Sx, slots, q, k, v, beta, gate, y, cfg.gate_kind)
        if (t + 1) % every == 0:
            states.append(Sx.clone())
    w = pin.w
    if what in ("impact", "calibrated"):
        w = calibrate.impact_weights(cfg.gate_kind, d, H, inputs)
    bits = pin.bits
    if what in ("allocated", "calibrated"):
        g = np.asarray(pin.gate, np.float32)
        if cfg.unit_kind == W.UNIT_ROW:
            gates = (g.reshape(-1) if cfg.gate_kind == W.GATE_DIAG else np.repeat(g, d))[None, :, None]
        else:
            gates = g[None] if g.ndim == 2 else g[None, :, None]
        n_piv = int(np.sum(pin.bits == 16))
        bits, _, _ = calibrate.calibrate_bits(d, d, H, cfg.gate_kind, cfg.unit_kind, w, states, gates,
                                              cfg.budget, n_piv)
    return W.PlanInputs(bits=bits, w=w, half_life=pin.half_life, gate=pin.gate)


def mode_plan(cfg, mode):
    m, ub, piv = MODES[mode]
    if mode in ("impact", "allocated", "calibrated"):
        return m, calibrated_plan(cfg, mode)
    return m, W.make_plan(cfg, uniform_bits=ub, pivots=piv)


def parse():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["stepq", "reference"], default="stepq")
    ap.add_argument("--config", choices=W.CONFIG_ORDER, default="gdn")
    ap.add_argument("--mode", choices=list(MODES), default="stepquant")
    ap.add_argument("--e2e-steps", type=int, default=0,
                    help="steps of the end-to-end pass (0: as many as the headline's --steps)")
    ap.add_argument("--fp32-steps", type=int, default=2000)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--kernel-steps", type=int, default=500,
                    help="steps of the separate pass that times each kernel inside the overlapped step")
    ap.add_argument("--config-steps", type=int, default=300,
                    help="steps of each further workload measured into the line's 'configs' (0: none)")
    ap.add_argument("--isolated-steps", type=int, default=500,
                    help="steps of the per-kernel timing with each kernel alone")
    ap.add_argument("--fit-streams", type=int, default=FIT_STREAMS,
                    help="side streams the layers' fit + pack launches take in turn (0: one per layer pool)")
    ap.add_argument("--main-priority", type=int, default=MAIN_PRIORITY,
                    help="priority of the readout stream (0: the default stream priority)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="skip the CUDA-graph replay of the same steps")
    ap.add_argument("--drift", action="store_true",
                    help="instead of the throughput line: quantised rollouts vs the fp32 rollout")
    ap.add_argument("--lifetime-study", action="store_true",
                    help="instead of the throughput line: per-unit accumulated error of quantised rollouts "
                         "vs the fp32 rollout, and its Spearman correlation with the unit's gate half-life")
    ap.add_argument("--timeline", action="store_true",
                    help="instead of the throughput line: start/end of each kernel of a few overlapped steps")
    ap.add_argument("--pipeline", action="store_true",
                    help="instead of the throughput line: per-token time of a layer stack with GEMM proxies")
    ap.add_argument("--drift-arms", default="stepquant,impact,allocated,calibrated,temporal,uniform8,uniform6",
                    help="comma-separated quantiser variants of the drift report")
    ap.add_argument("--drift-steps", type=int, default=0,
                    help="steps of the drift report (0: the workload's own step count)")
    ap.add_argument("--serial", action="store_true",
                    help="also time the step with both kernels on one stream, one layer")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
class Dist:
    """One process per GPU (torchrun env); NCCL on GPUs, gloo for host-only use.

    The step has no exchange: ranks meet only at the timing barriers and for
    the max-over-ranks reduction of the measured times."""

    def __init__(self, n=None, backend="nccl", timeout_s=120.0):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = None
        if self.world > 1:
            import datetime

            import torch
            import torch.distributed as dist
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            # a rank that is gone makes the others' next collective fail within this
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
            self.pg = dist

    def _device(self):
        return "cuda" if self.backend == "nccl" else "cpu"

    def barrier(self):
        if self.pg:
            import torch
            if self.backend == "nccl":
                self.pg.barrier(device_ids=[self.local])
                torch.cuda.synchronize()
            else:
                self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self._device())
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None
        self.idx = gpu_index
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-i", str(gpu_index), "-lms", "100"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = []
        with open(self.f.name) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# ---------------------------------------------------------------------------
# the workload on the device
# ---------------------------------------------------------------------------
def algorithmic_bytes(cfg, pin, slot_bytes_per_head):
    """Bytes one step must move: packed state read + written, q,k,v, beta, gate, y."""
    d = cfg.d
    per_req = 2 * sum(slot_bytes_per_head)
    qkv = 3 * d * (2 if cfg.bf16_inputs else 4)
    gate = 4 * d if cfg.gate_kind == W.GATE_DIAG else 4
    per_head_io = qkv + 4 + gate + 4 * d
    return cfg.requests * (per_req + cfg.heads * per_head_io)


def readout_bytes(cfg, slot_bytes_per_head):
    d = cfg.d
    qkv = 3 * d * (2 if cfg.bf16_inputs else 4)
    gate = 4 * d if cfg.gate_kind == W.GATE_DIAG else 4
    return cfg.requests * (sum(slot_bytes_per_head) + cfg.heads * (qkv + 4 + gate + 4 * d))


def fit_alu_ops(cfg, pin, mode=W.MODE_STEPQUANT):
    d = cfg.d
    if cfg.unit_kind == W.UNIT_HEAD:
        q_rows = sum(d for b in pin.bits if b != 16)
        p_rows = sum(d for b in pin.bits if b == 16)
    else:
        q_rows = int(np.sum(pin.bits != 16))
        p_rows = int(np.sum(pin.bits == 16))
    per = ALU_OPS_PER_ENTRY if mode == W.MODE_STEPQUANT else ALU_OPS_PER_ENTRY_UNIFORM
    return cfg.requests * d * (q_rows * per + p_rows * PIVOT_OPS_PER_ENTRY)


class DeviceWorkload:
    def __init__(self, cfg, mode, fit_streams=None):
        import torch

        import quantized_delta_rule_decode_b200 as S
        self.S, self.cfg = S, cfg
        self.mode, self.pin = mode_plan(cfg, mode)
        d, H, R = cfg.d, cfg.heads, cfg.requests
        self.plan = S.stepq_plan_create(d, d, H, cfg.gate_kind, cfg.unit_kind, self.mode,
                                        self.pin.bits, self.pin.w)
        self.slot_bytes = S.stepq_plan_slot_bytes(self.plan)
        self.head_bytes = [S.stepq_plan_head_layout(self.plan, h)[1] for h in range(H)]
        self.nslots = cfg.pool_slots
        pool_bytes = self.nslots * self.slot_bytes
        # at least two layers, as in any model: consecutive calls go to
        # different layers' pools, so one layer's fit can overlap the next
        # layer's readout; more when needed to make the cycled pools larger
        # than twice the L2
        self.layers = max(2, math.ceil(2 * L2_BYTES / pool_bytes))
        self.slots_np = W.slot_indices(cfg)
        self.slots = torch.from_numpy(self.slots_np).cuda()
        # pack S0 into layer 0, chunk by chunk, then copy into the other layers
        self.pools = []
        for layer in range(self.layers):
            buf = torch.zeros(pool_bytes, dtype=torch.uint8, device="cuda")
            self.pools.append(S.stepq_pool_alloc(self.plan, self.nslots, buf))
        chunk = max(1, (256 << 20) // (H * d * d * 4))
        for r0 in range(0, R, chunk):
            rr = list(range(r0, min(R, r0 + chunk)))
            X = torch.from_numpy(W.initial_state(cfg, rr)).cuda()
            S.stepq_pack(self.plan, self.pools[0], self.slots[r0:r0 + len(rr)].contiguous(), X)
            del X
        for p in self.pools[1:]:
            p.buf.copy_(self.pools[0].buf)
        torch.cuda.synchronize()
        # ring of fresh step inputs
        self.ring = []
        dt = torch.bfloat16 if cfg.bf16_inputs else torch.float32
        for step in range(16):
            si = W.step_inputs(cfg, step, self.pin)
            self.ring.append(dict(
                q=torch.from_numpy(si.q).to(dt).cuda(), k=torch.from_numpy(si.k).to(dt).cuda(),
                v=torch.from_numpy(si.v).to(dt).cuda(), beta=torch.from_numpy(si.beta).cuda(),
                gate=torch.from_numpy(si.gate).cuda(), host=si))
        self.dtype_code = S.DTYPE_BF16 if cfg.bf16_inputs else S.DTYPE_F32
        self.y = torch.empty((R, H, d), dtype=torch.float32, device="cuda")
        # one delta workspace per layer: layer l's fit may still read it while
        # layer l+1's readout runs
        self.ws = [torch.empty(S.stepq_workspace_bytes(self.plan, R), dtype=torch.uint8, device="cuda")
                   for _ in range(self.layers)]
        # The readout (the step's critical path: it produces y) runs on a
        # high-priority stream, so that its CTAs take SMs ahead of the fits as
        # soon as any retire; each layer's fit + pack runs on a side stream of
        # its own (or one of `fit_streams` taken in turn), so that one layer's
        # fit can start in the tail of the previous layer's.
        fs = FIT_STREAMS if fit_streams is None else fit_streams
        self.fit_streams = self.layers if fs <= 0 else min(fs, self.layers)
        self.main = torch.cuda.Stream(priority=MAIN_PRIORITY) if MAIN_PRIORITY else torch.cuda.current_stream()
        self.sides = [torch.cuda.Stream() for _ in range(self.fit_streams)]
        self.side = self.sides[0]
        L = S.load_library()
        self.L = L
        P = ctypes.c_void_p
        ms = P(self.main.cuda_stream)
        sp = P(self.slots.data_ptr())
        self.step_args, self.read_args, self.fit_args = [], [], []
        for layer in range(self.layers):
            ss = P(self.side_of_layer(layer).cuda_stream)
            wsp, wsb = P(self.ws[layer].data_ptr()), self.ws[layer].numel()
            for t in self.ring:
                common = (self.plan.handle, self.pools[layer].handle, sp, R, self.dtype_code)
                io = (P(t["q"].data_ptr()), P(t["k"].data_ptr()), P(t["v"].data_ptr()),
                      P(t["beta"].data_ptr()), P(t["gate"].data_ptr()), P(self.y.data_ptr()),
                      wsp, wsb)
                self.step_args.append(common + io + (ms, ss))
                self.read_args.append(common + io + (ms,))
                self.fit_args.append(common + (P(t["k"].data_ptr()), P(t["gate"].data_ptr()),
                                               wsp, wsb, ss))

    def side_of_layer(self, layer):
        return self.sides[layer % len(self.sides)]

    def side_of(self, step):
        return self.side_of_layer(step % self.layers)

    def args_index(self, step):
        return (step % self.layers) * 16 + (step % 16)

    def run_step(self, step):
        rc = self.L.stepq_decode_step(*self.step_args[self.args_index(step)])
        if rc:
            raise RuntimeError(self.L.stepq_last_error().decode())

    def run_step_timed(self, step, ev):
        """Same work as run_step, with CUDA events around each kernel on its own stream."""
        i = self.args_index(step)
        ev[0].record(self.main)
        if self.L.stepq_decode_readout(*self.read_args[i]):
            raise RuntimeError(self.L.stepq_last_error().decode())
        ev[1].record(self.main)
        side = self.side_of(step)
        side.wait_event(ev[1])
        ev[2].record(side)
        if self.L.stepq_decode_fitpack(*self.fit_args[i]):
            raise RuntimeError(self.L.stepq_last_error().decode())
        ev[3].record(side)

    def join(self):
        for side in self.sides:
            self.main.wait_stream(side)


def time_device(wl, steps, warmup, dist, clocks_gpu):
    """The headline: exactly `steps` plain stepq_decode_step calls between two
    events on the main stream (joined with the side stream), barrier and
    synchronize on both sides, max over ranks."""
    import torch
    for s in range(warmup):
        wl.run_step(s)
    wl.join()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    clk = Clocks(clocks_gpu)
    time.sleep(0.3)
    start.record(wl.main)
    for s in range(steps):
        wl.run_step(warmup + s)
    wl.join()
    end.record(wl.main)
    torch.cuda.synchronize()
    clocks = clk.stop()
    dist.barrier()
    ms = dist.max(start.elapsed_time(end))
    return ms, clocks


def time_kernels_overlapped(wl, steps, warmup):
    """A separate pass after the headline: the same overlapped schedule with
    CUDA events around each kernel on its own stream (the split calls
    stepq_decode_readout + stepq_decode_fitpack), for the per-kernel durations
    inside the step."""
    import torch
    for s in range(warmup):
        wl.run_step(s)
    wl.join()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for s in range(steps):
        wl.run_step_timed(warmup + s, evs[s])
    wl.join()
    torch.cuda.synchronize()
    t0 = evs[0][0]
    readout = [(t0.elapsed_time(e[0]), t0.elapsed_time(e[1])) for e in evs]
    fit = [(t0.elapsed_time(e[2]), t0.elapsed_time(e[3])) for e in evs]
    return busy_per_launch(readout), busy_per_launch(fit)


def busy_per_launch(intervals):
    """Time during which at least one of the launches was in flight, per
    launch: the union of their [start, end] intervals divided by their number.
    For launches that do not overlap this is their mean duration; for launches
    that overlap (layers' fits on different side streams) it is the time the
    kernel adds to the step per launch."""
    if not intervals:
        return 0.0
    total, cur_lo, cur_hi = 0.0, None, None
    for lo, hi in sorted(intervals):
        if cur_hi is None or lo > cur_hi:
            if cur_hi is not None:
                total += cur_hi - cur_lo
            cur_lo, cur_hi = lo, hi
        else:
            cur_hi = max(cur_hi, hi)
    total += cur_hi - cur_lo
    return total / len(intervals)


def time_isolated(wl, steps, warmup):
    """Each kernel alone: readout then fit + pack on the main stream, events around each."""
    import torch
    P = ctypes.c_void_p
    ms = P(wl.main.cuda_stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for s in range(warmup + steps):
        i = wl.args_index(s)
        ev = evs[s - warmup] if s >= warmup else None
        if ev:
            ev[0].record(wl.main)
        if wl.L.stepq_decode_readout(*wl.read_args[i]):
            raise RuntimeError(wl.L.stepq_last_error().decode())
        if ev:
            ev[1].record(wl.main)
        if wl.L.stepq_decode_fitpack(*(wl.fit_args[i][:-1] + (ms,))):
            raise RuntimeError(wl.L.stepq_last_error().decode())
        if ev:
            ev[2].record(wl.main)
    torch.cuda.synchronize()
    rd = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    ft = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    return rd, ft


def time_graph(wl, steps):
    """The same decode steps captured once into a CUDA graph and replayed.

    One graph holds one period of the step sequence (every layer x every
    input of the ring), both streams included; the pool views used in the
    capture are fresh, so no step waits on an event recorded outside it."""
    import torch
    S, L = wl.S, wl.L
    P = ctypes.c_void_p
    period = wl.layers * 16 // math.gcd(wl.layers, 16)
    cs = torch.cuda.Stream(priority=MAIN_PRIORITY) if MAIN_PRIORITY else torch.cuda.Stream()
    ss = [torch.cuda.Stream() for _ in range(wl.fit_streams)]
    pools = [S.stepq_pool_alloc(wl.plan, wl.nslots, p.buf) for p in wl.pools]
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    rcs = []
    with torch.cuda.stream(cs):
        g.capture_begin()
        try:
            for s in range(period):
                a = list(wl.step_args[wl.args_index(s)])
                a[1] = pools[s % wl.layers].handle
                a[-2], a[-1] = P(cs.cuda_stream), P(ss[(s % wl.layers) % len(ss)].cuda_stream)
                rcs.append(L.stepq_decode_step(*a))
            for side in ss:
                cs.wait_stream(side)
        finally:
            g.capture_end()
    if any(rcs):
        raise RuntimeError("decode step failed during graph capture: " + L.stepq_last_error().decode())
    reps = max(1, steps // period)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(cs):
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a.record(cs)
        for _ in range(reps):
            g.replay()
        b.record(cs)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / (reps * period)
    del g
    for p in pools:
        S.stepq_pool_free(p)
    cfg = wl.cfg
    return {"ms_per_step": ms, "value": cfg.requests * cfg.heads / (ms * 1e-3), "unit": UNIT,
            "steps_per_graph": period, "replays": reps, "kernel_nodes": 2 * period * reps}


def time_serial(wl, steps, warmup):
    """Both kernels on one stream, one layer after another, no overlap."""
    import torch
    for s in range(warmup):
        wl.run_step_timed(s, [torch.cuda.Event() for _ in range(4)])
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(wl.main)
    for s in range(steps):
        i = wl.args_index(warmup + s)
        args = list(wl.step_args[i])
        args[-1] = args[-2]   # side stream := main stream
        wl.L.stepq_decode_step(*args)
    b.record(wl.main)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def time_e2e(wl, steps, warmup):
    """Through the C ABI with host buffers: H2D of each step's inputs, the step, D2H of y."""
    import torch
    S, cfg = wl.S, wl.cfg
    R, H, d = cfg.requests, cfg.heads, cfg.d
    dt = torch.bfloat16 if cfg.bf16_inputs else torch.float32
    ring = []
    for t in wl.ring:
        si = t["host"]
        ring.append(dict(q=torch.from_numpy(si.q).to(dt).pin_memory(),
                         k=torch.from_numpy(si.k).to(dt).pin_memory(),
                         v=torch.from_numpy(si.v).to(dt).pin_memory(),
                         beta=torch.from_numpy(si.beta).pin_memory(),
                         gate=torch.from_numpy(si.gate).pin_memory()))
    y = torch.empty((R, H, d), dtype=torch.float32).pin_memory()
    # staging per layer: a layer's fit reads k and gate from it after the call returns
    wss = [torch.empty(S.stepq_host_workspace_bytes(wl.plan, R, wl.dtype_code), dtype=torch.uint8,
                       device="cuda") for _ in range(wl.layers)]
    P = ctypes.c_void_p
    args = []
    for layer in range(wl.layers):
        ws = wss[layer]
        for t in ring:
            args.append((wl.plan.handle, wl.pools[layer].handle, P(wl.slots.data_ptr()), R, wl.dtype_code,
                         P(t["q"].data_ptr()), P(t["k"].data_ptr()), P(t["v"].data_ptr()),
                         P(t["beta"].data_ptr()), P(t["gate"].data_ptr()), P(y.data_ptr()),
                         P(ws.data_ptr()), ws.numel(), P(wl.main.cuda_stream),
                         P(wl.side_of_layer(layer).cuda_stream)))
    for s in range(warmup):
        wl.L.stepq_decode_step_host(*args[wl.args_index(s)])
    wl.join()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(wl.main)
    for s in range(steps):
        if wl.L.stepq_decode_step_host(*args[wl.args_index(warmup + s)]):
            raise RuntimeError(wl.L.stepq_last_error().decode())
    wl.join()
    b.record(wl.main)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    t0 = ring[0]
    h2d = sum(t0[k].numel() * t0[k].element_size() for k in ("q", "k", "v", "beta", "gate"))
    d2h = y.numel() * y.element_size()
    return ms, h2d, d2h


def time_fp32(cfg, pin, steps, warmup):
    import torch

    import quantized_delta_rule_decode_b200 as S
    d, H, R = cfg.d, cfg.heads, cfg.requests
    per_layer = cfg.pool_slots * H * d * d * 4
    layers = max(1, math.ceil(2 * L2_BYTES / per_layer))
    if layers * per_layer > 40e9:
        return None
    pools = [torch.zeros((cfg.pool_slots, H, d, d), dtype=torch.float32, device="cuda") for _ in range(layers)]
    slots = torch.from_numpy(W.slot_indices(cfg)).cuda()
    dt = torch.bfloat16 if cfg.bf16_inputs else torch.float32
    si = W.step_inputs(cfg, 0, pin)
    q, k, v = (torch.from_numpy(a).to(dt).cuda() for a in (si.q, si.k, si.v))
    beta, gate = torch.from_numpy(si.beta).cuda(), torch.from_numpy(si.gate).cuda()
    y = torch.empty((R, H, d), dtype=torch.float32, device="cuda")
    L = S.load_library()
    P = ctypes.c_void_p
    st = torch.cuda.current_stream()
    code = S.DTYPE_BF16 if cfg.bf16_inputs else S.DTYPE_F32
    args = [(d, d, H, cfg.gate_kind, code, P(p.data_ptr()), cfg.pool_slots, P(slots.data_ptr()), R,
             P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(beta.data_ptr()),
             P(gate.data_ptr()), P(y.data_ptr()), None, P(st.cuda_stream)) for p in pools]
    for s in range(warmup):
        L.stepq_fp32_step(*args[s % layers])
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for s in range(steps):
        L.stepq_fp32_step(*args[s % layers])
    b.record(st)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    qkv = 3 * d * (2 if cfg.bf16_inputs else 4)
    gate_b = 4 * d if cfg.gate_kind == W.GATE_DIAG else 4
    bytes_step = R * H * (2 * d * d * 4 + qkv + 4 + gate_b + 4 * d)
    del pools
    return {"value": R * H / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
            "hbm_gbs": bytes_step / (ms * 1e-3) / 1e9, "bytes_per_step": bytes_step, "layers": layers}


# ---------------------------------------------------------------------------
# the CPU oracle (reference arm / cpu_baseline)
# ---------------------------------------------------------------------------
class OracleRunner:
    """The oracle as it stands: one (request, head) step per call, spread over host threads."""

    def __init__(self, cfg, mode):
        import oracle
        m, self.pin = mode_plan(cfg, mode)
        self.cfg = cfg
        self.plan = oracle.Plan(cfg.d, cfg.d, cfg.heads, cfg.gate_kind, cfg.unit_kind, m,
                                self.pin.bits, self.pin.w)
        self.threads = os.cpu_count() or 1
        self.R = min(cfg.requests, max(2, self.threads))
        X = W.initial_state(cfg, range(self.R))
        self.blobs = {}
        for r in range(self.R):
            for h in range(cfg.heads):
                blob, _ = self.plan.quantize_head(h, X[r, h])
                self.blobs[(r, h)] = blob
        self.si = W.step_inputs(cfg, 0, self.pin, range(self.R))
        self.keys = list(self.blobs)
        self.cursor = 0
        from concurrent.futures import ThreadPoolExecutor
        self.ex = ThreadPoolExecutor(self.threads)

    def _one(self, key):
        r, h = key
        si = self.si
        self.plan.step_head(h, self.blobs[key], si.q[r, h], si.k[r, h], si.v[r, h], si.beta[r, h],
                            si.gate[r, h])

    def run(self, count):
        keys = [self.keys[(self.cursor + i) % len(self.keys)] for i in range(count)]
        self.cursor += count
        # each key at most once per batch: distinct blobs per concurrent call
        for i in range(0, len(keys), len(self.keys)):
            list(self.ex.map(self._one, keys[i:i + len(self.keys)]))

    def rate_single(self, seconds):
        """One host thread, one (request, head) step after another."""
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < seconds:
            self._one(self.keys[self.cursor % len(self.keys)])
            self.cursor += 1
            n += 1
        return n / (time.perf_counter() - t0), n

    def rate(self, seconds):
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < seconds:
            self.run(self.threads)
            n += self.threads
        return n / (time.perf_counter() - t0), n


def run_drift(args, dist):
    """Quantised rollouts against the fp32 rollout of the same inputs.

    From one packed S0, the chosen quantiser variants (by default the
    workload's own plan with the STEPQuant fit, uniform INT8 and uniform
    INT6) step side by side with the unquantised fp32 state, with fresh
    seeded inputs every step.  At each
    checkpoint: the relative Frobenius error of every (request, head) state
    against the fp32 state, and the relative L2 error of y.  The pages report
    accuracy only on real models, so these numbers are reported, not checked."""
    import torch

    import quantized_delta_rule_decode_b200 as S
    cfg = W.CONFIGS[args.config]
    steps = args.drift_steps or cfg.steps
    d, H, R = cfg.d, cfg.heads, cfg.requests
    slots = torch.from_numpy(W.slot_indices(cfg)).cuda()
    pin = W.make_plan(cfg)
    X0 = torch.from_numpy(W.initial_state(cfg)).cuda()
    S32 = torch.zeros((cfg.pool_slots, H, d, d), dtype=torch.float32, device="cuda")
    S32[slots.long()] = X0
    arms = {}
    for name in args.drift_arms.split(","):
        mode, p = mode_plan(cfg, name)
        plan = S.stepq_plan_create(d, d, H, cfg.gate_kind, cfg.unit_kind, mode, p.bits, p.w)
        sb = S.stepq_plan_slot_bytes(plan)
        buf = torch.zeros(cfg.pool_slots * sb, dtype=torch.uint8, device="cuda")
        pool = S.stepq_pool_alloc(plan, cfg.pool_slots, buf)
        S.stepq_pack(plan, pool, slots, X0)
        arms[name] = {"plan": plan, "pool": pool, "slot_bytes": sb,
                      "ws": torch.empty(S.stepq_workspace_bytes(plan, R), dtype=torch.uint8, device="cuda"),
                      "y": torch.empty((R, H, d), dtype=torch.float32, device="cuda"), "points": []}
    del X0
    y32 = torch.empty((R, H, d), dtype=torch.float32, device="cuda")
    Sq = torch.empty((R, H, d, d), dtype=torch.float32, device="cuda")
    marks = sorted({m for m in (1, 16, 64, 256, 1024, 2048, 4096, steps) if m <= steps})
    dt = torch.bfloat16 if cfg.bf16_inputs else torch.float32
    t0 = time.perf_counter()
    for step in range(steps):
        si = W.step_inputs(cfg, step, pin)
        q, k, v = (torch.from_numpy(a).to(dt).cuda() for a in (si.q, si.k, si.v))
        beta, gate = torch.from_numpy(si.beta).cuda(), torch.from_numpy(si.gate).cuda()
        S.stepq_fp32_step(S32, slots, q, k, v, beta, gate, y32, cfg.gate_kind)
        for a in arms.values():
            S.stepq_decode_step(a["plan"], a["pool"], slots, q, k, v, beta, gate, a["y"], a["ws"])
        if step + 1 in marks:
            ref = S32[slots.long()]
            rn = ref.flatten(2).norm(dim=2)
            for name, a in arms.items():
                S.stepq_unpack(a["plan"], a["pool"], slots, Sq)
                e = (Sq - ref).flatten(2).norm(dim=2) / rn
                ey = float((a["y"] - y32).norm() / y32.norm())
                a["points"].append({"step": step + 1, "state_rel_fro_mean": float(e.mean()),
                                    "state_rel_fro_median": float(e.median()),
                                    "state_rel_fro_max": float(e.max()), "y_rel_l2": ey})
    torch.cuda.synchronize()
    status = {n: S.stepq_get_status(a["pool"]) for n, a in arms.items()}
    out = {"report": "rollout drift of quantised states vs the fp32 state", "config": args.config,
           "workload": workload_config(cfg, "stepquant", None)["workload"], "steps": steps,
           "data": "synthetic (seeded; workload.py)", "seconds": time.perf_counter() - t0,
           "arms": {n: {"slot_bytes": a["slot_bytes"],
                        "compression_vs_fp32": H * d * d * 4 / a["slot_bytes"],
                        "device_status": status[n], "points": a["points"]} for n, a in arms.items()}}
    if dist.rank == 0:
        print(json.dumps(out), flush=True)


def rank_average(x):
    """1-based ranks of x, tied values sharing the mean of their ranks."""
    x = np.asarray(x, np.float64)
    order = np.argsort(x, kind="mergesort")
    sx = x[order]
    ranks = np.empty(x.size, np.float64)
    i = 0
    while i < x.size:
        j = i
        while j + 1 < x.size and sx[j + 1] == sx[i]:
            j += 1
        ranks[order[i:j + 1]] = (i + j) / 2.0 + 1.0
        i = j + 1
    return ranks


def spearman_rho(a, b):
    """Spearman rank correlation: the Pearson correlation of the two rank
    vectors (average ranks for ties)."""
    ra, rb = rank_average(a), rank_average(b)
    ra -= ra.mean()
    rb -= rb.mean()
    den = math.sqrt(float(np.sum(ra * ra)) * float(np.sum(rb * rb)))
    return float(np.sum(ra * rb) / den) if den > 0 else float("nan")


LIFETIME_STUDIES = {
    # units = heads: scalar per-head gates, half-lives log-uniform in [1, 4096]
    "heads": dict(base="rollout", requests=8, heads=256),
    # units = key rows: per-row gates and half-lives (KDA)
    "rows": dict(base="kda", requests=16, heads=32),
}


def run_lifetime_study(args, dist):
    """How a unit's accumulated quantisation error relates to its memory lifetime.

    The pages find that a unit's gate half-life predicts how much INT6 error
    it accumulates (Spearman rho about 0.80 over a model's heads; rcap.io
    post, the "Temporal" paragraph; hyper.ai summary, Method, the lifetime
    paragraph).  This is the synthetic analogue: quantised rollouts beside the
    fp32 rollout of the same seeded inputs, for heads (scalar gates, one
    half-life per head) and for key rows (KDA: one half-life per row).  Per
    unit, the relative Frobenius error of its state against the fp32 state,
    averaged over requests, at checkpoints; the reported "accumulated" error
    is its mean over the checkpoints, and rho its Spearman rank correlation
    with the unit's half-life, for uniform INT6, the workload's STEPQuant plan
    (widths and pivots ranked by half-life) and the calibrated plan.
    Reported, not checked: the pages measure this on real models."""
    import dataclasses

    import torch

    import quantized_delta_rule_decode_b200 as S
    steps = args.drift_steps or 2048
    marks = [m for m in range(steps // 8, steps + 1, steps // 8)]
    out = {"report": "lifetime vs accumulated quantisation error (synthetic analogue)", "steps": steps,
           "checkpoints": marks, "data": "synthetic (seeded; workload.py)", "studies": {}}
    t0 = time.perf_counter()
    for study, spec in LIFETIME_STUDIES.items():
        base = W.CONFIGS[spec["base"]]
        cfg = dataclasses.replace(base, name=f"{base.name}-lifetime-{study}", requests=spec["requests"],
                                  heads=spec["heads"], pool_slots=spec["requests"], permute_slots=False,
                                  steps=steps)
        d, H, R = cfg.d, cfg.heads, cfg.requests
        slots = torch.arange(R, dtype=torch.int32, device="cuda")
        pin = W.make_plan(cfg)
        X0 = torch.from_numpy(W.initial_state(cfg)).cuda()
        S32 = X0.clone()
        arms = {}
        for name in ("uniform6", "stepquant", "calibrated"):
            mode, p = mode_plan(cfg, name)
            plan = S.stepq_plan_create(d, d, H, cfg.gate_kind, cfg.unit_kind, mode, p.bits, p.w)
            sb = S.stepq_plan_slot_bytes(plan)
            pool = S.stepq_pool_alloc(plan, R, torch.zeros(R * sb, dtype=torch.uint8, device="cuda"))
            S.stepq_pack(plan, pool, slots, X0)
            arms[name] = {"plan": plan, "pool": pool, "bits": p.bits,
                          "ws": torch.empty(S.stepq_workspace_bytes(plan, R), dtype=torch.uint8, device="cuda"),
                          "y": torch.empty((R, H, d), dtype=torch.float32, device="cuda"),
                          "err": []}
        del X0
        y32 = torch.empty((R, H, d), dtype=torch.float32, device="cuda")
        Sq = torch.empty((R, H, d, d), dtype=torch.float32, device="cuda")
        dt = torch.bfloat16 if cfg.bf16_inputs else torch.float32
        for step in range(steps):
            si = W.step_inputs(cfg, step, pin)
            q, k, v = (torch.from_numpy(a).to(dt).cuda() for a in (si.q, si.k, si.v))
            beta, gate = torch.from_numpy(si.beta).cuda(), torch.from_numpy(si.gate).cuda()
            S.stepq_fp32_step(S32, slots, q, k, v, beta, gate, y32, cfg.gate_kind)
            for a in arms.values():
                S.stepq_decode_step(a["plan"], a["pool"], slots, q, k, v, beta, gate, a["y"], a["ws"])
            if step + 1 in marks:
                for a in arms.values():
                    S.stepq_unpack(a["plan"], a["pool"], slots, Sq)
                    if cfg.unit_kind == W.UNIT_ROW:       # per key row: [R, H, d] -> [H * d]
                        e = (Sq - S32).norm(dim=3) / S32.norm(dim=3).clamp_min(1e-30)
                    else:                                  # per head: [R, H] -> [H]
                        e = (Sq - S32).flatten(2).norm(dim=2) / S32.flatten(2).norm(dim=2).clamp_min(1e-30)
                    a["err"].append(e.mean(dim=0).reshape(-1).double().cpu().numpy())
        torch.cuda.synchronize()
        half_life = np.asarray(pin.half_life, np.float64).reshape(-1)
        res = {"units": "key rows" if cfg.unit_kind == W.UNIT_ROW else "heads", "n_units": int(half_life.size),
               "workload": f"{R} requests x {H} heads, d_k=d_v={d}, "
                           f"{'per-key-row' if cfg.gate_kind else 'per-head'} gates, half-lives log-uniform "
                           f"in [1, {cfg.half_life_max:.0f}]", "arms": {}}
        for name, a in arms.items():
            errs = np.stack(a["err"])                       # [checkpoints, units]
            acc = errs.mean(axis=0)
            bits = np.asarray(a["bits"]).reshape(-1)
            res["arms"][name] = {
                "spearman_rho_accumulated": spearman_rho(half_life, acc),
                "spearman_rho_final": spearman_rho(half_life, errs[-1]),
                "mean_error_accumulated": float(acc.mean()),
                "mean_error_final": float(errs[-1].mean()),
                "units_by_bits": {int(b): int(np.sum(bits == b)) for b in (4, 6, 8, 16) if np.sum(bits == b)},
                "device_status": S.stepq_get_status(a["pool"])}
        out["studies"][study] = res
    out["seconds"] = time.perf_counter() - t0
    if dist.rank == 0:
        print(json.dumps(out), flush=True)


def run_timeline(args, dist):
    """Start and end of every kernel of a few overlapped decode steps, on one
    clock: CUDA events recorded on each kernel's own stream around the split
    calls (readout on the main stream, fit + pack on the side stream after an
    event), all read as offsets from one event at the start.  Shows where
    layer l's fit runs beside layer l + 1's readout (the schedule of the
    hyper.ai summary, Method, last paragraph)."""
    import torch
    cfg = W.CONFIGS[args.config]
    wl = DeviceWorkload(cfg, args.mode)
    steps = max(2 * wl.layers, 6)
    for s in range(args.warmup):
        wl.run_step(s)
    wl.join()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    t0.record(wl.main)
    for s in range(steps):
        wl.run_step_timed(args.warmup + s, evs[s])
    wl.join()
    torch.cuda.synchronize()
    rows = []
    for s, e in enumerate(evs):
        rows.append({"step": s, "layer": (args.warmup + s) % wl.layers,
                     "readout_us": [t0.elapsed_time(e[0]) * 1e3, t0.elapsed_time(e[1]) * 1e3],
                     "fit_us": [t0.elapsed_time(e[2]) * 1e3, t0.elapsed_time(e[3]) * 1e3]})
    overlap = 0.0
    for a, b in zip(rows, rows[1:]):
        lo = max(a["fit_us"][0], b["readout_us"][0])
        hi = min(a["fit_us"][1], b["readout_us"][1])
        overlap += max(0.0, hi - lo)
    out = {"report": "kernel timeline of overlapped decode steps (CUDA events on each kernel's stream)",
           "workload": workload_config(cfg, args.mode, wl)["workload"], "layers": wl.layers,
           "rows": rows, "readout_inside_previous_fit_us_total": overlap,
           "note": "a readout event pair brackets the call, which first waits for this layer's previous "
                   "fit; the readout kernel itself starts when SM resources free up"}
    if dist.rank == 0:
        print(json.dumps(out), flush=True)


PIPE_HIDDEN = 5120          # model width of the projection proxy (a 27B-class hybrid model)


def run_pipeline(args, dist):
    """Per-token critical path of a stack of layers (rcap.io post, the sentence
    after the pseudocode; hyper.ai summary, "Method", last paragraph: the fit
    and pack run on a separate stream, overlapped with later-layer compute).

    One token = L layers; each layer on the main stream: an input projection
    GEMM [R, hidden] x [hidden, 3 H d] (bf16, cuBLAS through torch), the
    readout kernel, an output projection GEMM [R, H d] x [H d, hidden]; the
    layer's fit + pack on the side stream after its readout.  The GEMMs stand
    in for the model's own compute (their outputs are not fed to the state
    step, which reads the seeded ring of inputs).  Variants: the two-stream
    design, the fit on the main stream, the GEMMs alone, and the fp32-state
    step in place of the quantised one.  Device time with CUDA events over K
    tokens after W warm-up tokens."""
    import torch
    cfg = W.CONFIGS[args.config]
    wl = DeviceWorkload(cfg, args.mode)
    L = wl.layers
    R, H, d = cfg.requests, cfg.heads, cfg.d
    hid = PIPE_HIDDEN
    g = torch.Generator(device="cuda").manual_seed(7)
    w_in = [torch.randn((hid, 3 * H * d), device="cuda", dtype=torch.bfloat16, generator=g) * 0.01
            for _ in range(L)]
    w_out = [torch.randn((H * d, hid), device="cuda", dtype=torch.bfloat16, generator=g) * 0.01
             for _ in range(L)]
    x = torch.randn((R, hid), device="cuda", dtype=torch.bfloat16, generator=g)
    y_in = torch.empty((R, 3 * H * d), device="cuda", dtype=torch.bfloat16)
    o_in = torch.randn((R, H * d), device="cuda", dtype=torch.bfloat16, generator=g)
    x_out = torch.empty((R, hid), device="cuda", dtype=torch.bfloat16)
    P = ctypes.c_void_p
    ms = P(wl.main.cuda_stream)
    # fp32 state per layer for the unquantised variant
    S32 = [torch.zeros((cfg.pool_slots, H, d, d), dtype=torch.float32, device="cuda") for _ in range(L)]
    t0 = wl.ring[0]
    y32 = torch.empty((R, H, d), dtype=torch.float32, device="cuda")

    def token(tok, variant):
        for l in range(L):
            torch.matmul(x, w_in[l], out=y_in)
            i = l * 16 + tok % 16
            if variant == "two_streams":
                if wl.L.stepq_decode_step(*wl.step_args[i]):
                    raise RuntimeError(wl.L.stepq_last_error().decode())
            elif variant == "one_stream":
                a = list(wl.step_args[i])
                a[-1] = ms
                if wl.L.stepq_decode_step(*a):
                    raise RuntimeError(wl.L.stepq_last_error().decode())
            elif variant == "fp32_state":
                wl.S.stepq_fp32_step(S32[l], wl.slots, t0["q"], t0["k"], t0["v"], t0["beta"], t0["gate"],
                                     y32, cfg.gate_kind)
            torch.matmul(o_in, w_out[l], out=x_out)

    torch.cuda.synchronize()   # the tensors above were made on the default stream
    out = {}
    for variant in ("two_streams", "one_stream", "gemm_only", "fp32_state"):
        # the GEMMs run on the readout's stream, so each readout follows its
        # layer's input projection as in a model
        with torch.cuda.stream(wl.main):
            for tok in range(args.warmup):
                token(tok, variant)
            wl.join()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(wl.main)
            for tok in range(args.steps):
                token(tok, variant)
            wl.join()
            b.record(wl.main)
            torch.cuda.synchronize()
        out[variant] = dist.max(a.elapsed_time(b) / args.steps)
    gemm = out["gemm_only"]
    line = {"report": "per-token critical path of a layer stack (GEMM proxy + state step)",
            "config": args.config, "mode": args.mode, "layers": L, "requests": R, "hidden": hid,
            "tokens": args.steps, "warmup": args.warmup, "data": "synthetic (seeded; workload.py)",
            "ms_per_token": out,
            "state_step_ms_per_layer": {k: (v - gemm) / L for k, v in out.items() if k != "gemm_only"},
            "overlap_saved_ms_per_token": out["one_stream"] - out["two_streams"]}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args):
    cfg = W.CONFIGS[args.config]
    orc = OracleRunner(cfg, args.mode)
    warm_rate, _ = orc.rate(2.0)
    budget = 150.0
    per_step = int(max(1, min(cfg.requests * cfg.heads,
                              budget * warm_rate / max(1, args.steps + args.warmup))))
    steps = args.steps
    if (args.steps + args.warmup) * per_step / warm_rate > budget * 1.5:
        steps = max(1, int(budget * warm_rate / per_step) - args.warmup)
    for _ in range(args.warmup):
        orc.run(per_step)
    t0 = time.perf_counter()
    for _ in range(steps):
        orc.run(per_step)
    dt = time.perf_counter() - t0
    value = steps * per_step / dt
    sample = (f"{per_step} (request, head) oracle steps per timed step ({args.config} workload, "
              f"{orc.R} requests x {cfg.heads} heads cycled), {steps} steps on {orc.threads} host threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup, "ms_per_step": dt / steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": workload_config(cfg, args.mode, None),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.threads, "kind": "oracle",
                             "sample": sample, "cpu": cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


SUB_CONFIGS = [("kda", "stepquant"), ("pool", "stepquant"), ("pool", "uniform8"), ("rollout", "stepquant")]


def measure_config(name, mode, steps, kernel_steps, warmup, hbm_peak, alu_peak, dist):
    """One more workload at full size on this GPU: plain decode steps between
    two events (as the headline), each kernel alone, the fp32-state step."""
    import torch
    cfg = W.CONFIGS[name]
    wl = DeviceWorkload(cfg, mode)

    for s in range(warmup):
        wl.run_step(s)
    wl.join()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(wl.main)
    for s in range(steps):
        wl.run_step(warmup + s)
    wl.join()
    b.record(wl.main)
    torch.cuda.synchronize()
    ms = dist.max(a.elapsed_time(b)) / steps
    rd_ms, fit_ms = time_isolated(wl, kernel_steps, warmup)
    alg = algorithmic_bytes(cfg, wl.pin, wl.head_bytes)
    rd_bytes = readout_bytes(cfg, wl.head_bytes)
    ops = fit_alu_ops(cfg, wl.pin, wl.mode)
    fp32 = time_fp32(cfg, wl.pin, kernel_steps, warmup)
    out = {"workload": workload_config(cfg, mode, wl)["workload"], "quantizer": mode,
           "value": dist.world * cfg.requests * cfg.heads / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
           "steps": steps, "hbm_gbs": dist.world * alg / (ms * 1e-3) / 1e9,
           "hbm_frac": alg / (ms * 1e-3) / 1e9 / hbm_peak, "bytes_per_step": alg,
           "slot_bytes": wl.slot_bytes, "compression_vs_fp32": W.fp32_state_bytes(cfg) / wl.slot_bytes,
           "readout": {"us_alone": rd_ms * 1e3, "gbs_alone": rd_bytes / (rd_ms * 1e-3) / 1e9,
                       "frac_hbm_alone": rd_bytes / (rd_ms * 1e-3) / 1e9 / hbm_peak},
           "fitpack": {"us_alone": fit_ms * 1e3, "fp32_ops": ops,
                       "frac_alu_alone": ops / (fit_ms * 1e-3) / 1e12 / alu_peak},
           "fp32_state_baseline": fp32}
    if fp32 is not None:
        fp32["frac_hbm"] = fp32["hbm_gbs"] / hbm_peak
    del wl
    torch.cuda.empty_cache()
    return out


def workload_config(cfg, mode, wl):
    pin = wl.pin if wl is not None else mode_plan(cfg, mode)[1]
    counts = {int(b): int(np.sum(pin.bits == b)) for b in (4, 6, 8, 16) if np.sum(pin.bits == b)}
    c = {"workload": f"{cfg.name}: {cfg.requests} requests x {cfg.heads} heads, d_k=d_v={cfg.d}, "
                     f"{'KDA per-key-row' if cfg.gate_kind else 'GDN scalar'} gates, "
                     f"{'bf16' if cfg.bf16_inputs else 'fp32'} q/k/v, 1 decode step per call",
         "requests": cfg.requests, "heads": cfg.heads, "d_k": cfg.d, "d_v": cfg.d,
         "quantizer": mode, "unit": "key row" if cfg.unit_kind else "head",
         "plan_units_by_bits": counts, "global_batch": cfg.requests, "seq_len": 1,
         "parallelism": "replicas (weak scaling)"}
    if wl is not None:
        c.update({"slot_bytes": wl.slot_bytes, "compression_vs_fp32": W.fp32_state_bytes(cfg) / wl.slot_bytes,
                  "layer_pools_cycled": wl.layers,
                  "l2": f"inputs larger than L2: {wl.layers} layer pools x "
                        f"{wl.nslots * wl.slot_bytes / 1e6:.1f} MB cycled, no flush",
                  "streams": (f"readout on a high-priority main stream, each layer's fit+pack on "
                              + ("its own side stream" if wl.fit_streams == wl.layers else
                                 f"one of {wl.fit_streams} side streams in turn")
                              + "; a layer's fit overlaps the next layer's readout and the tail of the "
                                "previous layer's fit")})
    return c


def src_sha():
    """Hash of the code (comments and spacing removed) that defines the device
    kernels, not the host API."""
    h = hashlib.sha256()
    for f in ("stepq_kernels.cu", "stepq_internal.cuh"):
        src = open(os.path.join(ROOT, "quantized_delta_rule_decode_b200", "csrc", f)).read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path)).get(kernel, {})
    except (OSError, ValueError):
        return None
    if rec.get("src_sha") != src_sha() or rec.get("workload") != workload:
        return None
    return rec.get("bytes_per_launch")


def main():
    global FIT_STREAMS, MAIN_PRIORITY
    args = parse()
    FIT_STREAMS, MAIN_PRIORITY = args.fit_streams, args.main_priority
    if args.impl == "reference":
        # the oracle on the host: rank 0 alone, no process group and no GPU
        if int(os.environ.get("RANK", "0")) == 0:
            run_reference(args)
        return
    dist = Dist(args.gpus)
    if args.drift or args.pipeline or args.lifetime_study or args.timeline:
        import torch
        torch.cuda.set_device(dist.local)
        (run_lifetime_study if args.lifetime_study else run_drift if args.drift else
         run_timeline if args.timeline else run_pipeline)(args, dist)
        dist.close()
        return
    import torch
    torch.cuda.set_device(dist.local)
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        pass
    hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    cfg = W.CONFIGS[args.config]
    if args.steps < 1 or args.warmup < 3:
        raise SystemExit("need --steps >= 1 and --warmup >= 3")

    wl = DeviceWorkload(cfg, args.mode)
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_index = cvd.split(",")[dist.local].strip() if cvd else str(dist.local)
    ms, clocks = time_device(wl, args.steps, args.warmup, dist, gpu_index)
    readout_ms, fit_ms = time_kernels_overlapped(wl, args.kernel_steps, args.warmup)
    # which kernel bounds the step: each kernel timed alone (the overlapped
    # durations above share the SMs with the other stream)
    iso_readout_ms, iso_fit_ms = time_isolated(wl, args.isolated_steps, args.warmup)
    ms_step = ms / args.steps
    hu = dist.world * cfg.requests * cfg.heads
    value = hu / (ms_step * 1e-3)
    alg_bytes = algorithmic_bytes(cfg, wl.pin, wl.head_bytes)
    hbm_gbs = dist.world * alg_bytes / (ms_step * 1e-3) / 1e9

    rd_bytes = readout_bytes(cfg, wl.head_bytes)
    rd_gbs = rd_bytes / (readout_ms * 1e-3) / 1e9
    ops = fit_alu_ops(cfg, wl.pin, wl.mode)
    clk_mhz = float(peaks.get("sm_max_mhz", 1965.0))
    alu_peak = SMS * FP32_LANES * clk_mhz * 1e6 / 1e12   # T fp32 lane-ops/s
    fit_tops = ops / (fit_ms * 1e-3) / 1e12
    iso_rd_gbs = rd_bytes / (iso_readout_ms * 1e-3) / 1e9
    iso_fit_tops = ops / (iso_fit_ms * 1e-3) / 1e12
    kern = {"readout": {"us": readout_ms * 1e3, "bytes": rd_bytes, "gbs": rd_gbs,
                        "frac_hbm": rd_gbs / hbm_peak, "us_alone": iso_readout_ms * 1e3,
                        "gbs_alone": iso_rd_gbs, "frac_hbm_alone": iso_rd_gbs / hbm_peak},
            "fitpack": {"us": fit_ms * 1e3, "fp32_ops": ops, "tops": fit_tops, "frac_alu": fit_tops / alu_peak,
                        "us_alone": iso_fit_ms * 1e3, "tops_alone": iso_fit_tops,
                        "frac_alu_alone": iso_fit_tops / alu_peak},
            "note": f"us: the kernel's busy time per launch (the union of its launches' event intervals / "
                    f"launches) in a separate pass of {args.kernel_steps} overlapped steps (the split calls with "
                    "events on each kernel's stream; the streams share the SMs, and consecutive layers' fits "
                    "on different side streams may overlap); "
                    f"us_alone: the kernel alone on one stream ({args.isolated_steps} steps); the headline "
                    "timed region runs plain stepq_decode_step calls only; the roofline kernel is the one "
                    "with the longer us_alone"}
    if iso_fit_ms >= iso_readout_ms:
        roof = {"kernel": "fitpack (k_quant, fit+pack)", "bound": "alu", "achieved": fit_tops,
                "peak": alu_peak, "unit": "T fp32 lane-ops/s", "frac": fit_tops / alu_peak,
                "traffic": ncu_traffic("fitpack", cfg.name),
                "peak_source": f"derived: {SMS} SMs x {FP32_LANES} FP32 lanes x {clk_mhz:.0f} MHz"}
    else:
        roof = {"kernel": "readout (k_readout)", "bound": "hbm", "achieved": rd_gbs, "peak": hbm_peak,
                "unit": "GB/s", "frac": rd_gbs / hbm_peak, "traffic": ncu_traffic("readout", cfg.name),
                "peak_source": peak_src}

    serial = None
    if args.serial and dist.world == 1:
        sm = time_serial(wl, min(args.steps, 5000), args.warmup)
        serial = {"ms_per_step": sm / min(args.steps, 5000)}
    if args.e2e_steps <= 0:
        args.e2e_steps = args.steps
    e2e_ms, h2d, d2h = time_e2e(wl, args.e2e_steps, args.warmup)
    e2e_ms = dist.max(e2e_ms)
    e2e_value = hu / (e2e_ms / args.e2e_steps * 1e-3)
    graph = time_graph(wl, args.steps) if args.graph else None
    graph_dev = dist.max(graph["ms_per_step"]) if graph else None
    if graph:
        graph["ms_per_step"] = graph_dev
        graph["value"] = dist.world * cfg.requests * cfg.heads / (graph_dev * 1e-3)
    fp32 = time_fp32(cfg, wl.pin, args.fp32_steps, 10)
    if fp32 is not None:
        fp32["frac_hbm"] = fp32["hbm_gbs"] / hbm_peak
        fp32["value"] *= dist.world

    config_obj = workload_config(cfg, args.mode, wl)
    configs = {}
    if args.config_steps > 0 and args.config == "gdn" and args.mode == "stepquant":
        del wl
        torch.cuda.empty_cache()
        for name, mode in SUB_CONFIGS:
            key = name if mode == "stepquant" else f"{name}_{mode}"
            configs[key] = measure_config(name, mode, args.config_steps, min(args.config_steps, 100),
                                          10, hbm_peak, alu_peak, dist)
        wl = None

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu:
        orc = OracleRunner(cfg, args.mode)
        rate, n = orc.rate(args.cpu_seconds)
        rate1, n1 = orc.rate_single(max(2.0, args.cpu_seconds / 4))
        cpu = {"value": rate, "unit": UNIT, "cores": orc.threads, "kind": "oracle",
               "value_1thread": rate1,
               "sample": f"{n} (request, head) oracle steps of the {cfg.name} workload "
                         f"({orc.R} requests x {cfg.heads} heads cycled) in {args.cpu_seconds:.0f} s",
               "cpu": cpu_model()}

    if dist.rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded; workload.py)",
                "config": config_obj,
                "hbm_gbs": hbm_gbs, "hbm_frac": hbm_gbs / hbm_peak, "hbm_peak_gbs": hbm_peak,
                "hbm_peak_source": peak_src, "bytes_per_step": alg_bytes,
                "roofline": roof, "kernels": kern,
                "fp32_state_baseline": fp32,
                "configs": configs or None,
                "serial_step": serial,
                "graph": graph,
                "cpu_baseline": cpu,
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.e2e_steps,
                        "steps": args.e2e_steps, "warmup": args.warmup,
                        "path": "stepq_decode_step_host (pinned host q,k,v,beta,gate in, y out)"},
                "gpu_launches": 2 * args.steps,
                "clocks": clocks}
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
