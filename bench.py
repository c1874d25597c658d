#!/usr/bin/env python
"""Benchmark of the fused selective-scan forward pass on B200.

One step = one call of ssm_scan_fwd over the whole workload (every step of the
scan: softplus step size, retention exp, write, recurrence, readout, D skip,
SiLU gate, y and h_last stores). Default workload: the Mamba-2.8B-shaped layer
(b=4, L=8192, E=5120, N=16, bfloat16 activations, float32 state), synthetic
seeded inputs (selective_state_space_51_b200.workloads, shape 3).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--shape I]
                    [--impl reference] [--op scan|conv|step|bwd|train]

Prints ONE JSON line (rank 0). Multi-GPU runs are launched by torchrun with
one process per GPU; each rank scans its own batch of sequences (weak
scaling, no collective on the data path); the time is the max over ranks.

The metric: scan elements (b*L*E*N) per second, with the achieved GB/s of
algorithmic traffic and the fraction of the min(HBM, SFU-exp) roofline:
T_roof = max(bytes / HBM peak, exps / SFU peak), fraction = T_roof / T.
`--impl reference` times the float64 CPU oracle instead (rank 0 only).

`--op bwd` times the backward pass (ssm_scan_bwd: a forward that writes a
state checkpoint every 8 steps, then the reverse sweep) on the same
workload, and `--op train` a training step (ssm_scan_fwd with
SSM_SAVE_CHECKPOINTS, whose forward keeps those checkpoints, then
ssm_scan_bwd with SSM_REUSE_CHECKPOINTS, the reverse sweep alone). Two more
operations print a line of the same form: `--op conv` times the scan
with the causal depthwise convolution (width 4) + SiLU fused in front
(ssm_scan_fwd_conv, same workload and roofline), and `--op step` times one
batched decode step (ssm_scan_step: conv buffer shift, conv + SiLU, state
update, readout) over a [1024 x 5120 x 16] float32 state with bfloat16
activations, against the HBM roofline (it moves the state twice and does
little arithmetic).
"""
from __future__ import annotations

import argparse
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

METRIC = ("selective-scan fwd GB/s and (b·L·E·N)/s; "
          "% of min(HBM, SFU-exp) roofline")
UNIT = "scan elements/s"
SFU_EX2_PER_CLK_PER_SM = 16      # MUFU.EX2 lanes per clock per SM
HBM_NOMINAL_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}


# ----------------------------------------------------------------- sharding
def shard_for_rank(rank: int, world: int, shape: int = 3):
    """Weak scaling: rank r scans its own batch of sequences, drawn with its
    own seed (the r-th slice of a global batch of world * b sequences)."""
    if not 0 <= rank < world:
        raise ValueError("rank %d outside world %d" % (rank, world))
    return {"shape": shape, "seed": 51000 + shape + 1000 * rank,
            "global_batch_offset": rank}


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a group)."""
    if dist is None or not dist.is_initialized():
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- workload
CONV_WIDTH = 4

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the timed kernel, from one ncu capture, keyed by (op, workload shape), with
# the hash of the kernel sources that capture was taken from. A figure whose
# sources have changed since is stale: the line then reports null.
NCU_TRAFFIC = {
    ("scan", 3): (1.012991232e9 + 0.337603072e9, "643d90762c9b8bb1"),
    ("conv", 3): (1.012476416e9 + 0.338547456e9, "643d90762c9b8bb1"),
    ("step", 3): (0.409533184e9 + 0.330125056e9, "5ea473594a5cc7eb"),
    # the reverse sweep, the dominant kernel of both (mean of 2 launches of
    # the training step's capture)
    ("bwd", 3): (2.744350464e9 + 1.043970944e9, "50a3de46dc861e30"),
    ("train", 3): (2.744350464e9 + 1.043970944e9, "50a3de46dc861e30"),
}



KERNEL_SOURCES = {
    "scan": ("kernel_chunked.cuh", "device_math.cuh", "scan_params.cuh",
             "ssm_scan_abi.cu"),
    "conv": ("kernel_chunked.cuh", "device_math.cuh", "scan_params.cuh",
             "ssm_scan_abi.cu"),
    "step": ("kernel_step.cuh", "device_math.cuh", "ssm_scan_abi.cu"),
    "bwd": ("kernel_bwd.cuh", "kernel_chunked.cuh", "device_math.cuh",
            "scan_params.cuh", "ssm_scan_abi.cu"),
    "train": ("kernel_bwd.cuh", "kernel_chunked.cuh", "device_math.cuh",
              "scan_params.cuh", "ssm_scan_abi.cu"),
}
DECODE_BATCH = 1024


def kernel_source_hash(op: str = "scan") -> str:
    """sha256 (first 16 hex digits) of the sources of an op's kernel."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[op]:
        with open(os.path.join(ROOT, "selective_state_space_51_b200", "csrc",
                               name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(op: str, shape: int):
    """(traffic, source description) for the roofline record."""
    entry = NCU_TRAFFIC.get((op, shape))
    if entry is None:
        return None, "no ncu capture of this kernel on this workload"
    value, src_hash = entry
    now = kernel_source_hash(op)
    if now != src_hash:
        return None, ("ncu capture of kernel sources %s; the sources are now "
                      "%s, so the figure is stale" % (src_hash, now))
    return value, ("ncu dram__bytes_read.sum + dram__bytes_write.sum, one "
                   "launch, kernel sources %s" % src_hash)


def workload_config(wl, op: str, world: int, shape: int) -> dict:
    """The config record both arms print for the same workload."""
    from selective_state_space_51_b200 import workloads as W
    name = W.shape_description(shape)
    if op == "conv":
        name += "; causal depthwise conv width %d + SiLU fused in front" % (
            CONV_WIDTH)
    elif op == "bwd":
        name += "; backward"
    elif op == "train":
        name += ("; training step: forward keeping its checkpoints + "
                 "backward from them")
    elif op == "step":
        name = ("decode step, Mamba-2.8B layer shape: %d sequences x E=%d x "
                "N=%d float32 state, conv width %d, %s activations" % (
                    wl.batch, wl.dim, wl.dstate, CONV_WIDTH, wl.dtype))
    return {"workload": name, "op": op, "global_batch": world * wl.batch,
            "seq_len": wl.seqlen, "dim": wl.dim, "dstate": wl.dstate,
            "parallelism": "dp%d" % world}


def algorithmic_bytes(wl, op: str = "scan") -> int:
    """Each input read once, y written once, h0/h_last once; no [b,L,E,N]."""
    b, L, E, N = wl.batch, wl.seqlen, wl.dim, wl.dstate
    act = 4 if wl.dtype == "f32" else 2
    n = 2 * b * L * E * act            # x, delta
    if wl.dev["z"] is not None:
        n += b * L * E * act
    n += b * L * E * act               # y
    n += 2 * b * L * N * act           # B, C
    n += E * N * 4                     # A_log
    n += E * 4 if wl.dev["D"] is not None else 0
    n += E * 4 if wl.dev["delta_bias"] is not None else 0
    n += b * E * N * 4                 # h_last
    n += b * E * N * 4 if wl.dev["h0"] is not None else 0
    if op == "conv":
        n += E * CONV_WIDTH * 4 + E * 4    # filter taps and bias
    return n


def decode_bytes(wl) -> int:
    """One decode step: the float32 state and the conv buffer are read and
    written once; x_new, raw step, z, y once per channel; B, C once per row;
    the parameters once."""
    b, E, N = wl.batch, wl.dim, wl.dstate
    act = 4 if wl.dtype == "f32" else 2
    n = 2 * b * E * N * 4                      # state in and out
    n += 2 * b * E * CONV_WIDTH * act          # conv buffer in and out
    n += 4 * b * E * act                       # x_new, delta, z, y
    n += 2 * b * N * act                       # B, C
    n += E * N * 4 + E * CONV_WIDTH * 4 + 3 * E * 4  # A_log, taps, biases, D
    return n


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]),
                "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples every 100 ms while running."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,"
             "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None
        self.span = None   # (first, last) sample index of the timed region

    def wait_first(self, timeout: float = 3.0):
        """Block until the sampler has produced a line (nvidia-smi takes a
        moment to start), at most `timeout` seconds."""
        t0 = time.time()
        while self.proc is not None and not self.lines and \
                time.time() - t0 < timeout:
            time.sleep(0.01)

    def mark(self, end: bool = False):
        """Note where the timed region starts (end=False) or ends in the
        sample stream; the summary then uses the samples taken inside it,
        plus the first one after it."""
        if not end:
            self.span = (len(self.lines), None)
        elif self.span is not None:
            t0 = time.time()
            # the sample that covers the region's last moments
            while self.proc is not None and len(self.lines) <= self.span[0] \
                    and time.time() - t0 < 0.5:
                time.sleep(0.01)
            self.span = (self.span[0], len(self.lines))

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" +
                 self.QUERY, "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        lines = self.lines
        if self.span is not None and self.span[1] is not None:
            lines = self.lines[self.span[0]:self.span[1]] or self.lines
        for ln in lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- CPU leg
def oracle_inputs(wl):
    return dict(x=wl.values("x"), delta=wl.values("delta"),
                A_log=wl.dev["A_log"], B=wl.values("B"), C=wl.values("C"),
                D=wl.dev["D"], z=wl.values("z"),
                delta_bias=wl.dev["delta_bias"], h0=wl.dev["h0"])


def cpu_oracle_rate(wl, target_s: float = 10.0, inputs=None, k=None):
    """Time the float64 oracle on a bounded sample of the workload: the first
    k channels of every sequence, k sized for about target_s seconds (or
    given). Returns the cpu_baseline record; its "channels" is k."""
    import oracle
    inputs = oracle_inputs(wl) if inputs is None else inputs
    per_channel = wl.batch * wl.seqlen * wl.dstate
    if k is None:
        k0 = min(wl.dim, 4)
        t0 = time.perf_counter()
        oracle.scan_channels(np.arange(k0), **inputs, delta_softplus=True)
        dt = time.perf_counter() - t0
        rate = k0 * per_channel / max(dt, 1e-9)
        k = int(min(wl.dim, max(k0, target_s * rate / per_channel)))
    t0 = time.perf_counter()
    oracle.scan_channels(np.arange(k), **inputs, delta_softplus=True)
    dt = time.perf_counter() - t0
    return {"value": k * per_channel / dt, "unit": UNIT,
            "cores": oracle.max_threads(), "kind": "oracle", "channels": k,
            "sample": "%d of %d channels x all %d sequences x L=%d (%.2f s)"
                      % (k, wl.dim, wl.batch, wl.seqlen, dt)}


def run_reference(args):
    """--impl reference: the float64 CPU oracle on the same workload. One
    step is the oracle over a bounded sample of the workload (every sequence,
    the first k channels, all L steps), k sized so that the whole run takes
    about --reference-budget seconds; ms_per_step is that step's wall time
    and value the sample's scan elements per second."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if args.op != "scan":
        print(json.dumps({"impl": "reference", "unavailable":
                          "the oracle arm times the forward scan only"}))
        return 0
    from selective_state_space_51_b200 import workloads as W
    wl = W.make(args.shape)
    steps_ms, rates = [], []
    sample = None
    target = max(0.05, args.reference_budget / (args.warmup + args.steps))
    inputs = oracle_inputs(wl)
    k = None
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        r = cpu_oracle_rate(wl, target_s=target, inputs=inputs, k=k)
        dt = time.perf_counter() - t0
        k = r["channels"]
        if i >= args.warmup:
            steps_ms.append(1e3 * dt)
            rates.append(r["value"])
            sample = r
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.median(steps_ms),
        "ms_per_step_full_workload_extrapolated": 1e3 * wl.elements / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, "scan", args.gpus, args.shape),
        "cpu_baseline": dict(sample, value=value),
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU leg
def _to_device(arrays, dev):
    import torch
    out = {}
    for k, v in arrays.items():
        if v is None:
            out[k] = None
        elif v.dtype == np.uint16:
            out[k] = torch.from_numpy(v.view(np.int16)).to(dev).view(
                torch.bfloat16)
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(dev)
    return out


class ScanOp:
    """One forward scan (optionally with the fused convolution) per step."""

    def __init__(self, args, plan, dev, scan):
        import torch
        from selective_state_space_51_b200 import workloads as W
        self.name = args.op
        self.launches_per_step = 1
        extra = {"dim": args.dim} if getattr(args, "dim", None) else {}
        self.wl = wl = W.make(plan["shape"], seed=plan["seed"], **extra)
        self.t = _to_device(wl.dev, dev)
        self.conv = None
        if args.op == "conv":
            w, cb = W.conv_params(wl.dim, CONV_WIDTH)
            self.conv = (torch.from_numpy(w).to(dev),
                         torch.from_numpy(cb).to(dev))
        self.scan = scan
        self.y = torch.empty_like(self.t["x"])
        self.h_last = torch.empty((wl.batch, wl.dim, wl.dstate),
                                  dtype=torch.float32, device=dev)
        self.per_step_in = ("x", "delta", "z", "B", "C", "h0")
        self.units = wl.elements             # b*L*E*N per step
        self.nbytes = algorithmic_bytes(wl, args.op)
        self.workload = W.shape_description(args.shape) + (
            "; causal depthwise conv width %d + SiLU fused in front"
            % CONV_WIDTH if self.conv else "")

    def run(self, t, stream):
        kw = {}
        if self.conv:
            kw = dict(conv_weight=self.conv[0], conv_bias=self.conv[1])
        self.scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                  z=t["z"], delta_bias=t["delta_bias"], h0=t["h0"], y=self.y,
                  h_last=self.h_last, stream=stream, **kw)

    def outputs(self):
        return (self.y, self.h_last)


class StepOp:
    """One batched decode step per step (state updated in place)."""

    def __init__(self, args, plan, dev, scan):
        import torch
        from selective_state_space_51_b200 import workloads as W
        self.name = "step"
        self.launches_per_step = 1
        wl = W.make(plan["shape"], seed=plan["seed"], batch=DECODE_BATCH,
                    seqlen=1, with_h0=True)
        self.wl = wl
        w, cb = W.conv_params(wl.dim, CONV_WIDTH)
        d = {k: (v if v is None or k in ("A_log", "D", "delta_bias", "h0")
                 else v.reshape(v.shape[0], v.shape[2]))
             for k, v in wl.dev.items()}
        self.t = _to_device(d, dev)
        self.state = self.t.pop("h0")
        act = self.t["x"].dtype
        self.conv_state = torch.zeros((wl.batch, wl.dim, CONV_WIDTH),
                                      dtype=act, device=dev)
        self.conv = (torch.from_numpy(w).to(dev), torch.from_numpy(cb).to(dev))
        self.scan = scan
        self.y = torch.empty_like(self.t["x"])
        self.per_step_in = ("x", "delta", "z", "B", "C")
        self.units = wl.batch * wl.dim * wl.dstate
        self.nbytes = decode_bytes(wl)
        self.workload = (
            "decode step, Mamba-2.8B layer shape: %d sequences x E=%d x N=%d "
            "float32 state, conv width %d, %s activations" % (
                wl.batch, wl.dim, wl.dstate, CONV_WIDTH, wl.dtype))

    def run(self, t, stream):
        self.scan.step(t["x"], t["delta"], t["A_log"], t["B"], t["C"],
                       self.state, conv_state=self.conv_state,
                       conv_weight=self.conv[0], conv_bias=self.conv[1],
                       D=t["D"], z=t["z"], delta_bias=t["delta_bias"],
                       y=self.y, stream=stream)

    def outputs(self):
        return (self.y,)


class BwdOp:
    """One backward pass (training forward with checkpoints + reverse
    sweep) per step, for seeded incoming gradients."""

    def __init__(self, args, plan, dev, scan):
        import torch
        from selective_state_space_51_b200 import workloads as W
        self.name = "bwd"
        self.launches_per_step = 2   # checkpointing forward, reverse sweep
        self.wl = wl = W.make(plan["shape"], seed=plan["seed"])
        d = dict(wl.dev)
        rng = np.random.Generator(np.random.PCG64(plan["seed"] + 7))
        dy = rng.standard_normal((wl.batch, wl.seqlen, wl.dim),
                                 dtype=np.float32)
        d["dy"] = W.round_to_bf16_bits(dy) if wl.dtype == W.BF16 else dy
        self.t = _to_device(d, dev)
        self.scan = scan
        self.per_step_in = ("x", "delta", "z", "B", "C", "h0", "dy")
        self.units = wl.elements
        act = 4 if wl.dtype == "f32" else 2
        b, L, E, N = wl.batch, wl.seqlen, wl.dim, wl.dstate
        gated = wl.dev["z"] is not None
        # inputs once (x, raw step, z, dy, B, C), gradients once (dx, d raw,
        # dz in the activation type; dB, dC float32), parameters
        self.nbytes = ((3 + gated) * b * L * E * act + 2 * b * L * N * act
                       + (2 + gated) * b * L * E * act + 2 * b * L * N * 4
                       + 2 * E * N * 4 + 4 * E * 4)
        self.grads = None
        self.det = bool(getattr(args, "deterministic", False))
        self.workload = W.shape_description(args.shape) + "; backward"

    def run(self, t, stream):
        self.grads = self.scan.backward(
            t["x"], t["delta"], t["A_log"], t["B"], t["C"], t["dy"],
            D=t["D"], z=t["z"], delta_bias=t["delta_bias"], h0=t["h0"],
            stream=stream, deterministic=self.det)

    def outputs(self):
        return tuple(v for v in self.grads.values() if v is not None)


class TrainOp(BwdOp):
    """One training step per step: the forward that keeps the backward's
    state checkpoints (y and h_last out), then the backward that starts from
    them (its reverse sweep alone)."""

    def __init__(self, args, plan, dev, scan):
        import torch
        from selective_state_space_51_b200 import workloads as W
        super().__init__(args, plan, dev, scan)
        self.name = "train"
        self.launches_per_step = 2   # forward with checkpoints, reverse sweep
        wl = self.wl
        self.y = torch.empty_like(self.t["x"])
        self.h_last = torch.empty((wl.batch, wl.dim, wl.dstate),
                                  dtype=torch.float32, device=dev)
        self.nbytes += algorithmic_bytes(wl, "scan")
        self.workload = W.shape_description(args.shape) + (
            "; training step: forward keeping its checkpoints + backward "
            "from them")

    def run(self, t, stream):
        self.scan(t["x"], t["delta"], t["A_log"], t["B"], t["C"], D=t["D"],
                  z=t["z"], delta_bias=t["delta_bias"], h0=t["h0"], y=self.y,
                  h_last=self.h_last, stream=stream, save_checkpoints=True)
        self.grads = self.scan.backward(
            t["x"], t["delta"], t["A_log"], t["B"], t["C"], t["dy"],
            D=t["D"], z=t["z"], delta_bias=t["delta_bias"], h0=t["h0"],
            stream=stream, reuse_checkpoints=True, deterministic=self.det)

    def outputs(self):
        return (self.y, self.h_last) + super().outputs()


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import selective_state_space_51_b200 as S

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE %d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    plan = shard_for_rank(rank, world, args.shape)
    scan = S.SelectiveScan(local)
    op = {"step": StepOp, "bwd": BwdOp, "train": TrainOp}.get(
        args.op, ScanOp)(args, plan, dev,
                                                              scan)
    t = op.t
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(args.warmup):
        op.run(t, stream)
    torch.cuda.synchronize(dev)
    if scan.sync_status(stream) != S.SSM_OK:
        raise SystemExit("device status error during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        clocks.wait_first()
        barrier()
        torch.cuda.synchronize(dev)
        clocks.mark()
        t_begin = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_begin.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            op.run(t, stream)
            ends[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        clocks.mark(end=True)
        barrier()
    status = scan.sync_status(stream)
    if status != S.SSM_OK:
        raise SystemExit("device status %d in the timed region" % status)
    local_ms = t_begin.elapsed_time(t_end)
    kernel_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms = max_over_ranks(local_ms, dist if world > 1 else None, dev)
    kernel_ms = max_over_ranks(kernel_ms, dist if world > 1 else None, dev)
    variant = scan.last_variant() if op.name in ("scan", "conv") else (0, 0)

    # ---- end to end through the public API with pinned host buffers
    if args.no_e2e:
        return _finish(args, op, world, rank, local, dev, dist, scan, clocks,
                       total_ms, kernel_ms, variant, None, 0, 0)
    # Each step copies its own inputs in from pinned host memory and its own
    # outputs back, all inside the timed region. Inputs are double-buffered:
    # step i+1's host-to-device copy (its own stream) overlaps step i's
    # kernel and device-to-host copy (a third stream); a buffer is refilled
    # only after the kernel that read it has finished, and a kernel starts
    # only after the previous step's outputs have been copied out.
    host = {k: (None if v is None else v.cpu().pin_memory())
            for k, v in t.items()}
    dev_in = [{k: (None if v is None else torch.empty_like(v))
               for k, v in t.items()} for _ in range(2)]
    for buf in dev_in:
        for k, v in host.items():
            if v is not None:
                buf[k].copy_(v)
    h2d = sum(host[k].numel() * host[k].element_size()
              for k in op.per_step_in if host.get(k) is not None)
    op.run(dev_in[0], stream)
    out_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory()
                for o in op.outputs()]
    d2h = sum(o.numel() * o.element_size() for o in out_host)
    s_h2d = torch.cuda.Stream(dev)
    s_d2h = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]
    ev_out = torch.cuda.Event()
    ev_d2h = torch.cuda.Event()
    torch.cuda.synchronize(dev)

    def e2e_step(i):
        j = i % 2
        s_h2d.wait_event(ev_free[j])
        with torch.cuda.stream(s_h2d):
            for k in op.per_step_in:
                if host.get(k) is not None:
                    dev_in[j][k].copy_(host[k], non_blocking=True)
        ev_in[j].record(s_h2d)
        stream.wait_event(ev_in[j])
        stream.wait_event(ev_d2h)
        op.run(dev_in[j], stream)
        ev_free[j].record(stream)
        outs = op.outputs()
        ev_out.record(stream)
        s_d2h.wait_event(ev_out)
        with torch.cuda.stream(s_d2h):
            for o, oh in zip(outs, out_host):
                o.record_stream(s_d2h)
                oh.copy_(o, non_blocking=True)
        ev_d2h.record(s_d2h)

    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_h2d)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(s_d2h)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps,
                            dist if world > 1 else None, dev)
    return _finish(args, op, world, rank, local, dev, dist, scan, clocks,
                   total_ms, kernel_ms, variant, e2e_ms, h2d, d2h)


def _finish(args, op, world, rank, local, dev, dist, scan, clocks, total_ms,
            kernel_ms, variant, e2e_ms, h2d, d2h):
    import torch
    peaks = load_peaks()
    clk = clocks.summary()
    wl = op.wl
    nbytes = op.nbytes
    units = op.units
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ms = total_ms / args.steps
    value = world * units / (ms * 1e-3)
    gbps = nbytes / (kernel_ms * 1e-3) / 1e9
    sfu_peak_max = sms * SFU_EX2_PER_CLK_PER_SM * peaks["sm_max_mhz"] * 1e6
    sfu_peak_run = (sms * SFU_EX2_PER_CLK_PER_SM * clk["sm_mhz"] * 1e6
                    if clk["sm_mhz"] else None)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_sfu = units / sfu_peak_max       # one retention exp per unit
    t_roof = max(t_hbm, t_sfu)
    achieved_exp = units / (kernel_ms * 1e-3)
    if op.name == "step":
        metric = ("decode step (b·E·N) state elements/s; GB/s; "
                  "% of HBM roofline")
        unit = "state elements/s"
        roof = {"bound": "hbm", "unit": "GB/s", "achieved": gbps,
                "peak": peaks["hbm_gbs"], "frac": gbps / peaks["hbm_gbs"],
                "peak_note": "%s HBM copy bandwidth" % peaks["source"],
                "traffic": None}
        l2 = ("state of %.0f MB, larger than L2, rewritten every step"
              % (wl.batch * wl.dim * wl.dstate * 4 / 1e6))
    else:
        metric, unit = METRIC, UNIT
        traffic, traffic_source = traffic_record(op.name, args.shape)
        roof = {"bound": "alu", "unit": "Gexp/s",
                "achieved": achieved_exp / 1e9,
                "peak": sfu_peak_max / 1e9,
                "frac": achieved_exp / sfu_peak_max,
                "peak_note": "SFU ex2: %d SMs x %d/clk x %.0f MHz (max SM "
                             "clock, %s)" % (sms, SFU_EX2_PER_CLK_PER_SM,
                                             peaks["sm_max_mhz"],
                                             peaks["source"]),
                "frac_at_sampled_clock": (achieved_exp / sfu_peak_run
                                          if sfu_peak_run else None),
                "traffic": traffic, "traffic_source": traffic_source,
                "algorithmic_bytes": nbytes}
        l2 = "inputs larger than L2 (%.0f MB read per step)" % (nbytes / 1e6)
    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "io_dtype": wl.dtype, "data": "synthetic",
        "config": dict(workload_config(wl, op.name, world, args.shape),
                       **({"deterministic_sums": True}
                          if getattr(op, "det", False) else {}),
                       **({"grid_study_dim": args.dim}
                          if getattr(args, "dim", None) else {})),
        "l2": l2,
        "gb_per_s": gbps,
        "roofline": roof,
        "e2e": (None if e2e_ms is None else
                {"value": world * units / (e2e_ms * 1e-3), "unit": unit,
                 "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                 "ms_per_step": e2e_ms}),
        "gpu_launches": args.steps * op.launches_per_step,
        "clocks": clk,
    }
    if op.name != "step":
        # the exp2 rate measured on this GPU right after the timed region
        try:
            import selective_state_space_51_b200 as S
            rate = S.ssm_measure_ex2_rate(local)
            line["roofline"]["ex2_measured_gexp_s"] = rate / 1e9
            line["roofline"]["frac_of_measured_ex2"] = achieved_exp / rate
        except Exception as exc:  # reported, never fatal to the bench line
            line["roofline"]["ex2_measured_error"] = str(exc)[:200]
    if op.name in ("bwd", "train"):
        line["roofline"]["peak_note"] += (
            "; one retention exp per element counted (the %s evaluates "
            "about 3.3: one each in the %sforward, the recompute and the "
            "reverse sweep, plus the softplus and gate per (t, e))" % (
                ("pass", "checkpointing ") if op.name == "bwd"
                else ("step", "")))
    if op.name != "step":
        line["roofline_min_hbm_sfu"] = {
            "t_hbm_us": t_hbm * 1e6, "t_sfu_us_at_max_clock": t_sfu * 1e6,
            "t_kernel_us": kernel_ms * 1e3,
            "frac": t_roof / (kernel_ms * 1e-3),
            "hbm_peak_gbs": peaks["hbm_gbs"], "hbm_source": peaks["source"],
            "frac_at_8tbs_hbm": max(nbytes / (HBM_NOMINAL_GBS * 1e9), t_sfu)
            / (kernel_ms * 1e-3)}
        if op.name not in ("bwd", "train"):
            line["kernel"] = {"variant": variant[0], "segments": variant[1]}
    if (rank == 0 and world == 1 and not args.no_cpu_baseline
            and op.name == "scan"):
        line["cpu_baseline"] = cpu_oracle_rate(wl, args.reference_seconds)
    scan.close()
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--shape", type=int, default=3,
                    help="workload shape index (default 3: Mamba-2.8B layer)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--op", choices=["scan", "conv", "step", "bwd", "train"],
                    default="scan",
                    help="scan (default), the scan with the fused "
                         "convolution, the batched decode step, the "
                         "backward pass, or a training step (forward "
                         "keeping checkpoints + backward from them)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--dim", type=int, default=None,
                    help="--op scan / conv: another channel count E for the "
                         "shape (for studies of the grid; not a bench line "
                         "of the stated workloads)")
    ap.add_argument("--deterministic", action="store_true",
                    help="--op bwd / train: bitwise reproducible summed "
                         "gradients (SSM_DETERMINISTIC)")
    ap.add_argument("--reference-seconds", type=float, default=10.0,
                    help="CPU seconds of the oracle sample in cpu_baseline")
    ap.add_argument("--reference-budget", type=float, default=120.0,
                    help="total CPU seconds of an --impl reference run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (host buffer) measurement")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
