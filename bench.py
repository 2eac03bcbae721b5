#!/usr/bin/env python
"""Throughput of the SSD scan forward (tokens/s) and of the decode state update
(us/step) on B200, one JSON line on stdout (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one ssd_fwd call (chunk_cumsum -> chunk_state -> state_passing ->
chunk_scan) over one batch of the headline workload, bf16 in / fp32 accumulate,
batch 4 x seqlen 1024, 24 heads x headdim 64, dstate 64, 1 group, chunk 256.
Inputs are seeded synthetic data already resident in HBM; the working set
(26 MB) fits in L2, so a 256 MB buffer is written and then read back before
every timed step (outside the timed events) to flush it: the read makes the
written lines leave L2 before the timed region, so their write-back is not
charged to the step.  Each step is timed with CUDA events on
the launching stream; ms_per_step is the mean over the K timed steps, the max
over ranks.  Under torchrun every rank runs its own independent batch (weak
scaling, no collective on the data path).

Also reported: the same metric end to end through the public API from pinned
host buffers (`e2e`), the roofline position of the dominant kernel, the other
workloads (seqlen 4096 with an initial state, seqlen 65536 with 8 groups, and
1024 successive decode steps replayed from one CUDA graph), SM clocks sampled
through NVML during the timed region, and the fp64 CPU oracle timed on a
bounded sample of the same workload (`cpu_baseline`).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEADLINE = "fwd_bf16_b1_L65536_G8"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0, "source": "fallback"}
N_SM = 148
FFMA_LANES_PER_SM = 128


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--single-pass", action="store_true",
                    help="time the opt-in single-pass kernel (SSD_FLAG_SINGLE_PASS) instead of "
                         "the default three-kernel forward")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flush-mb", type=int, default=256)
    ap.add_argument("--e2e-steps", type=int, default=20,
                    help="steps of the end-to-end (pinned host buffers) measurement")
    ap.add_argument("--plumbing-only", action="store_true",
                    help="run only the rank plumbing (launcher, process group, max over "
                         "ranks) on CPU with gloo and print a JSON line without a metric")
    ap.add_argument("--conv-only", action="store_true",
                    help="time only the convolution workloads (one JSON line of them)")
    ap.add_argument("--bwd-only", action="store_true",
                    help="time only the backward-pass workloads (one JSON line of them)")
    ap.add_argument("--sel-only", action="store_true",
                    help="time only the diagonal-A selective-scan workloads (one JSON line)")
    ap.add_argument("--norm-only", action="store_true",
                    help="time only the gated RMSNorm workloads (one JSON line of them)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    return dict(FALLBACK_PEAKS)


# ---------------------------------------------------------------------------
class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons through NVML
    in a background thread while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.reason_bits = 0
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hi = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hi)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    h = hi
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nvml, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: the line says so
            self.err = repr(e)
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                self.reason_bits |= int(n.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        reasons = [k for k, bit in self.REASONS.items() if self.reason_bits & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
def algorithmic_cost(cfg, elt):
    """Bytes (inputs read once, outputs written once) and FLOP (causal half of
    the chunk-square terms) of each kernel of the forward, per launch."""
    b, L, H, P, N, G, Q = (cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim, cfg.dstate,
                           cfg.ngroups, cfg.chunk)
    nc = -(-L // Q)
    tok = b * L
    x = tok * H * P * elt
    bc = tok * G * N * elt
    dtr = tok * H * elt
    vec = b * H * nc * Q * 4
    # chunk states: fp32 local states (chunk_state out, state passing in), and
    # the entering states as a hi / lo bf16 pair (state passing out,
    # chunk_scan in): 4 bytes per element either way
    states = b * nc * H * P * N * 4
    init = b * H * P * N * 4 if cfg.init_state else 0
    fin = b * H * P * N * 4 if cfg.return_final else 0
    causal = Q * (Q + 1) / 2
    flops_state = 2.0 * tok * H * P * N
    flops_scan = (2.0 * b * nc * G * causal * N      # C.B^T per group
                  + 2.0 * b * nc * H * causal * P    # masked (C.B^T) x per head
                  + 2.0 * tok * H * P * N)           # C . H_in per head
    return {
        "chunk_cumsum": (dtr + 2 * vec, 0.0),
        "chunk_state": (x + bc + 2 * vec + states, flops_state),
        "state_passing": (2 * states + b * H * nc * 4 + init + fin, 2.0 * states / 4),
        "chunk_scan": (x + 2 * bc + 2 * vec + states + x, flops_scan),
        "path": (x + 2 * bc + dtr + x + init + fin, flops_state + flops_scan),
    }


# ---------------------------------------------------------------------------
# multi-rank plumbing (weak scaling: every rank runs its own independent batch)
def gpu_head_start(ms: float):
    """Queue a GPU spin of about `ms` milliseconds ahead of a timed loop, so the
    host enqueues the loop's launches while the GPU is busy and no host-side
    launch latency falls between a step's two events.  It runs before the
    first event and is not part of any timed step."""
    import torch
    torch.cuda._sleep(int(ms * 2.0e6))  # ~2 GHz SM clock: cycles per ms


def rank_env():
    """(rank, world size, local rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch (independent problems, no data-path
    collective)."""
    return base + 1000 * rank


def max_over_ranks(v: float, world: int, device) -> float:
    """The step time of the job: the slowest rank's."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's
    time."""
    return world * units_per_rank / (ms_max * 1e-3)


def main_ours(args):
    import torch
    import torch.distributed as dist

    import mamba_ssd_scan_b200 as ssd
    from mamba_ssd_scan_b200 import synthetic

    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def ranks_max(v: float) -> float:
        return max_over_ranks(v, world, dev)

    ssd.load_library()
    peaks = load_peaks()
    flush_buf = torch.empty(args.flush_mb << 20, dtype=torch.uint8, device=dev)

    flush_f = flush_buf.view(torch.float32)
    flush_acc = torch.empty((), dtype=torch.float32, device=dev)

    def flush():
        # write a buffer larger than L2, then read it back: the written lines
        # are evicted (written back) here, outside the timed region, and L2
        # holds none of the step's data
        flush_buf.fill_(1)
        torch.sum(flush_f, dim=0, out=flush_acc)

    if args.conv_only or args.bwd_only or args.sel_only or args.norm_only:
        if args.norm_only:
            res = norm_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max)
        elif args.conv_only:
            res = conv_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max)
        elif args.bwd_only:
            res = bwd_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max)
        else:
            res = sel_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max)
        if rank == 0:
            print(json.dumps({"workloads": res, "peaks_source": peaks["source"]}), flush=True)
        return

    cfg = synthetic.FWD_CONFIGS[args.workload]
    seed = rank_seed(1234 + synthetic.SEED_OFFSET[cfg.name], rank)
    inp = synthetic.make_config_inputs(cfg, seed)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    elt = d["x"].element_size()
    stream = torch.cuda.current_stream()

    y = torch.empty_like(d["x"])
    fin = (torch.empty((cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate), device=dev)
           if cfg.return_final else None)
    fwd_flags = ssd.SSD_FLAG_SINGLE_PASS if args.single_pass else 0
    ws = torch.empty(ssd.ssd_fwd_workspace_size(cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim,
                                                cfg.dstate, cfg.ngroups, cfg.chunk,
                                                cfg.dtype, flags=fwd_flags),
                     dtype=torch.uint8, device=dev)

    def step():
        ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"], cfg.chunk,
                    d["init_state"], y=y, final_state=fin, workspace=ws, flags=fwd_flags)

    # ---- headline: K timed steps ----------------------------------------
    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(local)
    with clocks:
        barrier()
        torch.cuda.synchronize()
        gpu_head_start(min(50.0, 0.15 * args.steps))
        for k in range(args.steps):
            flush()
            ev[k][0].record(stream)
            step()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    ms = ranks_max(ms)
    tokens = cfg.tokens
    value = job_throughput(tokens, world, ms)
    tc = ssd.tensor_core_steps(cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim, cfg.dstate,
                               cfg.ngroups, cfg.chunk, cfg.dtype, flags=fwd_flags)
    cost = algorithmic_cost(cfg, elt)
    if "fused" in tc:
        # one kernel does the whole path: its bytes are the path's (inputs
        # read once, y written once; no intermediate counted)
        launches_per_step = 1
        kms = {"fused_fwd": ms}
        roofline = roofline_entry("fused_fwd", cost["path"], ms, peaks, clocks.summary(), True,
                                  cfg.name)
        roofline["duration_note"] = ("CUDA events around each ssd_fwd call: the kernel plus "
                                     "the memset of its carry ring")
    else:
        # ssd_fwd folds step 1 into the tensor-core chunk_state
        launches_per_step = 3 if "chunk_state" in tc else 4
        kms = split_kernel_ms(ssd, cfg, d, y, fin, dev, flush, args.steps)
        top = max(kms, key=lambda n: kms[n])
        roofline = roofline_entry(top, cost[top], kms[top], peaks, clocks.summary(),
                                  top in tc, cfg.name)
    # the whole step against the path's algorithmic bytes, whatever the kernel split
    path_bytes = cost["path"][0]
    roofline["path_bytes"] = path_bytes
    roofline["path_frac"] = path_bytes / (ms * 1e-3) / (peaks["hbm_gbs"] * 1e9)

    # ---- e2e through the public API from pinned host buffers ------------
    # Every step moves its own inputs host -> device and its y device -> host
    # inside the timed region.  Consecutive steps are pipelined the way a
    # serving loop runs them: step k+1's inputs go over PCIe on one copy
    # stream while step k computes and its y comes back on another (the link
    # is full duplex); two device input / output sets alternate.
    e2e_steps = max(2, min(args.steps, args.e2e_steps))
    host = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
    y_host = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = y_host[0].numel() * y_host[0].element_size()
    dev_in = [d] + [{k: (torch.empty_like(v, device=dev) if v is not None else None)
                     for k, v in host.items()}]
    y_dev = [y, torch.empty_like(y)]
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(k):
        i = k % 2
        with torch.cuda.stream(s_h2d):
            if k >= 2:
                s_h2d.wait_event(ev_done[i])  # step k-2 has consumed input set i
            for key, v in host.items():
                if v is not None:
                    dev_in[i][key].copy_(v, non_blocking=True)
            ev_in[i].record(s_h2d)
        stream.wait_event(ev_in[i])
        if k >= 2:
            stream.wait_event(ev_out[i])  # step k-2's y has been read back
        dd = dev_in[i]
        ssd.ssd_fwd(dd["x"], dd["dt"], dd["A"], dd["B"], dd["C"], dd["D"], dd["dt_bias"],
                    cfg.chunk, dd["init_state"], y=y_dev[i], final_state=fin, workspace=ws,
                    flags=fwd_flags)
        ev_done[i].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(ev_done[i])
            y_host[i].copy_(y_dev[i], non_blocking=True)
            ev_out[i].record(s_d2h)

    for k in range(min(args.warmup, 3)):
        e2e_step(k)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_h2d.wait_event(e0)
    for k in range(e2e_steps):
        e2e_step(k)
    stream.wait_event(ev_out[(e2e_steps - 1) % 2])
    stream.wait_event(ev_out[(e2e_steps - 2) % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    ems = ranks_max(e0.elapsed_time(e1) / e2e_steps)
    e2e = {"value": job_throughput(tokens, world, ems), "unit": "tokens/s",
           "ms_per_step": ems, "steps": e2e_steps, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h,
           "pipelined": "2 streams: next step's inputs in while this step's y goes out"}
    del host, y_host, dev_in, y_dev
    d = y = None
    torch.cuda.empty_cache()

    # ---- other workloads (rank-local, reported for context) --------------
    extra = {}
    if not args.no_extra:
        extra = other_workloads(ssd, synthetic, dev, flush, peaks, rank, world,
                                barrier, ranks_max, skip=cfg.name)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, inp, budget_s=12.0)

    clk = clocks.summary()
    line = {
        "metric": "SSD fwd tokens/s",
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cfg.dtype.__repr__().endswith("bfloat16") else "f32",
        "data": "synthetic",
        "config": {"workload": cfg.name, "batch": cfg.batch, "seqlen": cfg.seqlen,
                   "nheads": cfg.nheads, "headdim": cfg.headdim, "dstate": cfg.dstate,
                   "ngroups": cfg.ngroups, "chunk": cfg.chunk,
                   "global_batch":
                   cfg.batch * world, "parallelism": f"dp{world}" if world > 1 else "single",
                   "l2": f"inputs {input_bytes(inp) / 1e6:.0f} MB; L2 flushed before every "
                         f"timed step ({args.flush_mb} MB write, then a read of it, so its "
                         "write-back ends before the timed region)"},
        "path": "single pass" if "fused" in tc else "three kernels",
        "roofline": roofline,
        "kernel_ms": kms,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": {k: clk[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "cpu_baseline": cpu,
        "workloads": extra,
        "peaks_source": peaks.get("source"),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def input_bytes(inp) -> int:
    return sum(v.numel() * v.element_size() for v in inp.values() if v is not None)


KERNEL_SOURCES = {
    "fused_fwd": ["fused_fwd.cu", "tcgen05.cuh", "tma.cuh", "internal.cuh"],
    "chunk_scan": ["chunk_scan_tc.cu", "tcgen05.cuh", "tma.cuh", "internal.cuh"],
    "chunk_state": ["chunk_state_tc.cu", "tcgen05.cuh", "tma.cuh", "internal.cuh"],
    "state_passing": ["state_passing.cu", "internal.cuh"],
    "chunk_cumsum": ["chunk_cumsum.cu", "internal.cuh"],
    "conv1d": ["conv1d.cu", "tcgen05.cuh", "tma.cuh", "internal.cuh"],
    "conv1d_update": ["conv1d.cu", "tcgen05.cuh", "tma.cuh", "internal.cuh"],
}


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from
    profiles/dram_traffic.md, or None when that pair was not measured or the
    kernel's source has changed since."""
    import hashlib
    srcs = KERNEL_SOURCES.get(kernel)
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    if not srcs or not os.path.exists(path):
        return None
    h = hashlib.sha256()
    for f in srcs:
        with open(os.path.join(ROOT, "mamba_ssd_scan_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    digest = h.hexdigest()[:16]
    with open(path) as fh:
        for line in fh:
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if (len(cells) >= 5 and cells[0] == workload and cells[1] == kernel
                    and cells[2] == digest):
                return int(cells[3]) + int(cells[4])
    return None


def roofline_entry(name, cost, ms, peaks, clk, on_tensor_cores, workload):
    """Roofline position of one kernel: the larger of its HBM time (algorithmic
    bytes / measured copy bandwidth) and its compute time (algorithmic FLOP /
    the peak of the unit that executes them) names the bound."""
    nbytes, flops = cost
    sec = ms * 1e-3
    hbm = peaks["hbm_gbs"]
    t_hbm = nbytes / (hbm * 1e9)
    if on_tensor_cores:
        # the kernel is timed inside short steps: the burst GEMM figure
        cpeak, cunit = peaks["bf16_tflops"], "bf16 tensor (cuBLAS burst)"
    else:
        # fp32 FFMA: 148 SMs x 128 FP32 lanes x 2 FLOP x SM clock
        mhz = clk.get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)
        cpeak = N_SM * FFMA_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
        cunit = f"FFMA 148 SM x 128 lanes x 2 x {mhz:.0f} MHz"
    t_cmp = flops / (cpeak * 1e12) if flops else 0.0
    src = peaks.get("source")
    if t_cmp > t_hbm:
        ach = flops / sec / 1e12
        return {"kernel": name, "bound": "tensor" if on_tensor_cores else "alu",
                "achieved": ach, "peak": cpeak, "unit": "TFLOP/s", "frac": ach / cpeak,
                "traffic": None, "peak_note": f"{cunit}, {src}",
                "algorithmic_bytes": nbytes, "algorithmic_flops": flops}
    ach = nbytes / sec / 1e9
    return {"kernel": name, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
            "frac": ach / hbm, "traffic": measured_traffic(name, workload), "peak_note": f"copy bandwidth, {src}",
            "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
            "compute_frac": (flops / sec / 1e12) / cpeak if flops else 0.0}


def launch_timing(ssd, synthetic, dev, flush, name, rank, steps=200):
    """Per-step device time of a small workload three ways: L2 flushed before
    each step, warm (back to back), and replayed from a CUDA graph holding one
    step (launch latency left out)."""
    import torch
    cfg = synthetic.FWD_CONFIGS[name]
    inp = synthetic.make_config_inputs(cfg, rank_seed(1234 + synthetic.SEED_OFFSET[name], rank))
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    y = torch.empty_like(d["x"])
    fin = (torch.empty((cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate), device=dev)
           if cfg.return_final else None)
    ws = torch.empty(ssd.ssd_fwd_workspace_size(cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim,
                                                cfg.dstate, cfg.ngroups, cfg.chunk, cfg.dtype),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"], cfg.chunk,
                    d["init_state"], y=y, final_state=fin, workspace=ws)

    def timed(with_flush):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        torch.cuda.synchronize()
        gpu_head_start(0.2 * steps)
        for a, b_ in evs:
            if with_flush:
                flush()
            a.record(stream)
            step()
            b_.record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b_) for a, b_ in evs) / steps * 1e3

    for _ in range(3):
        step()
    res = {"flushed_us": timed(True), "warm_us": timed(False)}
    try:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        g.replay()
        torch.cuda.synchronize()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            g.replay()
        b_.record(stream)
        torch.cuda.synchronize()
        res["graph_us"] = a.elapsed_time(b_) / steps * 1e3
        del g
    except Exception as e:  # reported, not fatal
        res["graph_error"] = repr(e)[:200]
    res["tokens_per_s_warm"] = cfg.tokens / (res["warm_us"] * 1e-6)
    return res


def other_workloads(ssd, synthetic, dev, flush, peaks, rank, world, barrier, ranks_max,
                    skip=None):
    import torch
    out = {}
    stream = torch.cuda.current_stream()
    # launch-latency view of the two small workloads
    for name in ("fwd_f32_small", "fwd_bf16_b4_L1024"):
        out[name + "_launch"] = launch_timing(ssd, synthetic, dev, flush, name, rank)
    for name, steps in (("fwd_bf16_b4_L1024", 50), ("fwd_bf16_b8_L4096_init", 20),
                        ("fwd_bf16_b1_L65536_G8", 5)):
        if name == skip:
            continue
        cfg = synthetic.FWD_CONFIGS[name]
        inp = synthetic.make_config_inputs(cfg, rank_seed(1234 + synthetic.SEED_OFFSET[name], rank))
        d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
        del inp
        y = torch.empty_like(d["x"])
        fin = torch.empty((cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate), device=dev) \
            if cfg.return_final else None
        nbytes = algorithmic_cost(cfg, 2)["path"][0]

        def timed_ms(flags):
            ws = torch.empty(ssd.ssd_fwd_workspace_size(cfg.batch, cfg.seqlen, cfg.nheads,
                                                        cfg.headdim, cfg.dstate, cfg.ngroups,
                                                        cfg.chunk, cfg.dtype, flags=flags),
                             dtype=torch.uint8, device=dev)

            def step():
                ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"],
                            cfg.chunk, d["init_state"], y=y, final_state=fin, workspace=ws,
                            flags=flags)

            for _ in range(3):
                step()
            torch.cuda.synchronize()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
            gpu_head_start(2.0)
            for a, b_ in evs:
                flush()
                a.record(stream)
                step()
                b_.record(stream)
            torch.cuda.synchronize()
            del ws
            return ranks_max(sum(a.elapsed_time(b_) for a, b_ in evs) / steps)

        ms = timed_ms(0)
        tc = ssd.tensor_core_steps(cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim, cfg.dstate,
                                   cfg.ngroups, cfg.chunk, cfg.dtype)
        ent = {"tokens_per_s": job_throughput(cfg.tokens, world, ms), "ms": ms,
               "path_bytes": nbytes,
               "hbm_frac_of_path_bytes": nbytes / (ms * 1e-3) / (peaks["hbm_gbs"] * 1e9),
               "kernels": "fused_fwd" if "fused" in tc else "three kernels"}
        if "fused" not in tc:
            ent["kernel_ms"] = split_kernel_ms(ssd, cfg, d, y, fin, dev, flush, steps)
        # the opt-in single-pass kernel on the same workload, for comparison
        ms1 = timed_ms(ssd.SSD_FLAG_SINGLE_PASS)
        ent["single_pass"] = {"ms": ms1, "tokens_per_s": job_throughput(cfg.tokens, world, ms1),
                              "hbm_frac_of_path_bytes":
                                  nbytes / (ms1 * 1e-3) / (peaks["hbm_gbs"] * 1e9)}
        out[name] = ent
        del d, y, fin
        torch.cuda.empty_cache()

    # decode: 1024 successive steps captured in one CUDA graph
    cfg = synthetic.DECODE_CONFIGS["decode_b256_H80"]
    seed = rank_seed(1234 + synthetic.SEED_OFFSET[cfg.name], rank)
    prm = synthetic.make_decode_params(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate, seed)
    state = prm["state"].to(dev)
    A, D, bias = prm["A"].to(dev), prm["D"].to(dev), prm["dt_bias"].to(dev)
    n_distinct = 16  # step inputs cycle through 16 distinct draws (3.7 MB each)
    steps_in = [synthetic.make_decode_step(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate,
                                           cfg.ngroups, cfg.dtype, seed, s)
                for s in range(n_distinct)]
    steps_in = [{k: v.to(dev) for k, v in s.items()} for s in steps_in]
    ys = torch.empty((cfg.batch, cfg.nheads, cfg.headdim), dtype=cfg.dtype, device=dev)

    def run(n):
        for s in range(n):
            si = steps_in[s % n_distinct]
            ssd.ssd_state_update(state, si["x"], si["dt"], A, si["B"], si["C"], D, bias, y=ys)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run(3)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(cfg.steps)
    g.replay()
    torch.cuda.synchronize()
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g.replay()
    b_.record(stream)
    torch.cuda.synchronize()
    us = ranks_max(a.elapsed_time(b_) * 1e3 / cfg.steps)
    sbytes = cfg.batch * cfg.nheads * cfg.headdim * cfg.dstate * 4
    step_bytes = 2 * sbytes + cfg.batch * (2 * cfg.nheads * cfg.headdim + cfg.nheads +
                                           2 * cfg.ngroups * cfg.dstate) * 2
    out[cfg.name] = {"us_per_step": us, "steps": cfg.steps, "graph": True,
                     "achieved_gbs": step_bytes / (us * 1e-6) / 1e9,
                     "hbm_frac": step_bytes / (us * 1e-6) / (peaks["hbm_gbs"] * 1e9),
                     "bytes_per_step": step_bytes}
    del g, state, steps_in
    torch.cuda.empty_cache()
    out.update(conv_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max))
    out.update(bwd_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max))
    out.update(sel_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max))
    out.update(norm_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max))
    return out


def norm_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max, steps=10):
    """The gated RMSNorm over the scan output of the two forward workloads
    (rows = batch * seqlen, channels = nheads * headdim, one group per row),
    L2 flushed before each launch."""
    import torch
    out = {}
    stream = torch.cuda.current_stream()
    for fname in ("fwd_bf16_b4_L1024", "fwd_bf16_b8_L4096_init"):
        f = synthetic.FWD_CONFIGS[fname]
        rows, ch = f.batch * f.seqlen, f.nheads * f.headdim
        name = f"gated_rmsnorm_bf16_b{f.batch}_L{f.seqlen}_C{ch}"
        inp = synthetic.make_norm_inputs(rows, ch, f.dtype, rank_seed(1234 + 9, rank))
        d = {k: v.to(dev) for k, v in inp.items()}
        o = torch.empty_like(d["y"])

        def step():
            ssd.ssd_gated_rmsnorm(d["y"], d["z"], d["weight"], eps=1e-5, out=o)

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        gpu_head_start(2.0)
        for a, b_ in evs:
            flush()
            a.record(stream)
            step()
            b_.record(stream)
        torch.cuda.synchronize()
        ms = ranks_max(sum(a.elapsed_time(b_) for a, b_ in evs) / steps)
        nbytes = 3 * rows * ch * d["y"].element_size() + ch * 4
        out[name] = {"tokens_per_s": job_throughput(rows, world, ms), "ms": ms,
                     "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
                     "hbm_frac": nbytes / (ms * 1e-3) / (peaks["hbm_gbs"] * 1e9),
                     "bytes": nbytes, "group": ch, "l2": "flushed"}
        del d, o
    torch.cuda.empty_cache()
    return out


# MUFU (special-function) throughput: 16 results per clock per SM, 148 SMs, 1.965 GHz
MUFU_TOPS = 148 * 16 * 1.965e9 / 1e12


def sel_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max, steps=10):
    """The diagonal-A selective scan: the forward over a sequence (L2 flushed
    before each call; bound by the exponential of every (token, channel,
    state), reported against the MUFU rate) and the decode step (1024 steps in
    one CUDA graph over 8 layers' states, against HBM)."""
    import torch
    out = {}
    stream = torch.cuda.current_stream()
    cfg = synthetic.SEL_CONFIGS["sel_bf16_b4_L1024_D1536_N16"]
    seed = rank_seed(1234 + synthetic.SEED_OFFSET[cfg.name], rank)
    inp = synthetic.make_selective_inputs(cfg.batch, cfg.seqlen, cfg.channels, cfg.dstate,
                                          cfg.dtype, seed, init_state=True)
    d = {k: v.to(dev) for k, v in inp.items()}
    y = torch.empty_like(d["x"])
    fin = torch.empty_like(d["init_state"])
    ws = torch.empty(ssd.ssd_selective_scan_workspace_size(cfg.batch, cfg.seqlen, cfg.channels,
                                                           cfg.dstate, cfg.chunk, cfg.dtype),
                     dtype=torch.uint8, device=dev)

    def step():
        ssd.ssd_selective_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["dt_bias"],
                               chunk=cfg.chunk, init_state=d["init_state"], y=y,
                               final_state=fin, workspace=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    gpu_head_start(2.0)
    for a, b_ in evs:
        flush()
        a.record(stream)
        step()
        b_.record(stream)
    torch.cuda.synchronize()
    ms = ranks_max(sum(a.elapsed_time(b_) for a, b_ in evs) / steps)
    exps = cfg.batch * cfg.seqlen * cfg.channels * cfg.dstate  # one exp per (t, d, n)
    nbytes = (3 * cfg.batch * cfg.seqlen * cfg.channels * 2 + 2 * cfg.batch * cfg.seqlen *
              cfg.dstate * 2 + 2 * cfg.batch * cfg.channels * cfg.dstate * 4)
    out[cfg.name] = {"tokens_per_s": job_throughput(cfg.batch * cfg.seqlen, world, ms), "ms": ms,
                     "bound": "alu", "exp_per_s": exps / (ms * 1e-3),
                     "mufu_frac": exps / (ms * 1e-3) / (MUFU_TOPS * 1e12),
                     "hbm_frac": nbytes / (ms * 1e-3) / (peaks["hbm_gbs"] * 1e9),
                     "l2": "flushed"}
    del d, y, fin, ws

    cfg = synthetic.SEL_CONFIGS["sel_update_b256_D1536_N16"]
    seed = rank_seed(1234 + synthetic.SEED_OFFSET[cfg.name], rank)
    per = [synthetic.make_selective_inputs(cfg.batch, 16, cfg.channels, cfg.dstate, cfg.dtype,
                                           seed + 97 * l, init_state=True)
           for l in range(cfg.layers)]
    states = [p_["init_state"].to(dev) for p_ in per]
    As = [p_["A"].to(dev) for p_ in per]
    Ds = [p_["D"].to(dev) for p_ in per]
    bs = [p_["dt_bias"].to(dev) for p_ in per]
    tok = [{k: per[0][k][:, t].contiguous().to(dev) for k in ("x", "dt", "B", "C")}
           for t in range(16)]
    yd = torch.empty((cfg.batch, cfg.channels), dtype=cfg.dtype, device=dev)
    del per

    def run(n):
        for s_ in range(n):
            l = s_ % cfg.layers
            tk = tok[s_ % len(tok)]
            ssd.ssd_selective_state_update(states[l], tk["x"], tk["dt"], As[l], tk["B"], tk["C"],
                                           Ds[l], bs[l], y=yd)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run(3)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(cfg.steps)
    g.replay()
    torch.cuda.synchronize()
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g.replay()
    b_.record(stream)
    torch.cuda.synchronize()
    us = ranks_max(a.elapsed_time(b_) * 1e3 / cfg.steps)
    step_bytes = (2 * cfg.batch * cfg.channels * cfg.dstate * 4 + 3 * cfg.batch * cfg.channels * 2
                  + 2 * cfg.batch * cfg.dstate * 2 + cfg.channels * (cfg.dstate + 2) * 4)
    out[cfg.name] = {"us_per_step": us, "steps": cfg.steps, "graph": True, "layers": cfg.layers,
                     "achieved_gbs": step_bytes / (us * 1e-6) / 1e9,
                     "hbm_frac": step_bytes / (us * 1e-6) / (peaks["hbm_gbs"] * 1e9),
                     "bytes_per_step": step_bytes}
    del g, states
    torch.cuda.empty_cache()
    return out


# fp32 FMA peak of the CUDA cores: 148 SMs x 128 FMA lanes x 2 FLOP x 1.965 GHz
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def bwd_flops(cfg):
    """Algorithmic FLOP of one ssd_bwd call: per chunk and head the two causal
    score matrices (C.B over N, dy.x over P), the three products with them
    (dxs over P, dB and dC over N) and the four state products (dS, and the
    dH / H_c terms of dxs, dB, dC), 2 FLOP per multiply-add."""
    nc = (cfg.seqlen + cfg.chunk - 1) // cfg.chunk
    Q, P, N = cfg.chunk, cfg.headdim, cfg.dstate
    tri = Q * (Q + 1) // 2
    per = tri * (N + P) + tri * (P + 2 * N) + 4 * Q * P * N
    return 2.0 * per * nc * cfg.nheads * cfg.batch


def bwd_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max, steps=5):
    """The backward pass (forward recompute included) on two forward
    workloads' shapes, with an initial state and d_final, L2 flushed before
    each call."""
    import torch
    out = {}
    stream = torch.cuda.current_stream()
    for name in ("fwd_bf16_b4_L1024", "fwd_bf16_b8_L4096_init"):
        cfg = synthetic.FWD_CONFIGS[name]
        seed = rank_seed(1234 + synthetic.SEED_OFFSET[name], rank)
        inp = synthetic.make_fwd_inputs(cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim,
                                        cfg.dstate, cfg.ngroups, cfg.dtype, seed, init_state=True)
        gr = synthetic.make_bwd_grads((cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim),
                                      (cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate),
                                      cfg.dtype, seed)
        d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
        dy, dfin = gr["dy"].to(dev), gr["d_final"].to(dev)
        ws = torch.empty(ssd.ssd_bwd_workspace_size(cfg.batch, cfg.seqlen, cfg.nheads,
                                                    cfg.headdim, cfg.dstate, cfg.ngroups,
                                                    cfg.chunk, cfg.dtype),
                         dtype=torch.uint8, device=dev)
        res = {}

        def step():
            ssd.ssd_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dy, D=d["D"],
                        dt_bias=d["dt_bias"], chunk=cfg.chunk, init_state=d["init_state"],
                        d_final=dfin, out=res, workspace=ws)

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        gpu_head_start(2.0)
        for a, b_ in evs:
            flush()
            a.record(stream)
            step()
            b_.record(stream)
        torch.cuda.synchronize()
        ms = ranks_max(sum(a.elapsed_time(b_) for a, b_ in evs) / steps)
        fl = bwd_flops(cfg)
        tf = fl / (ms * 1e-3) / 1e12
        # bf16 shapes in range run the per-chunk products on the tensor cores:
        # their roofline is the bf16 tensor peak; the CUDA-core path's is the
        # fp32 FMA peak
        on_tc = (cfg.dtype == torch.bfloat16 and cfg.headdim == 64 and cfg.dstate in (64, 128)
                 and cfg.chunk in (128, 256))
        line = {"tokens_per_s": job_throughput(cfg.tokens, world, ms), "ms": ms, "tflops": tf,
                "flop": fl, "l2": "flushed"}
        if on_tc:
            line.update(bound="tensor", peak_tflops=peaks["bf16_tflops"],
                        tensor_frac=tf / peaks["bf16_tflops"])
        else:
            line.update(bound="alu", peak_tflops=FP32_FMA_TFLOPS, fp32_fma_frac=tf / FP32_FMA_TFLOPS)
        out["bwd_" + name] = line
        del d, dy, dfin, ws, res
        torch.cuda.empty_cache()
    return out


def conv_workloads(ssd, synthetic, dev, flush, peaks, rank, world, ranks_max, steps=10):
    """The causal depthwise convolution in front of the scan: the forward over
    a sequence (L2 flushed before each launch) and the decode step (1024 steps
    in one CUDA graph, cycling through several layers' carried states)."""
    import torch
    out = {}
    stream = torch.cuda.current_stream()
    cfg = synthetic.CONV_CONFIGS["conv1d_bf16_b8_L4096_C2304"]
    inp = synthetic.make_conv_inputs(cfg.batch, cfg.seqlen, cfg.channels, cfg.width, cfg.dtype,
                                     rank_seed(1234 + synthetic.SEED_OFFSET[cfg.name], rank))
    d = {k: v.to(dev) for k, v in inp.items()}
    y = torch.empty_like(d["x"])
    fin = torch.empty_like(d["init_state"])

    def step():
        ssd.ssd_causal_conv1d(d["x"], d["weight"], d["bias"], d["init_state"], y=y,
                              final_state=fin)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    gpu_head_start(2.0)
    for a, b_ in evs:
        flush()
        a.record(stream)
        step()
        b_.record(stream)
    torch.cuda.synchronize()
    ms = ranks_max(sum(a.elapsed_time(b_) for a, b_ in evs) / steps)
    elt = 2 if cfg.dtype == torch.bfloat16 else 4
    nbytes = 2 * cfg.batch * cfg.seqlen * cfg.channels * elt + \
        2 * cfg.batch * cfg.channels * (cfg.width - 1) * 4 + cfg.channels * (cfg.width + 1) * 4
    out[cfg.name] = {"tokens_per_s": job_throughput(cfg.batch * cfg.seqlen, world, ms), "ms": ms,
                     "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
                     "hbm_frac": nbytes / (ms * 1e-3) / (peaks["hbm_gbs"] * 1e9),
                     "bytes": nbytes, "traffic": measured_traffic("conv1d", cfg.name),
                     "l2": "flushed"}
    del d, y, fin

    cfg = synthetic.CONV_CONFIGS["conv1d_update_b256_C7168"]
    seed = rank_seed(1234 + synthetic.SEED_OFFSET[cfg.name], rank)
    per = [synthetic.make_conv_inputs(cfg.batch, 16, cfg.channels, cfg.width, cfg.dtype,
                                      seed + 97 * l) for l in range(cfg.layers)]
    states = [p_["init_state"].to(dev) for p_ in per]
    ws = [p_["weight"].to(dev) for p_ in per]
    bs = [p_["bias"].to(dev) for p_ in per]
    xs = [p_["x"][:, t].contiguous().to(dev) for p_ in per[:1] for t in range(16)]
    yd = torch.empty((cfg.batch, cfg.channels), dtype=cfg.dtype, device=dev)
    del per

    def run(n):
        for s in range(n):
            l = s % cfg.layers
            ssd.ssd_conv1d_update(states[l], xs[s % len(xs)], ws[l], bs[l], y=yd)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run(3)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(cfg.steps)
    g.replay()
    torch.cuda.synchronize()
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g.replay()
    b_.record(stream)
    torch.cuda.synchronize()
    us = ranks_max(a.elapsed_time(b_) * 1e3 / cfg.steps)
    step_bytes = 2 * cfg.batch * cfg.channels * (cfg.width - 1) * 4 + \
        2 * cfg.batch * cfg.channels * elt + cfg.channels * (cfg.width + 1) * 4
    out[cfg.name] = {"us_per_step": us, "steps": cfg.steps, "graph": True, "layers": cfg.layers,
                     "achieved_gbs": step_bytes / (us * 1e-6) / 1e9,
                     "hbm_frac": step_bytes / (us * 1e-6) / (peaks["hbm_gbs"] * 1e9),
                     "bytes_per_step": step_bytes,
                     "traffic": measured_traffic("conv1d_update", cfg.name)}
    del g, states
    torch.cuda.empty_cache()
    return out


def split_kernel_ms(ssd, cfg, d, y, fin, dev, flush, steps):
    """Mean duration of each of the four steps (CUDA events between the step
    entry points, which launch the kernels ssd_fwd does: with bf16 on the
    tensor cores, state passing and chunk_scan in their hi / lo form; ssd_fwd
    also folds step 1 into chunk_state, which the entry points keep apart)."""
    import torch
    stream = torch.cuda.current_stream()
    nc = -(-cfg.seqlen // cfg.chunk)
    dt_sp = torch.empty((cfg.batch, cfg.nheads, nc, cfg.chunk), device=dev)
    cumA = torch.empty_like(dt_sp)
    # fp32 chunk states (the default precision)
    states = torch.empty((cfg.batch, nc, cfg.nheads, cfg.headdim, cfg.dstate), device=dev,
                         dtype=torch.float32)
    hilo = "chunk_scan" in ssd.tensor_core_steps(cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim,
                                                 cfg.dstate, cfg.ngroups, cfg.chunk, cfg.dtype)
    states_hl = (torch.empty((2,) + tuple(states.shape), device=dev, dtype=torch.bfloat16)
                 if hilo else None)
    names = ["chunk_cumsum", "chunk_state", "state_passing", "chunk_scan"]
    tot = dict.fromkeys(names, 0.0)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps + 2)]
    torch.cuda.synchronize()
    gpu_head_start(2.0)
    for it in range(steps + 2):
        flush()
        ev = evs[it]
        ev[0].record(stream)
        ssd.ssd_chunk_cumsum(d["x"], d["dt"], d["A"], d["B"], d["C"], d["dt_bias"], cfg.chunk,
                             dt_out=dt_sp, cumA_out=cumA)
        ev[1].record(stream)
        ssd.ssd_chunk_state(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_sp, cumA, cfg.chunk,
                            states=states)
        ev[2].record(stream)
        if hilo:
            ssd.ssd_state_passing_hilo(d["x"], d["dt"], d["A"], d["B"], d["C"], cumA, states,
                                       cfg.chunk, init_state=d["init_state"], final_state=fin,
                                       states_hl=states_hl)
        else:
            ssd.ssd_state_passing(d["x"], d["dt"], d["A"], d["B"], d["C"], cumA, states,
                                  cfg.chunk, init_state=d["init_state"], final_state=fin)
        ev[3].record(stream)
        if hilo:
            ssd.ssd_chunk_scan_hilo(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_sp, cumA,
                                    states_hl, d["D"], cfg.chunk, y=y)
        else:
            ssd.ssd_chunk_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_sp, cumA, states,
                               d["D"], cfg.chunk, y=y)
        ev[4].record(stream)
    torch.cuda.synchronize()
    for ev in evs[2:]:
        for i, n in enumerate(names):
            tot[n] += ev[i].elapsed_time(ev[i + 1])
    del dt_sp, cumA, states, states_hl
    return {n: tot[n] / steps for n in names}


def oracle_sample(cfg, inp, heads: int, tokens: int):
    """Batch row 0, its first `heads` heads and first `tokens` tokens: the
    bounded unit of oracle work the CPU timings use (the recurrence's work per
    token is the same all along the sequence).  Head h reads its own group's B
    and C, given to the oracle as one group column per head."""
    hpg = cfg.nheads // cfg.ngroups
    gsel = [h // hpg for h in range(heads)]
    return {"x": inp["x"][:1, :tokens, :heads], "dt": inp["dt"][:1, :tokens, :heads],
            "A": inp["A"][:heads], "B": inp["B"][:1, :tokens, gsel],
            "C": inp["C"][:1, :tokens, gsel], "D": inp["D"][:heads],
            "dt_bias": inp["dt_bias"][:heads],
            "init_state": None if inp["init_state"] is None else inp["init_state"][:1, :heads]}


def calibrated_sample(cfg, inp, orc, heads: int, seconds: float):
    """The oracle sample (heads x tokens) whose one run takes about `seconds`:
    a first run on up to 2048 tokens sets the rate; tokens are then scaled to
    the target and rounded to a multiple of the chunk (at least one chunk, at
    most the whole sequence)."""
    t0_tokens = min(cfg.seqlen, 2048)
    sub = oracle_sample(cfg, inp, heads, t0_tokens)
    t0 = time.perf_counter()
    orc.ssd_fwd(**sub)
    dt = max(time.perf_counter() - t0, 1e-6)
    tok = int(t0_tokens * seconds / dt) // cfg.chunk * cfg.chunk
    tok = max(cfg.chunk, min(cfg.seqlen, tok))
    return oracle_sample(cfg, inp, heads, tok), tok


def cpu_baseline(cfg, inp, budget_s=12.0):
    """The fp64 oracle, as it stands, on a bounded sample of the workload: batch
    row 0, as many heads as host threads, the first tokens of the sequence (a
    run of about 2 s), repeated until about budget_s seconds of work; then the
    same on one thread and one head for a quarter of that, and a few decode
    steps of the decode workload on all threads.  Throughput is in
    token-equivalents: tokens x heads / nheads per run."""
    import oracle
    from mamba_ssd_scan_b200 import synthetic
    orc = oracle.load()
    threads = orc.num_threads()
    heads = max(1, min(cfg.nheads, threads))
    sub, tok = calibrated_sample(cfg, inp, orc, heads, 2.0)
    tok_equiv = tok * heads / cfg.nheads

    def fwd_rate(sample, budget):
        t0 = time.perf_counter()
        runs = 0
        while time.perf_counter() - t0 < budget:
            orc.ssd_fwd(**sample)
            runs += 1
        return runs, time.perf_counter() - t0

    runs, dt = fwd_rate(sub, budget_s)
    out = {"value": runs * tok_equiv / dt, "unit": "tokens/s", "cores": threads,
           "kind": "oracle", "sample": f"{runs} x (batch row 0, heads 0-{heads - 1} of "
                                       f"{cfg.nheads}, tokens 0-{tok - 1} of {cfg.seqlen}) of "
                                       f"{cfg.name}, {dt:.1f} s; token-equivalents = "
                                       f"{tok} x {heads}/{cfg.nheads} per run"}
    orc.set_num_threads(1)
    sub1, tok1 = calibrated_sample(cfg, inp, orc, 1, 1.0)
    runs1, dt1 = fwd_rate(sub1, budget_s / 4)
    orc.set_num_threads(threads)
    out["one_core"] = {"value": runs1 * tok1 / cfg.nheads / dt1, "unit": "tokens/s",
                       "sample": f"{runs1} x (batch row 0, head 0, tokens 0-{tok1 - 1}), "
                                 f"{dt1:.1f} s"}
    # decode: a few steps on 8 of the 256 batch rows (the rows are independent),
    # scaled to the whole batch
    dcfg = synthetic.DECODE_CONFIGS["decode_b256_H80"]
    rows_d = 8
    prm = synthetic.make_decode_params(dcfg.batch, dcfg.nheads, dcfg.headdim, dcfg.dstate, 1)
    st = prm["state"][:rows_d].double().numpy().copy()
    steps_in = [synthetic.make_decode_step(dcfg.batch, dcfg.nheads, dcfg.headdim, dcfg.dstate,
                                           dcfg.ngroups, dcfg.dtype, 1, s_) for s_ in range(4)]
    t0 = time.perf_counter()
    for si in steps_in:
        st, _ = orc.state_update(st, si["x"][:rows_d], si["dt"][:rows_d], prm["A"],
                                 si["B"][:rows_d], si["C"][:rows_d], prm["D"], prm["dt_bias"])
    per_step = (time.perf_counter() - t0) / len(steps_in) * dcfg.batch / rows_d
    out["decode"] = {"us_per_step": per_step * 1e6, "workload": dcfg.name, "cores": threads,
                     "sample": f"{len(steps_in)} steps on {rows_d} of {dcfg.batch} batch rows, "
                               f"scaled to the whole batch"}
    return out


# ---------------------------------------------------------------------------
def main_reference(args):
    """The reference arm: the fp64 CPU oracle on this arm's workload, each step a
    bounded sample (batch row 0, as many heads as host threads, the first tokens
    of the sequence) sized so that warm-up and timed steps together take about
    two minutes.  Under torchrun only rank 0 runs it; the others exit at once."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    from mamba_ssd_scan_b200 import synthetic
    cfg = synthetic.FWD_CONFIGS[args.workload]
    inp = synthetic.make_config_inputs(cfg)
    orc = oracle.load()
    heads = max(1, min(cfg.nheads, orc.num_threads()))
    per_step = min(2.0, 120.0 / max(1, args.steps + args.warmup))
    sub, tok = calibrated_sample(cfg, inp, orc, heads, per_step)
    for _ in range(args.warmup):
        orc.ssd_fwd(**sub)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.ssd_fwd(**sub)
    sec = (time.perf_counter() - t0) / args.steps
    # one step covers tokens x heads / nheads of one batch row
    tok_equiv = tok * heads / cfg.nheads
    value = tok_equiv / sec
    line = {"impl": "reference", "metric": "SSD fwd tokens/s", "value": value,
            "unit": "tokens/s", "n_gpus": 0, "ranks": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "batch": cfg.batch, "seqlen": cfg.seqlen,
                       "nheads": cfg.nheads, "headdim": cfg.headdim, "dstate": cfg.dstate,
                       "ngroups": cfg.ngroups, "chunk": cfg.chunk},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": orc.num_threads(),
                             "kind": "oracle",
                             "sample": f"per step: batch row 0, heads 0-{heads - 1} of "
                                       f"{cfg.nheads}, tokens 0-{tok - 1} of {cfg.seqlen} "
                                       f"(token-equivalents = {tok} x {heads}/{cfg.nheads}); "
                                       "runs on the host cores of rank 0 only, no GPU"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main_plumbing(args):
    """The rank plumbing alone (no GPU, no metric): process group over gloo,
    every rank's id gathered and a max over ranks of a per-rank number, so a
    CPU test can check what `--gpus N` launches."""
    import torch
    import torch.distributed as dist
    rank, world, local = rank_env()
    if world > 1:
        import datetime
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    seen = [rank]
    if world > 1:
        t = torch.tensor([rank], dtype=torch.int64)
        out = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(out, t)
        seen = [int(v.item()) for v in out]
    ms = max_over_ranks(1.0 + rank, world, torch.device("cpu"))
    if rank == 0:
        print(json.dumps({"plumbing": True, "n_gpus": world, "ranks_seen": seen,
                          "local_ranks_ok": local == rank, "ms_max_over_ranks": ms}),
              flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def launch_ranks(args) -> int:
    """`--gpus N` (N > 1) started without a rank environment: start N ranks of
    this same command on this node (torch.distributed.run, rendezvous on
    127.0.0.1) and return their exit status."""
    import socket
    import subprocess
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
           f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


if __name__ == "__main__":
    a = parse_args()
    if a.gpus < 1:
        sys.exit("--gpus must be at least 1")
    if "WORLD_SIZE" not in os.environ and a.gpus > 1:
        sys.exit(launch_ranks(a))
    if int(os.environ.get("WORLD_SIZE", "1")) != a.gpus:
        sys.exit(f"--gpus {a.gpus} but WORLD_SIZE={os.environ.get('WORLD_SIZE')}: "
                 "launch one rank per GPU")
    if a.plumbing_only:
        main_plumbing(a)
    elif a.impl == "reference":
        main_reference(a)
    else:
        main_ours(a)
