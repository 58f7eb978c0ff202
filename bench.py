"""Benchmark of the batched Muon step + batched EMA on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 6]

One step = muon_step_batched over the 66 matrices of the 11L x 512d GPT
(K = 5 fixed-quintic Newton-Schulz steps, momentum 0.99, lr 0.022, wd 0.105,
MuonEq-R) followed by ema_update_batched over every parameter of the same
model (38,071,388 fp32, decay 0.9965): every row of the hot path.  Inputs are
synthetic (seeded), resident in HBM and larger than L2 (about 0.67 GB for the 11L set).

For N > 1 it runs under torch.distributed.run, one rank per GPU; each rank
steps its own replica (weak scaling, no collective on the data path); the
time is the max over ranks.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0
only) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from muon_optimizer_step_02_b200 import workloads as wl  # noqa: E402

METRIC = ("Muon steps/s (66-matrix 11L×512d set); NS TFLOP/s & EMA "
          "GB/s as % of B200 peak")
UNIT = "steps/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}


# CUDA sources each recorded kernel is built from (its own code, the shared
# PTX wrappers and tables, and the host-built schedule that orders its work)
KERNEL_SOURCES = {
    "ns_mega_pair_kernel": ("k_ns_mega.cuh", "k_ns_common.cuh", "sm100_ptx.cuh",
                            "muon_types.cuh", "schedule.h", "muon_api.cu"),
}


def kernel_source_hash(kernel: str = "ns_mega_pair_kernel") -> str:
    """sha256 over the CUDA sources of `kernel`, to tell whether a recorded
    ncu traffic figure still belongs to the kernel being timed."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        path = os.path.join(ROOT, "muon_optimizer_step_02_b200", "csrc", name)
        h.update(name.encode())
        with open(path, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: int):
    """DRAM bytes per launch of `kernel` from the committed ncu summary
    (profiles/roofline_traffic.json), or None if it was taken on other
    kernel sources or another workload."""
    path = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    try:
        with open(path) as f:
            doc = json.load(f)
    except (OSError, ValueError):
        return None
    rec = doc.get(kernel)
    if not rec or rec.get("workload") != workload:
        return None
    if kernel not in KERNEL_SOURCES or rec.get("source_sha256") != kernel_source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


def load_workload(idx: int) -> wl.Workload:
    """Workload idx; the K=4 workload takes the committed 4-step minimax table
    (tests/golden/polar_express_k4.json, written by an oracle/ script) as its
    Newton-Schulz input."""
    if idx != 3:
        return wl.workload(idx)
    with open(os.path.join(ROOT, "tests", "golden", "polar_express_k4.json")) as f:
        return wl.workload(3, json.load(f)["coeffs"])


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------
# clocks
# --------------------------------------------------------------------------
class ClockSampler:
    """Samples SM clock and clock-event reasons of this process's GPU every
    few milliseconds (NVML, read-only) while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
               "sw_power_cap": 0x4}

    def __init__(self, cuda_index: int, period_s: float = 0.005):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = None
        self._thread = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            return pynvml.nvmlDeviceGetHandleByUUID(uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def start(self):
        import threading
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(
                h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(
                        h, pynvml.NVML_CLOCK_SM))
                    self.reasons |= int(
                        pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))
                except Exception:
                    pass
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=2)
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples),
                "sm_max_mhz": self.max_mhz,
                "reasons": sorted(k for k, bit in self.REASONS.items()
                                  if self.reasons & bit),
                "samples": len(self.samples), "source": "nvml"}


# --------------------------------------------------------------------------
# our implementation
# --------------------------------------------------------------------------
class Workload:
    """Device state of one replica of the benchmark workload."""

    def __init__(self, w: wl.Workload, seed: int):
        import torch
        from muon_optimizer_step_02_b200 import binding as B
        self.B = B
        self.w = w
        self.plan = B.MuonPlan(w.shapes, max_ns_steps=len(w.coeffs))
        self.ws = self.plan.alloc_workspace()
        self.W = [torch.from_numpy(wl.weight(w, i, seed)).cuda()
                  for i in range(w.n_mats)]
        self.M = [torch.zeros_like(x) for x in self.W]
        self.G_host = [torch.from_numpy(wl.grad_bits(w, i, 0, seed)
                                        .view(np.int16)).view(torch.bfloat16)
                       for i in range(w.n_mats)]
        self.G = [g.cuda() for g in self.G_host]
        self.scales = wl.update_scales(w)
        # EMA over every parameter: the matrices (their current W) plus the
        # non-matrix tensors.
        self.extra = []
        for j, n in enumerate(w.ema_extra_numels):
            _, p = wl.ema_pair(w, w.n_mats + j, seed)
            self.extra.append(torch.from_numpy(p).cuda())
        self.E = [x.clone() for x in self.W] + [x.clone() for x in self.extra]
        self.P = [x.view(-1) for x in self.W] + self.extra
        self.E = [e.view(-1) for e in self.E]

        # Arguments are marshalled once; a step only enqueues the launches.
        self._muon = self.plan.bind(self.W, self.M, self.G, self.w.hyper,
                                    self.w.coeffs, self.ws,
                                    update_scales=self.scales)
        self._ema = (B.ema_bind(self.E, self.P, self.w.ema_decay)
                     if self.w.ema_decay is not None else None)

    def step(self):
        self._muon()
        if self._ema is not None:
            self._ema()

    def launches_per_step(self) -> int:
        n = self.plan.step_launches(len(self.w.coeffs))
        if self.w.ema_decay is not None:
            n += self.B.ema_launches(len(self.E))
        return n

    def ns_flops_by_kind(self):
        """Dense FLOPs per launch of each Newton-Schulz launch kind."""
        gram = sum(2 * min(r, c) ** 2 * max(r, c) for r, c in self.w.shapes)
        poly = sum(2 * min(r, c) ** 3 for r, c in self.w.shapes)
        k = len(self.w.coeffs)
        return {"gram": gram, "poly": poly, "apply": gram,
                "ns": k * (2 * gram + poly)}

    def resident_bytes(self) -> int:
        """Device bytes the step reads or writes: W, M, G, the plan's
        workspace, the averages and the non-matrix parameters."""
        ts = self.W + self.M + self.G + self.E + self.extra + [self.ws]
        return sum(t.numel() * t.element_size() for t in ts)

    def state_bytes(self):
        elems = self.w.numel()
        return {"prologue": 12 * elems,  # G 2 + M 4+4 + X~ 2
                "ema": 12 * sum(self.w.ema_numels())}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    w = load_workload(args.workload)
    rep = Workload(w, seed=1337 + rank)
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()

    for _ in range(args.warmup):
        rep.step()
    torch.cuda.synchronize()
    assert rep.plan.last_error() == 0

    # One CUDA graph holds a whole step (the Muon step's launches and the
    # EMA), captured after the warm-up so that the plan's tables are on the
    # device; the headline replays it (eager launches with --eager).
    graph = None
    if not args.eager:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                rep.step()
        stream.wait_stream(side)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        assert rep.plan.last_error() == 0
    run_step = graph.replay if graph is not None else rep.step

    # ---- timed region: device time with CUDA events on the launching
    # stream.  The block of K steps is timed `repeats` times (each bracketed
    # by a barrier and synchronisations); the median block is reported, and
    # the clock sampler runs across all of them.
    clocks = ClockSampler(local_rank)
    blocks = []
    clocks.start()
    for _ in range(args.repeats):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            run_step()
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        blk = t0.elapsed_time(t1)
        if world > 1:
            t = torch.tensor([blk], device="cuda", dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            blk = float(t.item())
        blocks.append(blk)
    clk = clocks.stop()
    if rep.plan.last_error() != 0:
        raise RuntimeError("device-side error during the timed region")
    ms = statistics.median(blocks)
    ms_per_step = ms / args.steps
    value = world * args.steps / (ms / 1e3)

    # ---- per-launch times for the roofline: the same steps launched eagerly
    # with the plan's events between its launches (the events of a replayed
    # graph are not harvested)
    rep.plan.set_timing(True)
    rep.plan.timing_read()  # reset
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        rep.step()
    ev1.record(stream)
    torch.cuda.synchronize()
    eager_ms = ev0.elapsed_time(ev1)
    phase = rep.plan.timing_read()
    rep.plan.set_timing(False)
    if rep.plan.last_error() != 0:
        raise RuntimeError("device-side error during the eager timing loop")
    if world > 1:
        t = torch.tensor([eager_ms], device="cuda", dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        eager_ms = float(t.item())
    eager_value = world * args.steps / (eager_ms / 1e3)
    del graph

    # ---- EMA time (own events, the EMA kernel is launched on this stream)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    ema_ms = None
    if w.ema_decay is not None:
        reps = max(3, args.steps // 4)
        e0.record(stream)
        for _ in range(reps):
            rep._ema()
        e1.record(stream)
        torch.cuda.synchronize()
        ema_ms = e0.elapsed_time(e1) / reps

    # ---- the fused AdamW + EMA pass over the model's non-matrix parameters
    # (embeddings, vectors, scalars), each launch timed alone after an L2
    # flush by a 256 MB read (its 0.23 GB of traffic is about the size of L2;
    # a read flush also writes back the previous launch's dirty lines before
    # the timed one starts)
    adamw = adamw_ema_measure(w, stream, max(3, min(args.steps, 20)))

    # ---- end to end through the public API with host buffers: every step's
    # gradients are copied in from pinned host memory and every step's status
    # word is copied back to pinned host memory.  The gradients of all
    # matrices sit in one flat buffer (8-element aligned views), so an upload
    # is a single copy; two device buffers (one plan bound to each) let the
    # upload of step t + 1 run on a copy stream while step t computes; the
    # host reads a step's status one step later.
    from muon_optimizer_step_02_b200 import binding as B
    offs, tot = [], 0
    for r, c in w.shapes:
        offs.append(tot)
        tot += (r * c + 7) // 8 * 8
    host_flat = torch.zeros(tot, dtype=torch.bfloat16).pin_memory()
    for g, o in zip(rep.G_host, offs):
        host_flat[o:o + g.numel()].copy_(g.view(-1))
    h2d = tot * 2
    e2e_steps = max(3, min(args.steps, 50))
    dev_flat = [torch.empty(tot, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    bufs = []
    for k in range(2):
        dev_flat[k].copy_(host_flat)
        views = [dev_flat[k][o:o + r * c].view(r, c) for o, (r, c) in zip(offs, w.shapes)]
        plan_k = B.MuonPlan(w.shapes, max_ns_steps=len(w.coeffs))
        ws_k = plan_k.alloc_workspace()
        run_k = plan_k.bind(rep.W, rep.M, views, w.hyper, w.coeffs, ws_k,
                            update_scales=rep.scales)
        run_k()                              # uploads this plan's table
        bufs.append((run_k, dev_flat[k], plan_k, ws_k))
    copy_stream = torch.cuda.Stream()
    status = torch.zeros(2, dtype=torch.int32).pin_memory()
    ev_copied = [torch.cuda.Event() for _ in range(2)]
    ev_used = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    tt0 = torch.cuda.Event(enable_timing=True)
    tt1 = torch.cuda.Event(enable_timing=True)
    tt0.record(stream)
    for t in range(e2e_steps):
        k = t & 1
        run, Gk, plan_k, _ = bufs[k]
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(ev_used[k])     # step t - 2 has read Gk
            Gk.copy_(host_flat, non_blocking=True)
            ev_copied[k].record(copy_stream)
        stream.wait_event(ev_copied[k])
        run()
        if rep._ema is not None:
            rep._ema()
        ev_used[k].record(stream)
        plan_k.error_async(status[k:k + 1])      # 4 bytes back, no sync
        ev_done[k].record(stream)
        if t >= 1:
            ev_done[k ^ 1].synchronize()
            if int(status[k ^ 1]) != 0:
                raise RuntimeError("device-side error in the e2e loop")
    tt1.record(stream)
    torch.cuda.synchronize()
    if int(status[(e2e_steps - 1) & 1]) != 0:
        raise RuntimeError("device-side error in the e2e loop")
    e2e_ms = tt0.elapsed_time(tt1)
    if world > 1:
        t = torch.tensor([e2e_ms], device="cuda", dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    for _, _, plan_k, _ in bufs:
        plan_k.close()
    e2e_value = world * e2e_steps / (e2e_ms / 1e3)

    if rank != 0:
        return None

    # ---- the largest workload (24L x 2048d), one GPU only
    largest = None
    if world == 1 and not args.no_largest:
        largest = measure_largest(stream, local_rank, peaks, peak_src,
                                  args.largest_replays)

    # ---- yardstick: the same Newton-Schulz work as torch/cuBLAS GEMMs
    yard_ms = (torch_ns_yardstick(w, stream, max(3, min(args.steps, 20)))
               if not args.no_yardstick else None)

    # ---- roofline of the dominant kernel
    flops = rep.ns_flops_by_kind()
    ns_kinds = ("gram", "poly", "apply", "ns")
    dom = max(phase, key=lambda k: phase[k][1])
    launches_dom, ms_dom = phase[dom]
    # The Newton-Schulz launch is timed alone (about 0.4 ms per launch in a
    # loop of a few milliseconds), so its peak is the burst bf16 figure.
    burst = peaks["bf16_tflops"]
    if dom in ns_kinds:
        per_launch = flops[dom]
        dt = ms_dom / launches_dom / 1e3
        achieved = per_launch / dt / 1e12
        kname = "ns_mega_pair_kernel" if dom == "ns" else dom
        issued = ns_issued_flops(w) / dt / 1e12 if dom == "ns" else None
        roof = {"kernel": f"{kname} (all {len(w.coeffs)} Newton-Schulz steps)"
                if dom == "ns" else dom,
                "bound": "tensor",
                "achieved": round(achieved, 2), "peak": burst,
                "unit": "TFLOP/s", "frac": round(achieved / burst, 4),
                "issued_tflops": round(issued, 2) if issued else None,
                "issued_frac": round(issued / burst, 4) if issued else None,
                "traffic": recorded_traffic(kname, args.workload),
                "traffic_unit": "bytes per launch (ncu dram read + write)",
                "flops_per_launch": per_launch,
                "flops_count": "dense 4m^2n + 2m^3 per matrix and step; "
                               "issued = the pair k-blocks the kernel runs",
                "peak_source": f"{peak_src} burst bf16 (kernel timed per launch)"}
    else:
        per_launch = rep.state_bytes()["prologue"]
        achieved = per_launch / (ms_dom / launches_dom / 1e3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": None, "peak_source": f"{peak_src} HBM copy"}
    ns_ms = sum(phase[k][1] for k in ns_kinds if k in phase) / args.steps
    pro_ms = phase["prologue"][1] / max(phase["prologue"][0], 1)
    breakdown = {k: {"launches": v[0], "ms_per_step": round(v[1] / args.steps, 4)}
                 for k, v in phase.items() if v[0] > 0}
    ema_gbs = (rep.state_bytes()["ema"] / (ema_ms / 1e3) / 1e9) if ema_ms else None

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16+f32",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1e-3) bf16 grads)",
        "config": {"workload": w.name, "n_mats": w.n_mats,
                   "matrix_params": w.numel(),
                   "ema_params": sum(w.ema_numels()),
                   "ns_steps": len(w.coeffs), "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2 ({rep.resident_bytes() / 1e9:.2f} GB "
                         "resident, all of it read or written every step)",
                   "mode": "eager launches" if args.eager
                   else "CUDA graph replay (one graph per step)",
                   "timing": f"median of {args.repeats} timed blocks of "
                             f"{args.steps} steps each",
                   "eager_steps_per_s": round(eager_value, 3)},
        "clocks": clk,
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4,
                "how": "all gradients uploaded as one copy from pinned memory on a "
                       "copy stream, double-buffered; each step's status word copied "
                       "back and checked one step later.  Weights, momenta and "
                       "averages stay resident on the device (an optimizer's state "
                       "lives where the model does), so the only result read back "
                       "per step is the 4-byte status word"},
        "gpu_launches": rep.launches_per_step() * args.steps,
        "roofline": roof,
        "ns": ns_record(ns_ms, flops["ns"], ns_issued_flops(w), burst,
                        "burst (timed per launch)"),
        "prologue": prologue_record(pro_ms, w.numel(), peaks["hbm_gbs"]),
        "ema": {"gbs": round(ema_gbs, 1) if ema_gbs else None,
                "frac": round(ema_gbs / peaks["hbm_gbs"], 4) if ema_gbs else None,
                "ms": round(ema_ms, 4) if ema_ms else None},
        "breakdown": breakdown,
    }
    if yard_ms is not None:
        line["yardstick"] = {
            "impl": "torch.bmm + baddbmm (cuBLAS), bf16, dense products, "
                    "grouped by shape, one CUDA graph",
            "work": "the Newton-Schulz steps only (no prologue, scale or W update)",
            "ns_ms": round(yard_ms, 4),
            "tflops": round(flops["ns"] / (yard_ms / 1e3) / 1e12, 2),
            "fused_speedup": round(yard_ms / ns_ms, 3) if ns_ms > 0 else None}
    if largest is not None:
        line["largest"] = largest
    if adamw is not None:
        a_ms, a_params = adamw
        a_gbs = 36 * a_params / (a_ms / 1e3) / 1e9
        line["adamw_ema"] = {"params": a_params, "ms": round(a_ms, 4),
                             "gbs": round(a_gbs, 1),
                             "frac": round(a_gbs / peaks["hbm_gbs"], 4),
                             "bytes_per_param": 36}
    return line


def ns_record(ns_ms, dense_flops, issued_flops, peak, peak_name):
    """Newton-Schulz time per step with its dense (4m^2n + 2m^3 per matrix
    and step) and issued (pair k-blocks run) rates against `peak`."""
    if not ns_ms or ns_ms <= 0:
        return None
    dense = dense_flops / (ns_ms / 1e3) / 1e12
    issued = issued_flops / (ns_ms / 1e3) / 1e12
    return {"ms_per_step": round(ns_ms, 4), "tflops": round(dense, 2),
            "issued_tflops": round(issued, 2), "peak": peak, "peak_kind": peak_name,
            "frac": round(dense / peak, 4), "issued_frac": round(issued / peak, 4),
            "dense_flops": dense_flops, "issued_flops": issued_flops}


def prologue_record(pro_ms, elems, hbm_gbs):
    """The prologue's rate counted two ways: the algorithmic 10 B per matrix
    element of the momentum step (G read 2, M read 4 and written 4), and the
    12 B it moves (plus the bf16 working copy written)."""
    if not pro_ms or pro_ms <= 0:
        return None
    alg = 10 * elems / (pro_ms / 1e3) / 1e9
    moved = 12 * elems / (pro_ms / 1e3) / 1e9
    return {"ms": round(pro_ms, 4), "gbs": round(alg, 1), "frac": round(alg / hbm_gbs, 4),
            "bytes_per_elem": 10, "moved_gbs": round(moved, 1),
            "moved_frac": round(moved / hbm_gbs, 4), "moved_bytes_per_elem": 12}


def measure_largest(stream, local_rank, peaks, peak_src, replays):
    """The 24L x 2048d set (144 matrices, K=5 fixed quintic) plus the EMA over
    its 1.14 G parameters, one CUDA graph per step replayed `replays` times
    (about a second of dense tensor work, so the sustained bf16 peak
    applies), with its own clock record; then a few eager steps for the
    per-kernel split.  Inputs are drawn on the device from a seeded generator
    (same distributions as the 11L set's host-drawn inputs)."""
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    w = wl.workload(5)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1337)
    plan = B.MuonPlan(w.shapes, max_ns_steps=len(w.coeffs))
    ws = plan.alloc_workspace()
    W = [torch.randn(r, c, device="cuda", generator=gen).mul_(w.weight_std)
         for r, c in w.shapes]
    M = [torch.zeros_like(x) for x in W]
    G = [torch.randn(r, c, device="cuda", generator=gen).mul_(w.grad_std)
         .to(torch.bfloat16) for r, c in w.shapes]
    extra = [torch.randn(n, device="cuda", generator=gen).mul_(0.02)
             for n in w.ema_extra_numels]
    E = [x.clone().view(-1) for x in W] + [x.clone() for x in extra]
    P = [x.view(-1) for x in W] + extra
    muon = plan.bind(W, M, G, w.hyper, w.coeffs, ws, update_scales=wl.update_scales(w))
    ema = B.ema_bind(E, P, w.ema_decay)

    def step():
        muon()
        ema()

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    if plan.last_error() != 0:
        raise RuntimeError("device-side error in the 24L warm-up")
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            step()
    stream.wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(replays):
        graph.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / replays
    del graph
    # per-kernel split from eager steps (plan events; the EMA on own events)
    plan.set_timing(True)
    plan.timing_read()
    n_eager = 3
    e_ms = 0.0
    for _ in range(n_eager):
        muon()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        ema()
        a1.record(stream)
        torch.cuda.synchronize()
        e_ms += a0.elapsed_time(a1)
    phase = plan.timing_read()
    plan.set_timing(False)
    if plan.last_error() != 0:
        raise RuntimeError("device-side error in the 24L timing")
    ns_ms = phase["ns"][1] / max(phase["ns"][0], 1)
    pro_ms = phase["prologue"][1] / max(phase["prologue"][0], 1)
    ema_ms = e_ms / n_eager
    ema_params = sum(w.ema_numels())
    ema_gbs = 12 * ema_params / (ema_ms / 1e3) / 1e9
    dense = sum(2 * min(r, c) ** 2 * max(r, c) * 2 + 2 * min(r, c) ** 3
                for r, c in w.shapes) * len(w.coeffs)
    sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    rec = {"workload": w.name, "n_mats": w.n_mats, "matrix_params": w.numel(),
           "ema_params": ema_params, "ns_steps": len(w.coeffs),
           "data": "synthetic, drawn on the device (torch.Generator seed 1337): "
                   "W ~ N(0, 0.02^2), G ~ N(0, 1e-3^2) in bf16, E = W, M = 0",
           "steps_per_s": round(1e3 / ms, 3), "ms_per_step": round(ms, 3),
           "replays": replays, "mode": "CUDA graph replay (one graph per step)",
           "clocks": clk,
           "ns": ns_record(ns_ms, dense, ns_issued_flops(w), sustained,
                           f"{peak_src} sustained (a ~40 ms kernel in a "
                           "seconds-long loop)"),
           "prologue": prologue_record(pro_ms, w.numel(), peaks["hbm_gbs"]),
           "ema": {"ms": round(ema_ms, 4), "gbs": round(ema_gbs, 1),
                   "frac": round(ema_gbs / peaks["hbm_gbs"], 4), "bytes_per_param": 12},
           "per_kernel_from": f"{n_eager} eager steps, CUDA events on the stream"}
    plan.close()
    del W, M, G, E, P, extra, ws
    torch.cuda.empty_cache()
    return rec


def adamw_ema_measure(w, stream, reps):
    """Device time of one adamw_ema_batched launch over the non-matrix
    parameters of the 11L x 512d model (None for other workloads)."""
    import torch
    from muon_optimizer_step_02_b200 import binding as B
    if w.ema_decay is None or w.n_mats != 66:
        return None
    numels, _ = wl.gpt11_ema_extras()
    P, G, M, V, E = [], [], [], [], []
    for i, n in enumerate(numels):
        p, m, v, e = wl.adamw_state(n, i)
        P.append(torch.from_numpy(p).cuda())
        M.append(torch.from_numpy(m).cuda())
        V.append(torch.from_numpy(v).cuda())
        E.append(torch.from_numpy(e).cuda())
        G.append(torch.from_numpy(wl.adamw_grad(n, i, 1)).cuda())
    hyp = type("AdamW", (), dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8,
                                 weight_decay=0.0))
    run = B.adamw_ema_bind(P, G, M, V, E, hyp, w.ema_decay)
    flush = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    for t in range(1, 4):
        run(step_now=t)
    total = 0.0
    for t in range(reps):
        flush.sum()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        run(step_now=4 + t)
        a1.record(stream)
        torch.cuda.synchronize()
        total += a0.elapsed_time(a1)
    del flush
    return total / reps, sum(numels)


def ns_issued_flops(w: wl.Workload) -> int:
    """FLOPs the tensor cores issue in one Newton-Schulz launch: whole
    256 x 256 pair tiles and 64-deep K blocks (the ragged edges zero-padded),
    the gram and polynomial products on the upper pair tiles only."""
    def cdiv(a, b):
        return -(-a // b)
    blocks = 0
    for r, c in w.shapes:
        m, n = min(r, c), max(r, c)
        t2, tn = cdiv(m, 256), cdiv(n, 256)
        sym = t2 * (t2 + 1) // 2
        blocks += sym * cdiv(n, 64) + sym * cdiv(m, 64) + t2 * tn * cdiv(m, 64)
    return blocks * 2 * 256 * 256 * 64 * len(w.coeffs)


def torch_ns_yardstick(w: wl.Workload, stream, reps: int):
    """The same Newton-Schulz work as cuBLAS batched GEMMs through torch, as a
    yardstick for the fused kernel (not part of the library): per group of
    equal working shapes, every step runs A = X X^T, B = b A + c A A and
    X <- a X + B X (bmm and two baddbmm, bf16 in and out, the full dense
    products), all steps replayed from one CUDA graph.  Returns the device
    time of one replay in ms."""
    import torch
    groups = {}
    for r, c in w.shapes:
        key = (min(r, c), max(r, c))
        groups[key] = groups.get(key, 0) + 1
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    bufs = []
    for (m, n), cnt in groups.items():
        x0 = (torch.randn(cnt, m, n, device="cuda", generator=gen)
              / float(np.sqrt(m * n))).to(torch.bfloat16)
        bufs.append((x0, torch.empty_like(x0), torch.empty_like(x0),
                     torch.empty(cnt, m, m, device="cuda", dtype=torch.bfloat16),
                     torch.empty(cnt, m, m, device="cuda", dtype=torch.bfloat16)))

    def ns():
        cur = [b[0] for b in bufs]
        for k, (a, b, c) in enumerate(w.coeffs):
            for i, (_, x1, x2, A, Bm) in enumerate(bufs):
                x = cur[i]
                torch.bmm(x, x.transpose(1, 2), out=A)
                torch.baddbmm(A, A, A, beta=b, alpha=c, out=Bm)
                nxt = x1 if k % 2 == 0 else x2
                torch.baddbmm(x, Bm, x, beta=a, alpha=1.0, out=nxt)
                cur[i] = nxt

    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        ns()                                   # cuBLAS handles and workspaces
        side.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            ns()
    stream.wait_stream(side)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    y0 = torch.cuda.Event(enable_timing=True)
    y1 = torch.cuda.Event(enable_timing=True)
    y0.record(stream)
    for _ in range(reps):
        graph.replay()
    y1.record(stream)
    torch.cuda.synchronize()
    del graph
    return y0.elapsed_time(y1) / reps


# --------------------------------------------------------------------------
# the fp64 oracle on the host cores
# --------------------------------------------------------------------------
def oracle_sample(w: wl.Workload, budget_s: float, seed: int = 1337):
    """Times the oracle on whole layers (6 matrices each, in model order) plus
    the EMA over the same fraction of the parameters, until about budget_s
    seconds of CPU work; returns (seconds per full step, description,
    threads)."""
    import oracle.muon_oracle as mo
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()]
                      or [os.cpu_count()])
    except Exception:
        threads = os.cpu_count()
    hyp = mo.MuonHyper(momentum=w.hyper.momentum, lr=w.hyper.lr,
                       weight_decay=w.hyper.weight_decay,
                       eps_row=w.hyper.eps_row, eps_frob=w.hyper.eps_frob,
                       nesterov=w.hyper.nesterov, eq_r=w.hyper.eq_r)
    scales = wl.update_scales(w)
    per_layer = 6 if w.n_mats % 6 == 0 else 1
    n_groups = w.n_mats // per_layer
    done, spent = 0, 0.0
    while done < n_groups and spent < budget_s:
        idx = range(done * per_layer, (done + 1) * per_layer)
        ins = [(wl.weight(w, i, seed).astype(np.float64),
                np.zeros(w.shapes[i]),
                wl.bf16_bits_to_f32(wl.grad_bits(w, i, 0, seed))
                .astype(np.float64)) for i in idx]
        t = time.perf_counter()
        for (W, M, G), i in zip(ins, idx):
            mo.muon_step(W, M, G, hyp, w.coeffs, scales[i])
        spent += time.perf_counter() - t
        done += 1
    frac = done / n_groups
    ema_s = 0.0
    if w.ema_decay is not None:
        total = sum(w.ema_numels())
        n = max(int(total * frac), 1)
        E = np.random.default_rng(0).standard_normal(n).astype(np.float32) * 0.02
        P = np.random.default_rng(1).standard_normal(n).astype(np.float32) * 0.02
        t = time.perf_counter()
        mo.ema_update(E, P, w.ema_decay)
        ema_s = time.perf_counter() - t
    step_s = (spent + ema_s) / frac
    desc = (f"{done * per_layer} of {w.n_mats} matrices (whole layers) + EMA "
            f"over the same fraction of {sum(w.ema_numels())} params, "
            f"extrapolated x{1 / frac:.2f}")
    return step_s, desc, threads


def run_reference(args, rank):
    if rank != 0:
        return None
    w = load_workload(args.workload)
    budget = float(os.environ.get("MUONB200_ORACLE_BUDGET_S", "20"))
    times, desc, threads = [], "", os.cpu_count()
    for _ in range(args.warmup):
        oracle_sample(w, budget / 4)
    for _ in range(args.steps):
        s, desc, threads = oracle_sample(w, budget / max(args.steps, 1))
        times.append(s)
    step_s = statistics.mean(times)
    value = 1.0 / step_s
    return {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "impl": "reference", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "n_mats": w.n_mats,
                   "ns_steps": len(w.coeffs)},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT,
                         "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 6), "unit": UNIT,
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", type=int, default=6)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-yardstick", action="store_true",
                    help="skip timing the same Newton-Schulz work as torch/cuBLAS GEMMs")
    ap.add_argument("--repeats", type=int, default=5,
                    help="timed blocks of --steps steps; the median is reported")
    ap.add_argument("--no-largest", action="store_true",
                    help="skip the 24L x 2048d sub-record")
    ap.add_argument("--largest-replays", type=int, default=20)
    ap.add_argument("--eager", action="store_true",
                    help="time eager launches instead of one CUDA graph per step")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if line is None:
        return
    # the oracle's host-core baseline belongs to the one-GPU line only
    if not args.no_cpu_baseline and world == 1:
        budget = float(os.environ.get("MUONB200_ORACLE_BUDGET_S", "15"))
        s, desc, threads = oracle_sample(load_workload(args.workload), budget)
        line["cpu_baseline"] = {"value": round(1.0 / s, 6), "unit": UNIT,
                                "cores": threads, "kind": "oracle",
                                "sample": desc}
        # the same oracle on one host thread (BLAS limited to one thread),
        # over a smaller sample
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                s1, desc1, _ = oracle_sample(load_workload(args.workload), budget / 3)
            line["cpu_baseline"]["one_thread"] = {"value": round(1.0 / s1, 6),
                                                  "unit": UNIT, "sample": desc1}
        except ImportError:
            pass
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
