"""Benchmark: fused exact attention on B200 (forward + backward step, plus
the split-KV decode).

One step = the whole training hot path on one batch of the causal workload
B=8, H=16, N=2048, d=128, bf16: fa_fwd (forward kernel), then fa_bwd
(D = rowsum(dO∘O) preprocessing, the backward kernel, the dQ finalise).
``value`` is fwd+bwd TFLOPS over all ranks, counting 4·B·H·N²·d/2 for the
forward and 2.5× that for the backward (causal halves both).  Inputs live in
HBM before the timed region; each step touches ~0.4 GB, larger than the
126 MB L2, so no flush is inserted.  The decode workload (B=32, H=32,
Nk=32768, d=128) is timed separately and reported under "decode", and the
other training workloads (B4 H16 N1024 d64, B1 H32 N16384 d128 causal with
Q×3, the causal 2K one in fp16, and again with a head-shared additive bias)
under "other_workloads", each with its fwd, bwd and fwd+bwd TFLOPS against
both measured bf16 peaks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun each rank runs its own copy of the workload (attention heads
are independent: no collective on the data path; weak scaling); times are
the max over ranks.  ``--impl reference`` times the fp64 CPU oracle instead
(a bounded sample of the same workload, rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "attention fwd+bwd TFLOPS (bf16, 1xB200 per rank)"
UNIT = "TFLOP/s"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            return json.load(f), "measured"
    except OSError:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary
    (profiles/dram_traffic.json), or None when one of the kernel's sources
    listed there changed since that capture (sha256 mismatch)."""
    import hashlib

    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f)[kernel]
        m = hashlib.sha256()
        for p in rec["sources"]:
            with open(os.path.join(ROOT, p), "rb") as f:
                m.update(f.read())
    except (OSError, KeyError, ValueError):
        return None
    return rec["bytes_per_launch"] if m.hexdigest() == rec["source_sha256"] else None


def reduce_max(x: float, pg, device) -> float:
    """Max of a per-rank float over all ranks (identity without a group)."""
    if pg is None:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w, rank: int):
    """Each rank runs its own replica of the workload, drawn from its own seed."""
    return W.Workload(**{**w.__dict__, "seed": w.seed + rank})


def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """SM clock, power and throttle reasons sampled DURING the timed region.

    A thread polls NVML about every 2 ms (the driver's default 20-step
    region lasts ~15 ms, far shorter than nvidia-smi's sampling period), and
    one sample is taken right at the start and one right at the end of the
    region, so even a short region has a record.  Without NVML the record
    says so and holds no samples."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int):
        import threading

        self.dev = device_index
        self.samples = []
        self.smax = None
        self.handle = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nvml = pynvml
            props = torch.cuda.get_device_properties(device_index)
            try:
                self.handle = pynvml.nvmlDeviceGetHandleByUUID(f"GPU-{props.uuid}")
            except Exception:  # noqa: BLE001 - fall back to the PCI address
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - NVML missing or the device not found
            self.handle = None

    def sample(self):
        if self.handle is None:
            return
        n = self.nvml
        try:
            self.samples.append((n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM),
                                 n.nvmlDeviceGetPowerUsage(self.handle) / 1000.0,
                                 n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)))
        except Exception:  # noqa: BLE001
            pass

    def _run(self):
        while not self._stop.wait(0.002):
            self.sample()

    def start(self):
        """Call right before the timed region (after any warm-up)."""
        import threading

        self.samples = []
        self._stop.clear()
        self.sample()
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    def stop(self):
        """Call right after the timed region; returns the summary."""
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        self.sample()
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["NVML unavailable"],
                    "samples": 0}
        sm = [c for c, _, _ in self.samples]
        pw = [p for _, p, _ in self.samples]
        reasons = sorted({name for _, _, r in self.samples
                          for name, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_min_mhz": min(sm) if sm else None,
                "sm_max_mhz": self.smax, "power_w": statistics.median(pw) if pw else None,
                "reasons": reasons, "samples": len(sm), "source": "nvml, ~2 ms"}


def time_oracle_sample(w, budget_s=12.0):
    """fp64 oracle fwd+bwd on whole heads of the workload until ~budget_s of
    CPU time; returns (TFLOP/s, heads, seconds, cores)."""
    import numpy as np

    import oracle

    q, k, v, do = W.make_tensors(1, 1, w.Nq, w.Nk, w.d, w.dtype, seed=w.seed, q_mult=w.q_mult)
    f = lambda t: t[0, 0].float().double().numpy()
    qh, kh, vh, doh = f(q), f(k), f(v), f(do)
    heads, t0 = 0, time.perf_counter()
    while True:
        oracle.head_forward(qh, kh, vh, w.scale, w.causal)
        oracle.head_backward(qh, kh, vh, doh, w.scale, w.causal)
        heads += 1
        el = time.perf_counter() - t0
        if el >= budget_s or heads >= w.B * w.H:
            break
    flops_per_head = (w.fwd_flops + w.bwd_flops) / (w.B * w.H)
    cores = len(os.sched_getaffinity(0))
    return flops_per_head * heads / el / 1e12, heads, el, cores


def run_reference(args, w):
    world, rank, _ = dist_info()
    if rank != 0:
        return
    per_step, heads_total, el_total = [], 0, 0.0
    # About a minute of oracle work over the whole run (at least one head per
    # step, ~0.13 s), whatever K and W are.
    for i in range(args.warmup + args.steps):
        tf, heads, el, cores = time_oracle_sample(w, budget_s=60.0 / (args.warmup + args.steps))
        if i >= args.warmup:
            per_step.append(el)
            heads_total += heads
            el_total += el
    flops = (w.fwd_flops + w.bwd_flops) / (w.B * w.H) * heads_total
    value = flops / el_total / 1e12
    sample = f"{heads_total} of {w.B * w.H} heads per {args.steps} steps, fp64 numpy fwd+bwd"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "shape": w.describe(), "global_batch": w.B, "seq_len": w.Nq,
                   "parallelism": f"replicas{world}"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def peak_fracs(achieved, peaks):
    """achieved TFLOP/s against both measured bf16 peaks."""
    return {"frac_burst": achieved / float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])),
            "frac_sustained": achieved / float(peaks.get("bf16_tflops_sustained",
                                                         FALLBACK_PEAKS["bf16_tflops_sustained"]))}


def fill_queue():
    """Keep the device busy for ~10 ms (a bounded spin of torch's own) before
    a timed region starts, so that the host has queued the region's launches
    by the time the device reaches them: a short region (20 steps of the
    causal 2K workload are ~13 ms of device work) then measures the device,
    not the Python launch path and the clock-sampling thread."""
    torch.cuda._sleep(20_000_000)


def time_workload(fa, w, dev, stream, iters, peaks, peak_kind, flush=None, bias_shape=None,
                  sampler=None):
    """fwd and bwd of one workload, each launch bracketed by CUDA events on
    the launching stream (the main backward kernel by the library's own
    timing events); with ``flush`` (a buffer larger than L2) L2 is cleared
    before every timed launch; with ``bias_shape`` an additive N(0, 1) bias
    of that (broadcastable) shape is added to the scores.  FLOPs are counted
    without the bias.  The timed loop starts after a short pause, so that a
    workload is not measured at the clock its predecessor left (a long one
    runs into the power cap), and ``sampler`` records the clocks during it.
    Returns the workload's sub-object."""
    q, k, v, do = W.make_inputs(w, device=dev)
    bias = None
    if bias_shape is not None:
        g = torch.Generator(device=dev).manual_seed(w.seed + 1)
        bias = torch.randn(*bias_shape, generator=g, device=dev).to(q.dtype)
    O, L = fa.forward(q, k, v, causal=w.causal, bias=bias)
    dq, dk, dv = (torch.empty_like(x) for x in (q, k, v))
    ws = torch.empty(fa.bwd_workspace_bytes(w.B, w.H, w.Nq, w.Nk, w.d, q.dtype), dtype=torch.uint8,
                     device=dev)

    def fwd():
        fa.forward(q, k, v, causal=w.causal, out=O, lse=L, bias=bias)

    def bwd():
        fa.backward(q, k, v, O, do, L, causal=w.causal, dq=dq, dk=dk, dv=dv, workspace=ws, bias=bias)

    for _ in range(3):
        fwd()
        bwd()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(iters)]
    for e in ev:
        for x in e:
            x.record(stream)
    torch.cuda.synchronize()
    time.sleep(0.3)
    if sampler is not None:
        sampler.start()
    fill_queue()
    for e in ev:
        if flush is not None:
            flush.zero_()
        e[0].record(stream)
        fwd()
        e[1].record(stream)
        if flush is not None:
            flush.zero_()
        e[2].record(stream)
        fa.set_bwd_timing_events(e[4], e[5])
        bwd()
        e[3].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler is not None else None
    fa.set_bwd_timing_events(None, None)
    st = fa.status()
    if st != fa.FA_OK:
        raise RuntimeError(f"{w.name}: kernel status {fa.STATUS_NAMES.get(st, st)}")
    f_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    b_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    m_ms = statistics.mean(e[4].elapsed_time(e[5]) for e in ev)
    f_tf = w.fwd_flops / (f_ms * 1e-3) / 1e12
    b_tf = w.bwd_flops / (b_ms * 1e-3) / 1e12
    fb_tf = (w.fwd_flops + w.bwd_flops) / ((f_ms + b_ms) * 1e-3) / 1e12
    main_tf = w.bwd_flops / (m_ms * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    if w.dtype == "fp16":  # the same dense tensor rate as bf16 (kind::f16 MMAs)
        pk = f"{peak_kind} burst bf16 (fp16 runs at the bf16 rate)"
    else:
        pk = f"{peak_kind} burst bf16"
    name, shape = w.name, w.describe()
    if bias_shape is not None:
        name += "_bias" + "x".join(str(x) for x in bias_shape)
        shape += f", additive bias {list(bias_shape)} (FLOPs counted without it)"
    return {"workload": name, "shape": shape, "iters": iters,
            "l2": "flushed before every timed launch" if flush is not None
                  else "inputs larger than L2; no flush",
            "fwd": {"ms": f_ms, "tflops": f_tf, **peak_fracs(f_tf, peaks)},
            "bwd": {"ms": b_ms, "tflops": b_tf, "main_kernel_ms": m_ms,
                    "main_kernel_tflops": main_tf, **peak_fracs(b_tf, peaks)},
            "fwd_bwd": {"ms": f_ms + b_ms, "tflops": fb_tf, **peak_fracs(fb_tf, peaks)},
            "roofline": {"bound": "tensor", "kernel": "bwd_main_kernel", "achieved": main_tf,
                         "peak": peak, "unit": UNIT, "frac": main_tf / peak, "peak_kind": pk},
            "clocks": clocks}


# Decode shape for kernel captures: the decode workload with B = 4 instead of
# 32 (2.1 GB of K/V, far larger than L2, within a capture's memory budget);
# its bytes per key row are those of the full workload.
DECODE_PROFILE = W.Workload("decode_b4h32nk32768d128", 4, 32, 1, 32768, 128, False, "bf16",
                            decode=True)


def profile_case(name: str):
    """Three launches of one kernel's case: the causal B8 H16 N2048 d128
    forward (``fwd_bias``: with the bench's head-shared [1, 16, 2048, 2048]
    additive bias) or backward, or the reduced decode shape.  A capture
    skips the first two launches of the kernel (``-s 2 -c 1``)."""
    import exact_attention_115_b200 as fa

    dev = torch.device("cuda", 0)
    w = DECODE_PROFILE if name == "decode" else W.CAUSAL_2K
    q, k, v, do = W.make_inputs(w, device=dev, with_grad=name == "bwd")
    bias = None
    if name == "fwd_bias":
        g = torch.Generator(device=dev).manual_seed(w.seed + 1)
        bias = torch.randn(1, w.H, w.Nq, w.Nk, generator=g, device=dev).to(q.dtype)
    if name == "decode":
        for _ in range(3):
            fa.decode(q, k, v)
    else:
        O, L = fa.forward(q, k, v, causal=w.causal, bias=bias)
        for _ in range(3 if name == "bwd" else 2):
            if name == "bwd":
                fa.backward(q, k, v, O, do, L, causal=w.causal)
            else:
                fa.forward(q, k, v, causal=w.causal, out=O, lse=L, bias=bias)
    torch.cuda.synchronize(dev)
    st = fa.status()
    print(f"profile case {name}: {w.describe()} status {fa.STATUS_NAMES.get(st, st)}")
    if st != fa.FA_OK:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # ~1 s of timed steps by default, so that the 100 ms clock samples see the
    # kernels under sustained load (power cap included)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads (B4 H16 N1024 d64, the 16K causal one, fp16, with a bias)")
    ap.add_argument("--profile-case", choices=["fwd", "fwd_bias", "bwd", "decode"],
                    help="run one kernel's small profiling case three times and exit "
                         "(the command an ncu capture wraps; nothing is timed)")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return
    w = W.CAUSAL_2K
    if args.impl == "reference":
        run_reference(args, w)
        return

    world, rank, local = dist_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    import exact_attention_115_b200 as fa

    fa.lib()
    peaks, peak_kind = load_peaks()
    stream = torch.cuda.current_stream(dev)

    q, k, v, do = W.make_inputs(rank_workload(w, rank), device=dev)
    O, L = fa.forward(q, k, v, causal=True)
    dq, dk, dv = (torch.empty_like(x) for x in (q, k, v))
    ws = torch.empty(fa.bwd_workspace_bytes(w.B, w.H, w.Nq, w.Nk, w.d), dtype=torch.uint8,
                     device=dev)

    def step():
        fa.forward(q, k, v, causal=True, out=O, lse=L)
        fa.backward(q, k, v, O, do, L, causal=True, dq=dq, dk=dk, dv=dv, workspace=ws)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    st = fa.status()
    if st != fa.FA_OK:
        raise RuntimeError(f"kernel status after warm-up: {fa.STATUS_NAMES.get(st, st)}, "
                           f"first timed-out wait {fa.lib().fa_last_timeout_site()}")

    # The timed region: K plain steps, nothing recorded between the kernels.
    K = args.steps
    sampler = ClockSampler(local)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    fill_queue()
    t_start.record(stream)
    for _ in range(K):
        step()
    t_stop.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if pg:
        pg.barrier()
    st = fa.status()
    if st != fa.FA_OK:
        raise RuntimeError(f"kernel status {fa.STATUS_NAMES.get(st, st)}, "
                           f"first timed-out wait {fa.lib().fa_last_timeout_site()}")

    # The breakdown, after the timed region: K more steps with events around
    # the forward, the whole backward and (recorded by the library) the main
    # backward kernel.
    ev = {n: [torch.cuda.Event(enable_timing=True) for _ in range(K)]
          for n in ("s0", "f1", "b0", "b1", "s1")}
    # (torch's elapsed_time wants every event recorded through torch once;
    # b0 and b1 are then re-recorded by the library around the main kernel)
    for lst in ev.values():
        for e in lst:
            e.record(stream)
    for i in range(K):
        ev["s0"][i].record(stream)
        fa.forward(q, k, v, causal=True, out=O, lse=L)
        ev["f1"][i].record(stream)
        fa.set_bwd_timing_events(ev["b0"][i], ev["b1"][i])
        fa.backward(q, k, v, O, do, L, causal=True, dq=dq, dk=dk, dv=dv, workspace=ws)
        ev["s1"][i].record(stream)
    torch.cuda.synchronize()
    fa.set_bwd_timing_events(None, None)
    st = fa.status()
    if st != fa.FA_OK:
        raise RuntimeError(f"kernel status {fa.STATUS_NAMES.get(st, st)} in the breakdown pass")

    total_ms = t_start.elapsed_time(t_stop)
    fwd_ms = [ev["s0"][i].elapsed_time(ev["f1"][i]) for i in range(K)]
    bwd_main_ms = [ev["b0"][i].elapsed_time(ev["b1"][i]) for i in range(K)]
    bwd_ms = [ev["f1"][i].elapsed_time(ev["s1"][i]) for i in range(K)]
    total_ms = reduce_max(total_ms, pg, dev)
    ms_per_step = total_ms / K
    flops_step = w.fwd_flops + w.bwd_flops
    value = flops_step * K * world / (total_ms * 1e-3) / 1e12

    fwd_avg = statistics.mean(fwd_ms)
    bwd_main_avg = statistics.mean(bwd_main_ms)
    bwd_avg = statistics.mean(bwd_ms)
    # A timed region of half a second or more runs the kernels at the power
    # cap: their peak is the sustained GEMM figure; shorter runs take the burst.
    sustained = total_ms >= 500.0
    pkey = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    peak_bf16 = float(peaks.get(pkey, FALLBACK_PEAKS[pkey]))
    achieved_bwd = w.bwd_flops / (bwd_main_avg * 1e-3) / 1e12
    achieved_fwd = w.fwd_flops / (fwd_avg * 1e-3) / 1e12

    # End to end through the same public API: pinned host inputs copied in,
    # outputs (O, L, dQ, dK, dV) copied back, every step inside the region.
    e2e = None
    if rank == 0 or world > 1:
        hq, hk, hv, hdo = (x.cpu().pin_memory() for x in (q, k, v, do))
        ho, hl = torch.empty_like(hq).pin_memory(), torch.empty(L.shape, dtype=L.dtype).pin_memory()
        hdq, hdk, hdv = (torch.empty_like(x).pin_memory() for x in (hq, hk, hv))
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hdo))
        d2h = sum(x.numel() * x.element_size() for x in (ho, hl, hdq, hdk, hdv))
        ksteps = max(3, min(K, 10))
        # Pipelined by batch element: chunk c's inputs go in on one copy
        # stream while earlier chunks compute on the main stream and finished
        # chunks come back on another, so the PCIe transfers in both
        # directions overlap each other and the kernels.  Same public calls,
        # same bytes, every step.
        nck = w.B
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(nck)]
        ev_comp = [torch.cuda.Event() for _ in range(nck)]
        ev_out = [torch.cuda.Event() for _ in range(nck)]
        ws1 = torch.empty(fa.bwd_workspace_bytes(1, w.H, w.Nq, w.Nk, w.d), dtype=torch.uint8,
                          device=dev)
        started = [False] * nck

        def e2e_step():
            for c in range(nck):
                sl = slice(c, c + 1)
                with torch.cuda.stream(s_in):
                    if started[c]:
                        s_in.wait_event(ev_comp[c])  # the previous step's chunk c has read its inputs
                    for hsrc, dst in ((hq, q), (hk, k), (hv, v), (hdo, do)):
                        dst[sl].copy_(hsrc[sl], non_blocking=True)
                    ev_in[c].record(s_in)
                stream.wait_event(ev_in[c])
                if started[c]:
                    stream.wait_event(ev_out[c])  # its outputs went back to the host
                fa.forward(q[sl], k[sl], v[sl], causal=True, out=O[sl], lse=L[sl])
                fa.backward(q[sl], k[sl], v[sl], O[sl], do[sl], L[sl], causal=True,
                            dq=dq[sl], dk=dk[sl], dv=dv[sl], workspace=ws1)
                ev_comp[c].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[c])
                    for src, hdst in ((O, ho), (L, hl), (dq, hdq), (dk, hdk), (dv, hdv)):
                        hdst[sl].copy_(src[sl], non_blocking=True)
                    ev_out[c].record(s_out)
                started[c] = True
            stream.wait_event(ev_out[nck - 1])  # the step ends when its last outputs are home

        e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_in.wait_stream(stream)
        for _ in range(ksteps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        et = reduce_max(a.elapsed_time(b), pg, dev)
        e2e = {"value": flops_step * ksteps * world / (et * 1e-3) / 1e12,
               "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": ksteps}

    # The other workloads' fwd, bwd and fwd+bwd, each timed on its own (no
    # collective: every rank runs its own copy and rank 0 reports its own).
    del dq, dk, dv, ws, q, k, v, do, O, L
    torch.cuda.empty_cache()
    others = None
    if not args.no_extra:
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        flush = torch.empty(4 * l2, dtype=torch.uint8, device=dev)  # written before each launch
        iters = max(5, min(K, 20))
        others = [time_workload(fa, W.MEDIUM, dev, stream, iters, peaks, peak_kind, flush=flush,
                                sampler=sampler),
                  time_workload(fa, W.LONG_16K, dev, stream, iters, peaks, peak_kind, sampler=sampler),
                  time_workload(fa, W.CAUSAL_2K_FP16, dev, stream, iters, peaks, peak_kind,
                                sampler=sampler),
                  time_workload(fa, W.CAUSAL_2K, dev, stream, iters, peaks, peak_kind,
                                bias_shape=(1, W.CAUSAL_2K.H, W.CAUSAL_2K.Nq, W.CAUSAL_2K.Nk),
                                sampler=sampler)]
        del flush
        torch.cuda.empty_cache()

    # Decode (split-KV + combine), timed on its own.
    decode = None
    if not args.no_decode:
        wd = W.DECODE_32K
        dq_, dk_, dv_, _ = W.make_inputs(wd, device=dev, with_grad=False)
        Od, Ld = fa.decode(dq_, dk_, dv_)
        wsd = torch.empty(fa.decode_workspace_bytes(wd.B, wd.H, wd.Nk, wd.d), dtype=torch.uint8,
                          device=dev)
        for _ in range(3):
            fa.decode(dq_, dk_, dv_, out=Od, lse=Ld, workspace=wsd)
        torch.cuda.synchronize()
        nd = 10
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(nd):
            fa.decode(dq_, dk_, dv_, out=Od, lse=Ld, workspace=wsd)
        b.record(stream)
        torch.cuda.synchronize()
        dms = a.elapsed_time(b) / nd
        kv_bytes = 2 * wd.B * wd.H * wd.Nk * wd.d * 2
        gbs = kv_bytes / (dms * 1e-3) / 1e9
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        decode = {"workload": wd.name, "shape": wd.describe(), "ms": dms, "value": gbs,
                  "unit": "GB/s", "l2": "17.2 GB of K/V per call, far larger than L2",
                  "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                               "frac": gbs / hbm, "peak_kind": peak_kind,
                               "traffic": kernel_traffic("decode_split_kernel"),
                               "traffic_unit": "bytes per launch of decode_split_kernel "
                                               "(ncu dram read+write, 8x a B=4 capture)"}}
        assert fa.status() == fa.FA_OK

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, heads, el, cores = time_oracle_sample(w)
        cpu = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{heads} of {w.B * w.H} heads fwd+bwd in fp64 numpy ({el:.1f} s)"}

    if rank != 0:
        if pg:
            pg.destroy_process_group()
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "shape": w.describe(), "global_batch": w.B * world,
                   "seq_len": w.Nq, "heads": w.H, "head_dim": w.d, "causal": True,
                   "parallelism": f"replicas{world}",
                   "l2": "inputs ~0.4 GB per step > 126 MB L2; no flush"},
        "fwd": {"ms": fwd_avg, "tflops": achieved_fwd, **peak_fracs(achieved_fwd, peaks)},
        "bwd": {"ms": bwd_avg, "tflops": w.bwd_flops / (bwd_avg * 1e-3) / 1e12,
                "main_kernel_ms": bwd_main_avg,
                "timing": "a second pass of K steps after the timed region, with events "
                          "around the forward, the backward and its main kernel",
                **peak_fracs(w.bwd_flops / (bwd_avg * 1e-3) / 1e12, peaks)},
        # the 60 % target of the fwd+bwd step is stated against the burst
        # (isolated-GEMM) peak; the sustained one is the figure under the
        # power cap that a long run reaches
        "pct_of_peak": value / world / peak_bf16,
        "step_fracs": {**peak_fracs(value / world, peaks), "target": 0.60,
                       "target_uses": "frac_burst"},
        "roofline": {"bound": "tensor", "kernel": "bwd_main_kernel", "achieved": achieved_bwd,
                     "peak": peak_bf16, "unit": "TFLOP/s", "frac": achieved_bwd / peak_bf16,
                     **peak_fracs(achieved_bwd, peaks),
                     "peak_kind": f"{peak_kind} {'sustained' if sustained else 'burst'} bf16",
                     "fwd_kernel": {"achieved": achieved_fwd, **peak_fracs(achieved_fwd, peaks),
                                    "traffic": kernel_traffic("fwd_kernel")},
                     "traffic": kernel_traffic("bwd_main_kernel"),
                     "traffic_unit": "bytes per launch (ncu dram read+write)"},
        "e2e": e2e,
        "gpu_launches": 4 * K,
        "clocks": clocks,
        "decode": decode,
        "other_workloads": others,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
