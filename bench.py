"""Benchmark of the Parallax hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload W]

One step = one pass of the whole hot path over one batch of synthetic input:
  * decode  (headline, 1.7B-layer decode step): parallax_decode on B=64, H=16,
    d=128 against a contiguous 4096-token bf16 KV cache -> HBM TB/s;
  * prefill (1.7B-layer prefill): parallax_rho_proj (x [8,4096,2048] @ W_R
    [2048,2048]) then parallax_fwd (B=8, T=4096, H=16, d=128, causal) -> TFLOP/s
    counted as 8d flops per unmasked (i, j) pair (the four UMMAs).
``value`` is the decode throughput; the prefill numbers ride in ``prefill``.
All inputs are seeded synthetic data already resident in HBM; every input set
is larger than the 126 MB L2, so no flush is needed between steps.

The reference arm (--impl reference) times the fp64 CPU oracle on the host
cores on a bounded sample of the same workloads and prints the same line.
With N > 1 (torchrun) each rank runs an independent replica (the operator has
no cross-GPU exchange); time is the max over ranks and value sums the ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Parallax attn: decode HBM TB/s, prefill TFLOP/s, % of roofline (1×B200)"
DECODE_CFG = dict(B=64, H=16, Tcap=4096, d=128)
PREFILL_CFG = dict(B=8, T=4096, H=16, d=128, d_model=2048)
LONG_CFG = dict(B=1, T=32768, H=16, d=128, d_model=2048)


def rank_env():
    """(rank, world, local_rank) as the launcher (torchrun) sets them; one process per GPU."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, world, device):
    """Element-wise max of per-rank timings over the process group: the slowest rank times the job."""
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank, max_ms, world):
    """Units all ranks processed per second (every rank runs the same work: weak scaling, replicas)."""
    return world * units_per_rank / (max_ms * 1e-3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def decode_bytes(B, H, d, seqlens):
    """Algorithmic bytes of one decode call: K and V rows read + q, rho read + y (fp32) written."""
    kv = int(np.sum(seqlens)) * H * d * 2 * 2
    return kv + B * H * d * 2 * 2 + B * H * d * 4


# DRAM bytes per algorithmic byte of the decode split kernel, from an ncu
# capture of the default step's decode (B=64 H=16 ctx 4096: 2.148242 GB read +
# 0.008331 GB written for 2.148532 GB of K/V rows, q, rho and y; the B=16
# ctx 8192 capture gave 1.009).  Traffic grows in proportion to the cached
# tokens read, so a launch's traffic is this ratio times its algorithmic bytes.
DECODE_TRAFFIC_RATIO = (2.148242 + 0.008331) / 2.148532

# DRAM bytes of one prefill forward kernel launch (ncu, dram__bytes_read.sum +
# dram__bytes_write.sum of k_fwd) at the two prefill shapes the bench runs,
# beside its algorithmic bytes (q, k, rho and the fp16 V read once, y written):
# the K/V tiles are re-read from DRAM by the query tiles of a head whose
# earlier reads have left L2.
PREFILL_TRAFFIC = {(8, 4096): 3.934873e9 + 0.248365e9, (1, 32768): 4.051134e9 + 0.250774e9}


def prefill_pairs(B, H, T, causal=True):
    return B * H * (T * (T + 1) // 2 if causal else T * T)


def prefill_flops(B, H, T, d):
    return 8 * d * prefill_pairs(B, H, T)


def rho_proj_flops(B, T, d_model, H, d):
    return 2 * B * T * d_model * H * d


# --------------------------------------------------------------------------- #
# clocks sampled during the timed region
# --------------------------------------------------------------------------- #
class ClockSampler:
    """SM clock and clock-event reasons of the benchmark's GPU while the timed
    region runs.  NVML is read from a background thread every 5 ms (the timed
    region can be a few tens of ms); only the samples taken between mark_start()
    and mark_end() count (the nearest ones if none fell inside).  The device is
    matched to the CUDA device by PCI bus id.  Without NVML, nvidia-smi at its
    shortest interval is the fallback.  Read-only: no setting is changed."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []          # (host time, sm MHz, max MHz, set of reasons)
        self.t0 = self.t1 = None
        self.thread = None
        self.proc = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.gpu)
        try:
            bus = "%04x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            bits = [(name, getattr(nv, attr)) for name, attr in self.REASONS]
            smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.stop_flag = False

            def loop():
                while not self.stop_flag:
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        r = get_reasons(h) if get_reasons else 0
                        self.samples.append((time.perf_counter(), float(sm), float(smax),
                                             {n for n, b in bits if r & b}))
                    except Exception:
                        pass
                    time.sleep(0.005)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
        except Exception:
            self.thread = None
            try:
                fd, self.path = tempfile.mkstemp(prefix=f"parallax_clocks_{self.gpu}_", suffix=".csv")
                self.f = os.fdopen(fd, "w")
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
            except Exception:
                self.proc = None

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def _from_smi(self):
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        names = [n for n, _ in self.REASONS]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                self.samples.append((None, float(parts[1]), float(parts[2]),
                                     {n for n, v in zip(names, parts[5:9]) if v.lower() == "active"}))
            except ValueError:
                continue
        try:
            os.unlink(self.path)
        except OSError:
            pass

    def stop(self):
        time.sleep(0.02)   # a sample or two after the region ends
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=2)
        elif self.proc is not None:
            self._from_smi()
        if not self.samples:
            return None
        inside = [x for x in self.samples if x[0] is not None and self.t0 is not None and self.t0 <= x[0] <= self.t1]
        source = "nvml, 5 ms" if self.thread is not None else "nvidia-smi, 100 ms"
        if not inside:   # nothing inside: the samples nearest to the region
            mid = None if self.t0 is None else (self.t0 + (self.t1 or self.t0)) / 2
            key = (lambda x: abs(x[0] - mid)) if mid is not None and self.samples[0][0] is not None else None
            inside = sorted(self.samples, key=key)[:3] if key else self.samples
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": inside[0][2],
                "reasons": sorted(set().union(*(x[3] for x in inside))), "samples": len(inside),
                "source": source}


# --------------------------------------------------------------------------- #
# our arm
# --------------------------------------------------------------------------- #
def run_profile_case(args):
    """Small single-kernel loops for ncu captures (inputs still larger than L2, a few GB at most).

    profile_fwd    : parallax_fwd, B=2 H=16 T=8192 d=128 causal (plus its rho input)
    profile_fwd_b8 : parallax_fwd, B=8 H=16 T=4096 d=128 causal (the prefill of the default step)
    profile_fwd_long : parallax_fwd, B=1 H=16 T=32768 d=128 causal (the long prefill)
    profile_decode : parallax_decode, B=16 H=16 d=128, 8192-token cache
    profile_decode_b64 : parallax_decode, B=64 H=16 d=128, 4096-token cache (the default step's decode)
    profile_rho    : parallax_rho_proj, x [2, 8192, 2048] @ W_R [2048, 2048]
    profile_paged  : parallax_decode_paged, B=64 Hq=32 Hkv=8, 64-token pages, ctx 4096 (1.07 GB)
    profile_bwd    : parallax_bwd, B=2 H=16 T=4096 d=128 causal (after one parallax_fwd_train)
    """
    import torch

    import softmax_learned_covariance_b200 as plx
    from softmax_learned_covariance_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.workload in ("profile_fwd", "profile_fwd_b8", "profile_fwd_long"):
        B, T = {"profile_fwd": (2, 8192), "profile_fwd_b8": (8, 4096), "profile_fwd_long": (1, 32768)}[args.workload]
        q, k, v, r = (t.torch().to(dev) for t in inputs.fwd_bf16_inputs(B, 16, T, 128, seed=5 if B == 1 else 3))
        y = torch.empty(q.shape, dtype=torch.float32, device=dev)
        call = lambda: plx.parallax_fwd(q, k, v, r, y=y, want_lse=False)
        work, unit = prefill_flops(B, 16, T, 128), "TFLOP/s"
    elif args.workload in ("profile_decode", "profile_decode_b64"):
        B, ctx = (16, 8192) if args.workload == "profile_decode" else (64, 4096)
        q, r, kc, vc, sl = inputs.decode_inputs(B, 16, ctx, 128, seed=2)
        q, r, kc, vc = (t.torch().to(dev) for t in (q, r, kc, vc))
        dsl = torch.from_numpy(sl).to(dev)
        y = torch.empty((B, 16, 128), dtype=torch.float32, device=dev)
        call = lambda: plx.parallax_decode(q, r, kc, vc, dsl, y=y, want_lse=False)
        work, unit = decode_bytes(B, 16, 128, sl), "TB/s"
    elif args.workload == "profile_paged":
        c = PAGED_CFG
        mp = c["ctx"] // c["page_size"]
        g = torch.Generator(device=dev)
        g.manual_seed(11)

        def randn_bf16(shape, scale=1.0):
            return (torch.randn(shape, generator=g, device=dev, dtype=torch.float32) * scale).to(torch.bfloat16)

        q, r = randn_bf16((c["B"], c["Hq"], c["d"])), randn_bf16((c["B"], c["Hq"], c["d"]), 0.05)
        kp = randn_bf16((c["B"] * mp, c["Hkv"], c["page_size"], c["d"]))
        vp = randn_bf16((c["B"] * mp, c["Hkv"], c["page_size"], c["d"]))
        tb = torch.randperm(c["B"] * mp, generator=g, device=dev).to(torch.int32).view(c["B"], mp)
        dsl = torch.full((c["B"],), c["ctx"], dtype=torch.int32, device=dev)
        y = torch.empty((c["B"], c["Hq"], c["d"]), dtype=torch.float32, device=dev)
        call = lambda: plx.parallax_decode_paged(q, r, kp, vp, tb, dsl, y=y, want_lse=False)
        work = c["B"] * c["Hkv"] * c["ctx"] * c["d"] * 4 + c["B"] * c["Hq"] * c["d"] * 8
        unit = "TB/s"
    elif args.workload == "profile_bwd":
        g = torch.Generator(device=dev)
        g.manual_seed(1)
        mk = lambda s=1.0: (torch.randn((2, 16, 4096, 128), generator=g, device=dev) * s).to(torch.bfloat16)
        q, k, v, r, dy = mk(), mk(), mk(), mk(0.905), mk()
        y, lse, o, abar = plx.parallax_fwd_train(q, k, v, r)
        call = lambda: plx.parallax_bwd(q, k, v, r, y, o, abar, lse, dy)
        work, unit = 16 * 128 * prefill_pairs(2, 16, 4096), "TFLOP/s"
    else:
        x, w = (t.torch().to(dev) for t in inputs.rho_proj_inputs(2, 8192, 2048, 16, 128, seed=3))
        r = torch.empty((2, 16, 8192, 128), dtype=torch.bfloat16, device=dev)
        call = lambda: plx.parallax_rho_proj(x, w, 16, 128, rho=r)
        work, unit = rho_proj_flops(2, 8192, 2048, 16, 128), "TFLOP/s"
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        call()
    b.record()
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    ms = a.elapsed_time(b) / args.steps
    return {"workload": args.workload, "ms": ms, "value": work / (ms * 1e-3) / 1e12, "unit": unit}


def time_decode_cell(plx, torch, dev, b, ctx, idx, steps, warmup, flush, peak):
    """One decode sweep cell: H=16, d=128, batch b, context ctx, ragged lengths in
    [ctx/2, ctx] (seeded by the cell index), inputs drawn on the device.  Cells
    whose cache could stay in L2 are timed call by call with a 256 MB write
    between calls; the others stream past L2 anyway."""
    from softmax_learned_covariance_b200 import inputs

    sl = inputs.ragged_seqlens(b, ctx, 4 + idx)
    q, r, kc, vc, dsl = inputs.decode_inputs_device(b, 16, ctx, 128, sl, seed=4 + idx, device=dev)
    y = torch.empty((b, 16, 128), dtype=torch.float32, device=dev)
    for _ in range(warmup):
        plx.parallax_decode(q, r, kc, vc, dsl, y=y, want_lse=False)
    torch.cuda.synchronize()
    nbytes = 2 * b * 16 * ctx * 128 * 2
    small = nbytes < (256 << 20)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps if small else 1)]
    if small:
        for a, e in ev:
            flush.fill_(1)
            a.record()
            plx.parallax_decode(q, r, kc, vc, dsl, y=y, want_lse=False)
            e.record()
    else:
        ev[0][0].record()
        for _ in range(steps):
            plx.parallax_decode(q, r, kc, vc, dsl, y=y, want_lse=False)
        ev[0][1].record()
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    ms = sum(a.elapsed_time(e) for a, e in ev) / steps
    nb = decode_bytes(b, 16, 128, sl)
    gbs = nb / (ms * 1e-3) / 1e9
    del q, r, kc, vc, dsl, y
    torch.cuda.empty_cache()
    return {"B": b, "ctx": ctx, "ms": round(ms, 4), "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4),
            "bytes": nb, "l2_flushed": small, "long_context": bool(ctx >= 8192 and b * 16 >= 128)}


def run_sweep(args):
    """Decode sweep: heads 16, d 128, batch x context grid with ragged lengths in
    [ctx/2, ctx]; cells whose cache exceeds 120 GB are skipped."""
    import torch

    import softmax_learned_covariance_b200 as plx
    from softmax_learned_covariance_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    cells = []
    for idx, b, ctx, nbytes, skipped in inputs.sweep_cells():
        if skipped:
            cells.append({"B": b, "ctx": ctx, "skipped": "cache %.0f GB > 120 GB" % (nbytes / 1e9)})
            continue
        cells.append(time_decode_cell(plx, torch, dev, b, ctx, idx, args.steps, args.warmup, flush,
                                      peaks["hbm_gbs"]))
    longc = [c["frac"] for c in cells if c.get("long_context")]
    return {"workload": "decode sweep H=16 d=128, ragged lengths in [ctx/2, ctx]", "unit": "GB/s",
            "steps": args.steps, "warmup": args.warmup,
            "peak": peaks["hbm_gbs"], "peak_note": "measured HBM copy bandwidth" if peaks["source"] == "measured"
            else "fallback", "long_context_min_frac": min(longc) if longc else None, "cells": cells}


# Long-context cells of the decode sweep measured in the default line (ctx >= 8192
# with B*H >= 128, where the sweep's >= 70 % of HBM gate applies); the larger
# ones (up to 69 GB of cache) are left to --workload sweep.
DECODE_LONG_CELLS = ((8, 8192), (8, 32768), (64, 8192), (256, 8192))


def measure_decode_long(args, peaks):
    import torch

    import softmax_learned_covariance_b200 as plx
    from softmax_learned_covariance_b200 import inputs

    dev = torch.cuda.current_device()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    index = {(b, c): i for i, b, c, _, _ in inputs.sweep_cells()}
    cells = [time_decode_cell(plx, torch, dev, b, c, index[(b, c)], args.steps, args.warmup, flush,
                              peaks["hbm_gbs"]) for b, c in DECODE_LONG_CELLS]
    del flush
    torch.cuda.empty_cache()
    return {"workload": "decode sweep long-context cells, H=16 d=128, ragged lengths in [ctx/2, ctx]",
            "unit": "GB/s", "peak": peaks["hbm_gbs"], "gate": 0.70,
            "min_frac": min(c["frac"] for c in cells), "cells": cells}


def run_ours(args, rank, world):
    import torch

    import softmax_learned_covariance_b200 as plx
    from softmax_learned_covariance_b200 import inputs

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks = load_peaks()

    # ---------------- inputs (seeded, resident in HBM) ----------------
    dc = DECODE_CFG
    q, rho, kc, vc, sl = inputs.decode_inputs(dc["B"], dc["H"], dc["Tcap"], dc["d"], seed=2)
    dq, drho, dk, dv = (t.torch().to(dev) for t in (q, rho, kc, vc))
    dsl = torch.from_numpy(sl).to(dev)
    yd = torch.empty((dc["B"], dc["H"], dc["d"]), dtype=torch.float32, device=dev)
    d_bytes = decode_bytes(dc["B"], dc["H"], dc["d"], sl)
    host_dec = [t.torch().pin_memory() for t in (q, rho, kc, vc)] + [torch.from_numpy(sl).pin_memory()]
    del q, rho, kc, vc

    pc = PREFILL_CFG if args.workload != "prefill_long" else LONG_CFG
    x, w = inputs.rho_proj_inputs(pc["B"], pc["T"], pc["d_model"], pc["H"], pc["d"], seed=3)
    pq, pk, pv, _ = inputs.fwd_bf16_inputs(pc["B"], pc["H"], pc["T"], pc["d"], seed=3)
    dx, dw, dpq, dpk, dpv = (t.torch().to(dev) for t in (x, w, pq, pk, pv))
    drho_p = torch.empty((pc["B"], pc["H"], pc["T"], pc["d"]), dtype=torch.bfloat16, device=dev)
    yp = torch.empty((pc["B"], pc["H"], pc["T"], pc["d"]), dtype=torch.float32, device=dev)
    lp = torch.empty((pc["B"], pc["H"], pc["T"]), dtype=torch.float32, device=dev)
    host_pre = [t.torch().pin_memory() for t in (x, w, pq, pk, pv)]
    del x, w, pq, pk, pv
    p_flops = prefill_flops(pc["B"], pc["H"], pc["T"], pc["d"])
    r_flops = rho_proj_flops(pc["B"], pc["T"], pc["d_model"], pc["H"], pc["d"])

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        plx.parallax_decode(dq, drho, dk, dv, dsl, y=yd, want_lse=False, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        plx.parallax_rho_proj(dx, dw, pc["H"], pc["d"], rho=drho_p, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        plx.parallax_fwd(dpq, dpk, dpv, drho_p, y=yp, lse=lp, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    assert plx.parallax_last_device_error() == 0
    nsplit_units = plx.parallax_decode_workspace_bytes(dc["B"], dc["H"], dc["Tcap"], dc["d"])
    # decode split (+ combine), rho_proj, and fwd's two kernels (V to block-scaled fp16, then k_fwd)
    launches_per_step = (2 if nsplit_units > 0 else 1) + 1 + 2

    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    clocks.mark_start()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    barrier()
    clocks.mark_end()
    clk = clocks.stop()
    assert plx.parallax_last_device_error() == 0
    total_ms = start.elapsed_time(end)
    dec_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    rp_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    fwd_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps

    total_ms, dec_ms, rp_ms, fwd_ms = max_over_ranks([total_ms, dec_ms, rp_ms, fwd_ms], world, dev)

    # ---------------- end to end through the public API, host buffers ----------------
    e2e = e2e_pre = None
    if not args.no_e2e:
        ksteps = max(1, min(args.steps, 3))
        h2d_d = sum(t.numel() * t.element_size() for t in host_dec)
        d2h_d = yd.numel() * 4
        yhost = torch.empty(yd.shape, dtype=torch.float32).pin_memory()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        t0.record(stream)
        for _ in range(ksteps):
            for dst, src in zip((dq, drho, dk, dv, dsl), host_dec):
                dst.copy_(src, non_blocking=True)
            plx.parallax_decode(dq, drho, dk, dv, dsl, y=yd, want_lse=False, stream=stream)
            yhost.copy_(yd, non_blocking=True)
        t1.record(stream)
        barrier()
        e_ms = max_over_ranks([t0.elapsed_time(t1)], world, dev)[0]
        e2e = {"value": whole_job_rate(d_bytes, e_ms / ksteps, world) / 1e12, "unit": "TB/s",
               "h2d_bytes_per_step": h2d_d, "d2h_bytes_per_step": d2h_d, "steps": ksteps}
        h2d_p = sum(t.numel() * t.element_size() for t in host_pre)
        yph = torch.empty(yp.shape, dtype=torch.float32).pin_memory()
        barrier()
        t0.record(stream)
        for _ in range(ksteps):
            for dst, src in zip((dx, dw, dpq, dpk, dpv), host_pre):
                dst.copy_(src, non_blocking=True)
            plx.parallax_rho_proj(dx, dw, pc["H"], pc["d"], rho=drho_p, stream=stream)
            plx.parallax_fwd(dpq, dpk, dpv, drho_p, y=yp, lse=lp, stream=stream)
            yph.copy_(yp, non_blocking=True)
        t1.record(stream)
        barrier()
        e_ms = max_over_ranks([t0.elapsed_time(t1)], world, dev)[0]
        e2e_pre = {"value": whole_job_rate(p_flops + r_flops, e_ms / ksteps, world) / 1e12, "unit": "TFLOP/s",
                   "h2d_bytes_per_step": h2d_p, "d2h_bytes_per_step": yp.numel() * 4, "steps": ksteps}

    extras = measure_extras(args, stream, barrier, world, peaks, pc, dpq, dpk, dpv, yp, lp, fwd_ms, dx, dw,
                            rp_ms + fwd_ms)
    decode_long = None if args.no_decode_long else measure_decode_long(args, peaks)

    dec_tbs = whole_job_rate(d_bytes, dec_ms, world) / 1e12
    fwd_tfs = whole_job_rate(p_flops, fwd_ms, world) / 1e12
    pre_tfs = whole_job_rate(p_flops + r_flops, fwd_ms + rp_ms, world) / 1e12
    rp_tfs = whole_job_rate(r_flops, rp_ms, world) / 1e12
    hbm = peaks["hbm_gbs"]
    bf16 = peaks["bf16_tflops"]
    tag = "of measured" if peaks["source"] == "measured" else "of fallback"
    line = {
        "metric": METRIC,
        "value": round(dec_tbs, 4),
        "unit": "TB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q,k,v; rho ~ N(0,0.05^2) for decode; x ~ N(0,1), W_R ~ N(0,0.02^2) for prefill)",
        "config": {"workload": "decode step B=64 H=16 d=128 ctx=4096 (headline) + prefill B=%d T=%d H=16 d=128 "
                               "d_model=2048 causal" % (pc["B"], pc["T"]),
                   "decode": dict(DECODE_CFG), "prefill": dict(pc), "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (2.1 GB decode cache, 0.6 GB prefill tensors); no flush"},
        "roofline": {"bound": "hbm", "kernel": "parallax_decode (split + combine)", "achieved": round(dec_tbs * 1e3 / world, 1),
                     "peak": hbm, "unit": "GB/s", "frac": round(dec_tbs * 1e3 / world / hbm, 4),
                     "traffic": round(d_bytes * DECODE_TRAFFIC_RATIO), "traffic_unit": "bytes/launch",
                     "peak_note": f"{tag} HBM copy bandwidth",
                     "algorithmic_bytes_per_launch": d_bytes, "ms_per_launch": round(dec_ms, 5)},
        "prefill": {"value": round(pre_tfs, 2), "unit": "TFLOP/s", "ms_per_step": round(fwd_ms + rp_ms, 4),
                    "fwd": {"ms": round(fwd_ms, 4), "tflops": round(fwd_tfs / world, 2), "flops": p_flops,
                            "roofline": {"bound": "tensor", "achieved": round(fwd_tfs / world, 2), "peak": bf16,
                                         "unit": "TFLOP/s", "frac": round(fwd_tfs / world / bf16, 4),
                                         "peak_note": f"{tag} dense bf16 (burst)",
                                         "traffic": PREFILL_TRAFFIC.get((pc["B"], pc["T"])),
                                         "traffic_unit": "bytes/launch (k_fwd)",
                                         "algorithmic_bytes_per_launch": pc["B"] * pc["H"] * pc["T"] * pc["d"] * (4 * 2 + 4)}},
                    "rho_proj": {"ms": round(rp_ms, 4), "tflops": round(rp_tfs / world, 2), "flops": r_flops,
                                 "frac": round(rp_tfs / world / bf16, 4)},
                    "e2e": e2e_pre},
        "e2e": e2e,
        "decode_paged": extras["decode_paged"],
        "softmax_only_fwd": extras["softmax_only_fwd"],
        "fwd_fused": extras["fwd_fused"],
        "bwd": extras["bwd"],
        "softmax_decode": dict(extras["softmax_decode"],
                               parallax_over_io_matched=round(dec_ms / extras["softmax_decode"]["d"]["ms"], 3),
                               parallax_over_compute_matched=round(dec_ms / extras["softmax_decode"]["2d"]["ms"], 3)),
        "decode_long": decode_long,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "peaks": peaks,
    }
    return line


PAGED_CFG = dict(B=64, Hq=32, Hkv=8, page_size=64, ctx=4096, d=128)


def measure_extras(args, stream, barrier, world, peaks, pc, dpq, dpk, dpv, yp, lp, fwd_ms, dx, dw, pipe_ms):
    """Measurements beside the step (not part of it, not in its timed region):
    the paged grouped-head decode, the softmax-only instantiation of the
    prefill on the same inputs (the compute-matched reference point), and the
    prefill with the probe computed inside the kernel (parallax_fwd_fused)
    against the two-launch pipeline rho_proj + fwd."""
    import torch

    import softmax_learned_covariance_b200 as plx

    dev = dpq.device

    def timed(fn, n):
        for _ in range(args.warmup):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        barrier()
        return max_over_ranks([a.elapsed_time(b) / n], world, dev)[0]

    # ---- paged KV cache, grouped query heads ----
    c = PAGED_CFG
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    mp = c["ctx"] // c["page_size"]
    npages = c["B"] * mp

    def randn_bf16(shape, scale=1.0):
        return (torch.randn(shape, generator=g, device=dev, dtype=torch.float32) * scale).to(torch.bfloat16)

    q = randn_bf16((c["B"], c["Hq"], c["d"]))
    r = randn_bf16((c["B"], c["Hq"], c["d"]), 0.05)
    kp = randn_bf16((npages, c["Hkv"], c["page_size"], c["d"]))
    vp = randn_bf16((npages, c["Hkv"], c["page_size"], c["d"]))
    table = torch.randperm(npages, generator=g, device=dev).to(torch.int32).view(c["B"], mp)
    sl = torch.full((c["B"],), c["ctx"], dtype=torch.int32, device=dev)
    y = torch.empty((c["B"], c["Hq"], c["d"]), dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        p_ms = timed(lambda: plx.parallax_decode_paged(q, r, kp, vp, table, sl, y=y, want_lse=False, stream=stream),
                     args.steps)
    assert plx.parallax_last_device_error(stream) == 0
    uniq = c["B"] * c["Hkv"] * c["ctx"] * c["d"] * 2 * 2 + c["B"] * c["Hq"] * c["d"] * (2 + 2 + 4)
    gbs = uniq / (p_ms * 1e-3) / 1e9
    paged = {"config": dict(c), "ms": round(p_ms, 4), "unit": "GB/s", "value": round(world * gbs, 1),
             "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                          "frac": round(gbs / peaks["hbm_gbs"], 4), "unit": "GB/s",
                          "bytes": "unique K/V rows + q, rho, y; the 4 query heads of a KV head re-read its rows "
                                   "through L2"}}
    del q, r, kp, vp, table, sl, y

    # ---- softmax-only forward on the prefill inputs ----
    with torch.cuda.stream(stream):
        s_ms = timed(lambda: plx.parallax_fwd(dpq, dpk, dpv, None, y=yp, lse=lp, stream=stream), args.steps)
    pairs = prefill_pairs(pc["B"], pc["H"], pc["T"])
    s_tf = 4 * pc["d"] * pairs / (s_ms * 1e-3) / 1e12
    smx = {"ms": round(s_ms, 4), "tflops": round(s_tf, 2), "flops": 4 * pc["d"] * pairs,
           "parallax_over_softmax_time": round(fwd_ms / s_ms, 3),
           "note": "rho = NULL instantiation of the same kernel (2 of the 4 GEMMs); same inputs and shape"}
    # ---- softmax attention decode, the pages' comparison baseline: at the same
    # head dim (same KV bytes: I/O-matched) and at twice it (same arithmetic per
    # cached token: compute-matched), on the decode step's shape ----
    dc = DECODE_CFG
    gsd = torch.Generator(device=dev)
    gsd.manual_seed(17)
    sd = {}
    for dd in (dc["d"], 2 * dc["d"]):
        qs = torch.randn((dc["B"], dc["H"], dd), generator=gsd, device=dev).to(torch.bfloat16)
        kcs = torch.randn((dc["B"], dc["H"], dc["Tcap"], dd), generator=gsd, device=dev).to(torch.bfloat16)
        vcs = torch.randn((dc["B"], dc["H"], dc["Tcap"], dd), generator=gsd, device=dev).to(torch.bfloat16)
        sls = torch.full((dc["B"],), dc["Tcap"], dtype=torch.int32, device=dev)
        ys = torch.empty((dc["B"], dc["H"], dd), dtype=torch.float32, device=dev)
        with torch.cuda.stream(stream):
            ms_ = timed(lambda: plx.parallax_softmax_decode(qs, kcs, vcs, sls, y=ys, want_lse=False, stream=stream),
                        args.steps)
        nb = decode_bytes(dc["B"], dc["H"], dd, np.full((dc["B"],), dc["Tcap"])) - dc["B"] * dc["H"] * dd * 2
        sd[dd] = {"ms": round(ms_, 4), "GB/s": round(nb / (ms_ * 1e-3) / 1e9, 1)}
        del qs, kcs, vcs, sls, ys
    torch.cuda.empty_cache()
    softmax_decode = {"d": sd[dc["d"]], "2d": sd[2 * dc["d"]],
                      "note": "parallax_softmax_decode on B=64 H=16 ctx 4096; ratios are the Parallax decode "
                              "call's time over these (> 1 means Parallax is slower)",
                      "parallax_over_io_matched": None, "parallax_over_compute_matched": None}

    # ---- probe rho = x W_R inside the prefill kernel ----
    with torch.cuda.stream(stream):
        f_ms = timed(lambda: plx.parallax_fwd_fused(dpq, dpk, dpv, dx, dw, y=yp, lse=lp, stream=stream), args.steps)
    f_flops = prefill_flops(pc["B"], pc["H"], pc["T"], pc["d"]) + rho_proj_flops(pc["B"], pc["T"], pc["d_model"],
                                                                                 pc["H"], pc["d"])
    fused = {"ms": round(f_ms, 4), "tflops": round(f_flops / (f_ms * 1e-3) / 1e12, 2), "flops": f_flops,
             "two_launch_ms": round(pipe_ms, 4), "speedup_vs_two_launch": round(pipe_ms / f_ms, 3),
             "note": "parallax_fwd_fused (rho computed per query tile in the kernel, never in HBM) vs "
                     "parallax_rho_proj + parallax_fwd on the same inputs; flops count both GEMM families"}
    # ---- training: forward keeping o and abar, then the gradients ----
    g = torch.Generator(device=dev)
    g.manual_seed(13)
    dpr = (torch.randn(dpq.shape, generator=g, device=dev) * 0.905).to(torch.bfloat16)
    ddy = torch.randn(dpq.shape, generator=g, device=dev).to(torch.bfloat16)
    with torch.cuda.stream(stream):
        fwd_state = plx.parallax_fwd_train(dpq, dpk, dpv, dpr, stream=stream)
        tr_ms = timed(lambda: plx.parallax_fwd_train(dpq, dpk, dpv, dpr, stream=stream), max(2, args.steps // 4))
        grads = [torch.empty_like(fwd_state[0]) for _ in range(4)]
        b_ms = timed(lambda: plx.parallax_bwd(dpq, dpk, dpv, dpr, *fwd_state[:1], fwd_state[2], fwd_state[3],
                                              fwd_state[1], ddy, stream=stream, out=grads), max(2, args.steps // 4))
    assert plx.parallax_last_device_error(stream) == 0
    b_flops = 16 * pc["d"] * pairs   # dV, dK (two), dQ, dR and the three recomputed score products: 8 GEMMs
    bwd = {"ms": round(b_ms, 4), "tflops": round(b_flops / (b_ms * 1e-3) / 1e12, 2), "flops": b_flops,
           "roofline": {"bound": "tensor", "achieved": round(b_flops / (b_ms * 1e-3) / 1e12, 2),
                        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": round(b_flops / (b_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)},
           "fwd_train_ms": round(tr_ms, 4),
           "note": "parallax_bwd (tcgen05 dq/drho and dk/dv kernels; S, A, G recomputed in both, 11 products "
                   "executed per pair) after parallax_fwd_train on the prefill shape; flops count 8 GEMMs of 2d per pair"}
    del dpr, ddy, fwd_state, grads
    return {"decode_paged": paged, "softmax_only_fwd": smx, "fwd_fused": fused, "bwd": bwd,
            "softmax_decode": softmax_decode}


# --------------------------------------------------------------------------- #
# reference arm: the fp64 oracle on host cores, bounded samples of the same workloads
# --------------------------------------------------------------------------- #
def _oracle_decode_sample():
    """The first 4 sequences of the decode step (64 of its 1024 heads), same recipe and seed, as fp64."""
    from softmax_learned_covariance_b200 import inputs

    dc = DECODE_CFG
    nbs = 4
    q, rho, kc, vc, sl = inputs.decode_inputs(nbs, dc["H"], dc["Tcap"], dc["d"], seed=2)
    return (q.f64, rho.f64, kc.f64, vc.f64, sl), nbs


def _oracle_decode_1thread(oracle, args_f64):
    """The oracle decode on one thread, on the first sequence (16 heads): TB/s."""
    qf, rf, kf, vf, sl = args_f64
    cores = oracle.max_threads()
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        oracle.decode(qf[:1], rf[:1], kf[:1], vf[:1], sl[:1])
        dt1 = time.perf_counter() - t0
    finally:
        oracle.set_threads(cores)
    return decode_bytes(1, DECODE_CFG["H"], DECODE_CFG["d"], sl[:1]) / dt1 / 1e12


def _oracle_prefill_sample(oracle):
    """The oracle prefill on every 8th causal row of one T=4096 head: TFLOP/s and a description."""
    from softmax_learned_covariance_b200 import inputs

    pc = PREFILL_CFG
    pq, pk, pv, pr = inputs.fwd_bf16_inputs(1, 1, pc["T"], pc["d"], seed=3)
    rows = np.arange(0, pc["T"], 8, dtype=np.int64)
    t0 = time.perf_counter()
    oracle.fwd_rows(pq.f64, pk.f64, pv.f64, pr.f64, rows)
    dt = time.perf_counter() - t0
    pairs = int(np.sum(rows + 1))
    pre_tfs = 8 * pc["d"] * pairs / dt / 1e12
    return pre_tfs, f"{rows.size} causal rows (every 8th) of one T={pc['T']} head, {pairs} pairs, {pairs / dt:.3e} pairs/s"


def oracle_sample(budget_s=12.0):
    """The oracle on a bounded sample of the step, timed for about budget_s / 2 on all host cores."""
    import oracle

    cores = oracle.max_threads()
    args_f64, nbs = _oracle_decode_sample()
    dc = DECODE_CFG
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.decode(*args_f64)
        reps += 1
        if time.perf_counter() - t0 > budget_s / 2:
            break
    dt = (time.perf_counter() - t0) / reps
    sl = args_f64[4]
    dec_tbs = decode_bytes(nbs, dc["H"], dc["d"], sl) / dt / 1e12
    dec_sample = f"{nbs * dc['H']} of the {dc['B'] * dc['H']} heads x {dc['Tcap']} tokens, x{reps}"
    dec_tbs_1t = _oracle_decode_1thread(oracle, args_f64)
    pre_tfs, pre_sample = _oracle_prefill_sample(oracle)
    return cores, dec_tbs, dec_sample, pre_tfs, pre_sample, dec_tbs_1t


def run_reference(args, rank, world):
    """The oracle as it stands, on the host cores: W untimed and K timed steps, each one oracle decode
    of the same bounded sample of the decode step (64 of its 1024 heads, the full 4096-token cache);
    the value is that sample's algorithmic bytes over the mean step time.  The 1-thread figure and the
    prefill sample are measured once, after the timed steps."""
    if rank != 0:
        return None
    import oracle

    cores = oracle.max_threads()
    args_f64, nbs = _oracle_decode_sample()
    dc = DECODE_CFG
    for _ in range(args.warmup):
        oracle.decode(*args_f64)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.decode(*args_f64)
    dt = (time.perf_counter() - t0) / args.steps
    dec_tbs = decode_bytes(nbs, dc["H"], dc["d"], args_f64[4]) / dt / 1e12
    dec_sample = f"{nbs * dc['H']} of the {dc['B'] * dc['H']} heads x {dc['Tcap']} tokens per step"
    dec_1t = _oracle_decode_1thread(oracle, args_f64)
    pre_tfs, pre_sample = _oracle_prefill_sample(oracle)
    line = {
        "metric": METRIC, "value": dec_tbs, "unit": "TB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": "decode step B=64 H=16 d=128 ctx=4096 (headline) + prefill B=8 T=4096 H=16 d=128",
                   "decode": dict(DECODE_CFG), "prefill": dict(PREFILL_CFG)},
        "cpu_baseline": {"value": dec_tbs, "unit": "TB/s", "cores": cores, "kind": "oracle", "sample": dec_sample,
                         "value_1_thread": dec_1t},
        "prefill": {"value": pre_tfs, "unit": "TFLOP/s", "sample": pre_sample},
        "e2e": {"value": dec_tbs, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["default", "prefill_long", "sweep", "profile_fwd", "profile_decode",
                                           "profile_rho", "profile_paged", "profile_fwd_long", "profile_bwd",
                                           "profile_fwd_b8", "profile_decode_b64"],
                    default="default")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode-long", action="store_true", help="skip the long-context decode cells")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank, world, local_rank = rank_env()
    if world > 1 and args.impl == "ours":
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    if args.workload.startswith("profile_"):
        print(json.dumps(run_profile_case(args)), flush=True)
        return
    if args.workload == "sweep":
        print(json.dumps(run_sweep(args)), flush=True)
        return
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_ours(args, rank, world)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            cores, dec_tbs, dec_sample, _, _, dec_1t = oracle_sample(budget_s=10.0)
            line["cpu_baseline"] = {"value": dec_tbs, "unit": "TB/s", "cores": cores, "kind": "oracle",
                                    "sample": dec_sample, "value_1_thread": dec_1t}
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1 and args.impl == "ours":
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
