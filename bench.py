#!/usr/bin/env python3
"""Benchmark of the host-streamed NF4 LoRA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qwen2.5-72b-stack|qwen2.5-72b-layer|qwen2.5-7b-layer|
                                llama-3.1-8b-stack|qwen2.5-32b-stack]
                    [--mode streamed|resident] [--block-size B] [--seq T]

One step = forward + backward of every LoRA-targeted projection (q, k, v,
o, gate, up, down) of the workload's layers at T tokens, with the frozen NF4
base streamed from pinned host RAM into the 2-slot VRAM ring one block
ahead (mode "streamed") or read from VRAM (mode "resident").  The default
workload is the Qwen2.5-72B-shaped stack: 80 layers, 512 tokens, blocks of
4 layers, its 39.5 GB NF4 base pinned in host RAM and streamed every step
(71.1 GB over PCIe per steady step: forward, then backward in reverse, the
blocks still resident at each turn-around reused).  qwen2.5-7b-layer is a
single layer re-streamed every step.

Prints one JSON line (rank 0).  `value` is device-timed whole-job tokens/s
with inputs resident in HBM; `e2e` is the same metric through the public
API with the step's inputs copied from pinned host memory and its adapter
gradients read back, every step.  `--impl reference` times the CPU oracle
(the slow, obviously-correct implementation the tests check against) on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "tokens/s fwd+bwd NF4-streamed LoRA layers; % of PCIe/tensor roofline"
PCIE_GEN5_X16_GBPS = 63.0  # per direction, theoretical (32 GT/s x 16 lanes, 128b/130b)

WORKLOADS = {
    # name: (family, layers, default block size, default mode)
    "qwen2.5-7b-layer": ("qwen2.5-7b", 1, 1, "streamed"),
    # one layer of the 72B stack: the same grouped launches, small enough to profile
    "qwen2.5-72b-layer": ("qwen2.5-72b", 1, 1, "streamed"),
    "llama-3.1-8b-stack": ("llama-3.1-8b", 32, 4, "streamed"),
    "qwen2.5-32b-stack": ("qwen2.5-32b", 64, 4, "streamed"),
    "qwen2.5-72b-stack": ("qwen2.5-72b", 80, 4, "streamed"),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="qwen2.5-72b-stack")
    ap.add_argument("--mode", choices=["streamed", "resident"], default=None)
    ap.add_argument("--block-size", type=int, default=None)
    ap.add_argument("--slots", type=int, default=2, help="ring slots (2 = prefetch one ahead)")
    ap.add_argument("--seq", type=int, default=512)
    ap.add_argument("--grouping", choices=["decoder", "layer", "none"], default="layer",
                    help="how a layer's projections are batched into grouped launches")
    ap.add_argument("--base", choices=["nf4", "bf16"], default="nf4",
                    help="frozen base format: NF4 (default) or dense bf16 (bf16_bitwise)")
    ap.add_argument("--model", choices=["projections", "decoder"], default="projections",
                    help="projections: the 7 LoRA linears per layer on seeded inputs; decoder: "
                         "full decoder layers (norms, attention, SwiGLU, residuals) with "
                         "per-block rematerialization")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="LoRA dropout on the adapter branch (the configs use 0)")
    ap.add_argument("--no-shard-h2d", dest="shard_h2d", action="store_false",
                    help="with N > 1 GPUs every rank streams whole blocks (default: each "
                         "streams 1/N and the ranks all-gather)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=4.0,
                    help="target seconds per step of the oracle sample")
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    fam, L, bs, mode = WORKLOADS[a.workload]
    a.family, a.layers = fam, L
    a.block_size = a.block_size or bs
    a.mode = a.mode or mode
    return a


# ---------------------------------------------------------------------- dist

def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch
        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and throttle reasons sampled every 10 ms during the timed
    region (NVML; nvidia-smi as a fallback)."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None
        self._nv = self._h = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.cuda_index)
        bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def _sample(self):
        nv, h = self._nv, self._h
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
        mask = get_reasons(h)
        for bit, name in self.REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _run_nvml(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            self._stop.wait(0.01)

    def sample_while(self, busy, limit_s: float = 600.0):
        """Also sample from the calling thread while busy() holds (the GPU is
        still working through the timed region's queued steps), so that a
        short region still gets samples.  NVML only; never raises."""
        if self._nv is None:
            return
        t0 = time.monotonic()
        try:
            while busy() and time.monotonic() - t0 < limit_s:
                self._sample()
                time.sleep(0.002)
        except Exception:
            return

    def __enter__(self):
        try:
            self._nv, self._h = self._nvml_handle()
            self.max_mhz = self._nv.nvmlDeviceGetMaxClockInfo(self._h, self._nv.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run_nvml, daemon=True)
            self._thread.start()
        except Exception:
            self._nv = self._h = None
            self._start_smi()
        return self

    def _start_smi(self):
        q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self._proc = None
            return

        def read():
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for line in self._proc.stdout:
                f = [x.strip() for x in line.split(",")]
                try:
                    self.samples.append(float(f[0]))
                    self.max_mhz = float(f[1])
                except (ValueError, IndexError):
                    continue
                for n, v in zip(names, f[2:6]):
                    if v.lower() == "active":
                        self.reasons.add(n)
        self._thread = threading.Thread(target=read, daemon=True)
        self._thread.start()

    def __exit__(self, *exc):
        self._stop.set()
        if self._proc:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------- peaks

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs"), d.get("bf16_tflops"), d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def gemm_source_digest():
    h = hashlib.sha256()
    for f in ("lora_gemm.cu", "ptx.cuh", "nf4_device.cuh"):
        h.update(open(os.path.join(ROOT, "host_streamed_nf4_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from a committed ncu summary under
    profiles/ (a line `traffic_record: {json}`), if it was taken on the
    current kernel source; else None."""
    for p in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(p, errors="replace"):
            if not line.startswith("traffic_record:"):
                continue
            try:
                d = json.loads(line.split(":", 1)[1])
            except ValueError:
                continue
            if d.get("kernel") == kernel and d.get("workload") == workload and \
                    d.get("source_digest") == gemm_source_digest():
                return d.get("dram_bytes_per_launch")
    return None


# ---------------------------------------------------------------------- our arm

def run_ours(args, ws, rank, local):
    import numpy as np
    import torch

    from host_streamed_nf4_b200 import dist as hdist
    from host_streamed_nf4_b200 import hsnf4, synth
    from host_streamed_nf4_b200.stack import LayerStack

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fam = synth.FAMILIES[args.family]
    streamed = args.mode == "streamed"
    single = args.layers == 1
    # A one-layer workload re-streams its layer every step (the layer's bytes
    # cross PCIe once per step, the next copy overlapping this step's
    # compute); a stack reuses the blocks still resident at each turn-around.
    # data-parallel ranks share the frozen base and the adapters (seed 42)
    # and see their own tokens (data_seed); with N > 1 the ranks share the
    # stream too: each copies 1/N of every block and an NCCL all-gather on
    # the copy stream rebuilds the block in every ring
    shard = (rank, ws, hdist.ring_gather) if (streamed and ws > 1 and args.shard_h2d) else None
    from host_streamed_nf4_b200.decoder import DecoderStack
    cls = DecoderStack if args.model == "decoder" else LayerStack
    if args.model == "decoder":
        args.grouping = "decoder"
    stack = cls(fam, args.layers, args.seq, block_size=args.block_size, streamed=streamed,
                       reuse_resident=not single, seed=42, data_seed=42 + rank, device=dev,
                       shard=shard,
                       grouping=args.grouping, n_slots=args.slots, base=args.base,
                       dropout=args.dropout)
    compute = stack.compute

    def one_step():
        if streamed and single:
            stack.step_single_block()
        else:
            stack.step()
        # data parallel: the adapter gradients are summed over ranks each step
        hdist.allreduce_grads(stack.grad_flat)

    def drain_copies():
        # make the compute stream wait for the copy stream, so that an
        # interval closed on the compute stream includes every copy issued
        if streamed:
            ev = torch.cuda.Event()
            ev.record(stack.copy_stream)
            compute.wait_event(ev)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize(dev)
    assert hsnf4.device_status() == 0, "a kernel wait gave up during warm-up"
    st0 = stack.streamer.stats() if streamed else None

    # ------------------------------------------------ device-timed region
    # The library times each fused-GEMM launch (the dominant kernel) with CUDA
    # events on the launch stream throughout the region (hsnf4_profile): its
    # roofline below comes from the same steps, clocks and power state as
    # `value`.  The other kernels are timed in a short pass after it, so that
    # their events do not delay launches inside the region.
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier(ws)
        torch.cuda.synchronize(dev)
        launches0 = hsnf4.kernel_launches()
        hsnf4.profile(True, kinds=("lora_gemm_fwd", "lora_gemm_dx"))
        e0.record(compute)
        for _ in range(K):
            one_step()
        drain_copies()
        e1.record(compute)
        launches = hsnf4.kernel_launches() - launches0
        clocks.sample_while(lambda: not e1.query())  # the GPU is still inside the region
        torch.cuda.synchronize(dev)
        barrier(ws)
    ms_total = hdist.max_over_ranks(e0.elapsed_time(e1))
    ms_step = ms_total / K
    tokens_per_step = stack.tokens_per_step()
    value = hdist.job_throughput(tokens_per_step, K, ms_total, ws)
    h2d_step = 0
    if streamed:
        st1 = stack.streamer.stats()
        h2d_step = (st1["h2d_bytes"] - st0["h2d_bytes"]) / K
    assert hsnf4.device_status() == 0, "a kernel wait gave up in the timed region"

    # ------------------------------------------------ per-kernel timing (roofline)
    kt = hsnf4.profile_read()  # every fused-GEMM launch of the timed region
    hsnf4.profile(True, kinds=("lora_project", "lora_grad"))
    for _ in range(max(2, min(K, 5))):
        one_step()
    torch.cuda.synchronize(dev)
    kt.update(hsnf4.profile_read())
    hsnf4.profile(False)
    _, bf16_burst, bf16_sus, peak_src = measured_peaks()
    clock_summary = clocks.summary()
    # the burst cuBLAS figure, unless the power cap held the clocks down
    # during the timed region (then the sustained, power-capped figure)
    capped = "sw_power_cap" in clock_summary["reasons"]
    peak = bf16_sus if capped else bf16_burst
    gemms = {k: v for k, v in kt.items() if k.startswith("lora_gemm")}
    dom = max(gemms, key=lambda k: gemms[k]["total_ms"])
    d = gemms[dom]
    achieved_tflops = d["work"] / (d["total_ms"] / 1e3) / 1e12
    flops_per_launch = d["work"] / d["launches"]
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved_tflops, 1),
                "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved_tflops / peak, 4),
                "peak_source": (f"{peak_src} bf16_tflops_sustained (sw_power_cap seen in the "
                                f"timed region)" if capped else
                                f"{peak_src} bf16_tflops (burst; no power cap seen in the "
                                f"timed region)"),
                "frac_vs_sustained": round(achieved_tflops / bf16_sus, 4),
                "sustained_peak": bf16_sus,
                "traffic": recorded_traffic(dom, args.workload),
                "flops_per_launch": flops_per_launch,
                "avg_launch_us": round(d["total_ms"] / d["launches"] * 1e3, 2),
                "all_kernels": {k: {"launches": v["launches"],
                                    "avg_us": round(v["total_ms"] / v["launches"] * 1e3, 2),
                                    "achieved": round(v["work"] / (v["total_ms"] / 1e3) / 1e12, 1)}
                                for k, v in gemms.items()}}

    # the rank-r kernels (HBM-bound: each reads its activation operand once)
    hbm_peak, _, _, hbm_src = measured_peaks()
    rank_r = {k: {"launches": v["launches"],
                  "avg_us": round(v["total_ms"] / v["launches"] * 1e3, 2),
                  "bytes_per_launch": int(v["work"] / v["launches"]),
                  "achieved_GBps": round(v["work"] / (v["total_ms"] / 1e3) / 1e9, 1),
                  "frac": round(v["work"] / (v["total_ms"] / 1e3) / 1e9 / hbm_peak, 4),
                  "peak_GBps": hbm_peak, "peak_source": f"{hbm_src} hbm_gbs"}
              for k, v in kt.items() if k in ("lora_project", "lora_grad")}

    # standalone NF4 dequant on the layer's largest weight (HBM-bound; the
    # output, 2 B per element, is far larger than L2)
    dequant = dequant_roofline(stack, fam, dev) if args.base == "nf4" else None
    merge = merge_roofline(stack, dev)

    # step-level binding roofline: max(PCIe bytes / link rate, FLOPs / tensor peak)
    flops_step = sum(2.0 * args.seq * n * k * 2 for _, n, k in fam.projections()) * args.layers
    flops_step += sum(2.0 * args.seq * stack.r * (2 * k + 2 * n) + 2.0 * args.seq * stack.r * (k + n)
                      for _, n, k in fam.projections()) * args.layers
    if args.model == "decoder":
        # the backward recomputes each block's forward: the projections' forward
        # again, plus causal attention (forward, its recompute, backward ~3.5x)
        flops_step += sum(2.0 * args.seq * n * (k + stack.r) + 2.0 * args.seq * stack.r * k
                          for _, n, k in fam.projections()) * args.layers
        attn_fwd = 2.0 * args.seq * args.seq * fam.head_dim * fam.heads
        flops_step += (2 * attn_fwd + 3.5 * attn_fwd) * args.layers
    link = link_probe(stack, dev) if streamed else None
    roofline["cublas_same_shapes"] = cublas_probe(fam, args.seq, dom, dev)
    roofline["frac_vs_cublas_same_shapes"] = round(
        achieved_tflops / roofline["cublas_same_shapes"]["tflops"], 4)
    t_pcie = h2d_step / (PCIE_GEN5_X16_GBPS * 1e9)
    t_tensor = flops_step / (bf16_sus * 1e12)
    t_bound = max(t_pcie, t_tensor)
    step_roofline = {"binding": "pcie" if t_pcie >= t_tensor else "tensor",
                     "bound_ms": round(t_bound * 1e3, 4), "ms_per_step": round(ms_step, 4),
                     "frac": round(t_bound / (ms_step / 1e3), 4),
                     "h2d_bytes_per_step": int(h2d_step),
                     "h2d_GBps": round(h2d_step / (ms_step / 1e3) / 1e9, 2) if streamed else None,
                     "pcie_peak_GBps": PCIE_GEN5_X16_GBPS, "flops_per_step": flops_step}
    if link:
        step_roofline["pcie_link"] = link
        step_roofline["frac_vs_probe"] = round(
            (h2d_step / (ms_step / 1e3) / 1e9) / link["probe_GBps"], 4)

    # ------------------------------------------------ result check
    # one more step (no gradient exchange), then layers 0 and L-1 recomputed
    # from weights drawn afresh and held in VRAM: their outputs and adapter
    # gradients must equal the streamed step's bit for bit
    check = None
    if args.model == "projections":
        if streamed and single:
            stack.step_single_block()
        else:
            stack.step()
        res = stack.resident_check()
        check = {"layers": {str(k): v for k, v in res.items()}, "bitwise": all(res.values()),
                 "what": "t, dA, dB of layers 0 and L-1, Y of layer L-1, dX of layer 0, vs a "
                         "resident recomputation"}

    # ------------------------------------------------ end to end through the API
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, stack, one_step, drain_copies, ws, dev)

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded normal weights/activations; no dataset)",
        "config": {"workload": args.workload + ("-decoder" if args.model == "decoder" else ""),
                   "model": args.model, "family": args.family, "layers": args.layers,
                   "tokens": args.seq, "batch": 1, "mode": args.mode, "base": args.base,
                   "dropout": args.dropout,
                   "block_size": args.block_size, "rank": stack.r, "alpha": stack.alpha,
                   "grouping": args.grouping, "ring_slots": args.slots,
                   "projections": [p[0] for p in fam.projections()],
                   "parallelism": (f"dp{ws} (per-rank tokens, adapter-gradient all-reduce per "
                                   f"step" + (", sharded H2D + per-block all-gather)"
                                              if shard else ")") if ws > 1 else "single"),
                   "l2": "no flush: every step reads > 126 MB L2 (NF4 weights + activations)"},
        "roofline": roofline, "step_roofline": step_roofline, "rank_r": rank_r,
        "resident_check": check,
        "dequant": dequant, "merge": merge,
        "peak_vram_GB": round(torch.cuda.max_memory_allocated(dev) / 1e9, 3), "e2e": e2e,
        # page-locked host bytes of the frozen base on this rank (a sharded
        # stream pins only the rank's shards)
        "pinned_host_GB_per_rank": round(stack.pinned_bytes() / 1e9, 3),
        "gpu_launches": launches,  # counted by the library over the timed region
        "clocks": clock_summary,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args, fam)
    stack.close()
    return out


def busy_ahead(ms: float = 2.0):
    """Keep the current stream busy for about `ms` so that the host enqueues
    the next launches (and their timing events) while the GPU is still
    working: the events then bracket back-to-back kernels, not the host's
    per-call marshalling between them."""
    import torch
    torch.cuda._sleep(int(ms * 2.0e6))  # ~2 GHz SM clock: cycles per ms


def dequant_roofline(stack, fam, dev):
    """nf4_dequant of the layer's largest projection, timed with CUDA events
    (library-side, on the launch stream) against the measured HBM copy rate.
    Launches rotate over several input/output sets that together hold at
    least 4x the L2 capacity, so no launch finds its operands, or dirty
    lines of its output, still in L2."""
    import math

    import torch

    from host_streamed_nf4_b200 import hsnf4
    p = max(range(len(stack.projs)), key=lambda i: stack.projs[i][1] * stack.projs[i][2])
    _, n, k = stack.projs[p]
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    set_bytes = n * k * 2 + n * k // 2 + n * k // 16
    n_sets = max(2, math.ceil(4 * l2 / set_bytes))
    W0 = stack.device_weight(0, p)
    sets = []
    for _ in range(n_sets):
        sets.append((hsnf4.Nf4Weight(W0.codes.clone(), W0.absmax.clone(), n, k),
                     torch.empty(n, k, dtype=torch.bfloat16, device=dev)))
    del W0
    for W, out in sets:
        hsnf4.nf4_dequant(W, out)
    torch.cuda.synchronize(dev)
    reps = max(10, 2 * n_sets)
    hsnf4.profile(True)
    busy_ahead()  # the launches below queue up behind it: no host gaps inside the events
    for i in range(reps):
        W, out = sets[i % n_sets]
        hsnf4.nf4_dequant(W, out)
    torch.cuda.synchronize(dev)
    d = hsnf4.profile_read()["nf4_dequant"]
    hsnf4.profile(False)
    del sets
    hbm, _, _, src = measured_peaks()
    gbs = d["work"] / (d["total_ms"] / 1e3) / 1e9
    return {"bound": "hbm", "shape": [n, k], "achieved": round(gbs, 1), "peak": hbm,
            "unit": "GB/s", "frac": round(gbs / hbm, 4),
            "bytes_per_launch": int(d["work"] / d["launches"]),
            "avg_launch_us": round(d["total_ms"] / d["launches"] * 1e3, 2),
            "rotation": {"sets": n_sets, "bytes": n_sets * set_bytes, "l2_bytes": l2},
            "peak_source": f"{src} hbm_gbs (copy read+write)"}


def pcie_link_info(dev):
    """Current and maximum PCIe generation and width of the device (NVML)."""
    try:
        import pynvml
        import torch
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(dev)
        h = pynvml.nvmlDeviceGetHandleByPciBusId(
            f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0")
        return {"gen": pynvml.nvmlDeviceGetCurrPcieLinkGeneration(h),
                "width": pynvml.nvmlDeviceGetCurrPcieLinkWidth(h),
                "max_gen": pynvml.nvmlDeviceGetMaxPcieLinkGeneration(h),
                "max_width": pynvml.nvmlDeviceGetMaxPcieLinkWidth(h)}
    except Exception as e:  # NVML missing or not permitted: report why
        return {"error": type(e).__name__}


def link_probe(stack, dev, reps=8):
    """A plain pinned-host -> device cudaMemcpyAsync of one ring slot's bytes
    (the streamer's copy size), repeated on a side stream and timed with CUDA
    events: the practical rate of this link, beside the theoretical 63 GB/s."""
    import torch
    nbytes = min(stack.slab.numel(), stack.ring.numel() // max(1, stack.streamer.n_slots))
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    src = stack.slab[:nbytes]
    s = torch.cuda.Stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        dst.copy_(src, non_blocking=True)
        e0.record(s)
        for _ in range(reps):
            dst.copy_(src, non_blocking=True)
        e1.record(s)
    torch.cuda.synchronize(dev)
    gbs = nbytes * reps / (e0.elapsed_time(e1) / 1e3) / 1e9
    out = {"probe_GBps": round(gbs, 2), "probe_bytes": int(nbytes), "probe_copies": reps}
    out.update(pcie_link_info(dev))
    del dst
    return out


def cublas_probe(fam, T, kernel, dev, reps=10):
    """cuBLAS bf16 GEMMs of the same shapes as the dominant grouped kernel
    (torch.mm; fwd: [T,K] x [K,N] per projection, dx: [T,N] x [N,K]), timed
    with CUDA events: a same-shape library reference for the tensor peak."""
    import torch
    g = torch.Generator(device=dev).manual_seed(7)
    pairs = []
    for _, n, k in fam.projections():
        a_rows, inner, outer = (T, k, n) if kernel == "lora_gemm_fwd" else (T, n, k)
        a = torch.randn(a_rows, inner, generator=g, device=dev, dtype=torch.bfloat16)
        b = torch.randn(inner, outer, generator=g, device=dev, dtype=torch.bfloat16)
        pairs.append((a, b, 2.0 * a_rows * inner * outer))
    for a, b, _ in pairs:
        torch.mm(a, b)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        for a, b, _ in pairs:
            torch.mm(a, b)
    e1.record()
    torch.cuda.synchronize(dev)
    sec = e0.elapsed_time(e1) / 1e3
    flops = reps * sum(f for _, _, f in pairs)
    return {"tflops": round(flops / sec / 1e12, 1), "gemms_per_pass": len(pairs),
            "us_per_pass": round(sec / reps * 1e6, 2)}


def merge_roofline(stack, dev):
    """lora_merge (merge_and_unload) of the layer's largest projection, timed
    with CUDA events on the launch stream, against the measured HBM copy
    rate: algorithmic bytes are the base read plus the bf16 W' written.
    Launches rotate over base/output sets that together hold at least 4x the
    L2 capacity, so no launch finds its base, or dirty lines of its output,
    still in L2."""
    import math

    import torch

    from host_streamed_nf4_b200 import hsnf4
    p = max(range(len(stack.projs)), key=lambda i: stack.projs[i][1] * stack.projs[i][2])
    _, n, k = stack.projs[p]
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    base_bytes = n * k * 2 if stack.base == "bf16" else n * k // 2 + n * k // 16
    set_bytes = base_bytes + n * k * 2
    n_sets = max(2, math.ceil(4 * l2 / set_bytes))
    W0 = stack.device_weight(0, p)
    A, B = stack.A[0][p], stack.B[0][p]
    sets = []
    for _ in range(n_sets):
        W = (hsnf4.Bf16Weight(W0.w.clone()) if stack.base == "bf16" else
             hsnf4.Nf4Weight(W0.codes.clone(), W0.absmax.clone(), n, k))
        sets.append((W, torch.empty(n, k, dtype=torch.bfloat16, device=dev)))
    del W0
    for W, out in sets:
        hsnf4.lora_merge(W, A, B, stack.alpha, out=out)
    torch.cuda.synchronize(dev)
    reps = max(10, 2 * n_sets)
    hsnf4.profile(True)
    busy_ahead()
    for i in range(reps):
        W, out = sets[i % n_sets]
        hsnf4.lora_merge(W, A, B, stack.alpha, out=out)
    torch.cuda.synchronize(dev)
    d = hsnf4.profile_read()["lora_merge"]
    hsnf4.profile(False)
    del sets
    hbm, _, _, src = measured_peaks()
    gbs = d["work"] / (d["total_ms"] / 1e3) / 1e9
    return {"bound": "hbm", "shape": [n, k], "base": stack.base, "achieved": round(gbs, 1),
            "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
            "bytes_per_launch": int(d["work"] / d["launches"]),
            "avg_launch_us": round(d["total_ms"] / d["launches"] * 1e3, 2),
            "rotation": {"sets": n_sets, "bytes": n_sets * set_bytes, "l2_bytes": l2},
            "peak_source": f"{src} hbm_gbs (copy read+write)"}


def run_e2e(args, stack, one_step, drain_copies, ws, dev):
    """Same step through the public API with host buffers: each step copies
    its activations and upstream gradients from pinned host memory and reads
    the layer stack's adapter gradients back (device-timed).

    The next step's inputs are copied on their own stream into one of two
    device staging sets while the current step computes (its weights stream
    on the copy stream meanwhile), and moved into the stack's input tensors
    with one on-device copy at the start of the step, so the host link is
    not left idle while a step's kernels run."""
    import torch
    dev_in = stack.step_inputs()  # the tensors a step reads from the host
    host_in = [torch.empty_like(v, device="cpu").pin_memory() for v in dev_in]
    for h, v in zip(host_in, dev_in):
        h.copy_(v)
    stage = [[torch.empty_like(v) for v in dev_in] for _ in range(2)]
    grads = [stack.grad_flat]  # every dA/dB of the stack, summed over ranks
    host_grads = [torch.empty_like(g, device="cpu").pin_memory() for g in grads]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_grads)
    compute = stack.compute
    in_stream = torch.cuda.Stream(dev)
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]

    def prefetch(buf, after=None):
        # host -> staging set `buf`, once the compute stream is done with it
        if after is not None:
            in_stream.wait_event(after)
        in_stream.wait_event(free[buf])
        with torch.cuda.stream(in_stream):
            for d, h in zip(stage[buf], host_in):
                d.copy_(h, non_blocking=True)
        ready[buf].record(in_stream)

    def run(n, start=None):
        for b in range(2):
            free[b].record(compute)
        prefetch(0, start)
        for i in range(n):
            buf = i % 2
            compute.wait_event(ready[buf])
            for d, st in zip(dev_in, stage[buf]):
                d.copy_(st, non_blocking=True)
            free[buf].record(compute)
            if i + 1 < n:
                prefetch(1 - buf)
            one_step()
            for h, g in zip(host_grads, grads):
                h.copy_(g, non_blocking=True)

    run(2)
    torch.cuda.synchronize(dev)
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize(dev)
    e0.record(compute)
    run(K, start=e0)
    compute.wait_stream(in_stream)
    drain_copies()
    e1.record(compute)
    torch.cuda.synchronize(dev)
    barrier(ws)
    from host_streamed_nf4_b200 import dist as hdist
    ms = hdist.max_over_ranks(e0.elapsed_time(e1))
    return {"value": round(hdist.job_throughput(stack.tokens_per_step(), K, ms, ws), 1),
            "unit": "tokens/s",
            "ms_per_step": round(ms / K, 4), "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h)}


# ---------------------------------------------------------------------- oracle

_ORACLE_W = {}


def oracle_sample(family, tokens: int, seed: int = 7, base: str = "nf4"):
    """Inputs for `tokens` tokens through one layer of `family` (host arrays);
    the layer's weights are drawn (and, for an NF4 base, quantized) once per
    family.  A dense base is carried as (bf16 bits, absmax None)."""
    import numpy as np

    import oracle
    from host_streamed_nf4_b200 import synth
    key = (family.name, base)
    if key not in _ORACLE_W:
        rng = np.random.default_rng(seed)
        ws = []
        for name, n, k in family.projections():
            w = synth.normal_bf16(rng, (n, k), synth.W_STD)
            codes, absmax = oracle.quantize(w) if base == "nf4" else (w, None)
            ws.append((n, k, codes, absmax,
                       synth.normal_bf16(rng, (synth.RANK, k), synth.A_STD),
                       synth.normal_bf16(rng, (n, synth.RANK), synth.B_STD)))
        _ORACLE_W[key] = ws
    rng = np.random.default_rng(seed + tokens)
    cases = []
    for n, k, codes, absmax, A, B in _ORACLE_W[key]:
        cases.append((n, k, codes, absmax, synth.normal_bf16(rng, (tokens, k), 1.0), A, B,
                      synth.normal_bf16(rng, (tokens, n), 1.0)))
    return cases


def oracle_decoder_sample(family, tokens: int, seed: int = 7):
    """One decoder layer of `family` on the oracle (NF4 weights drawn once per
    family, unit norm gains) and `tokens` tokens of input and output gradient."""
    import numpy as np

    from host_streamed_nf4_b200 import synth
    from oracle import decoder as odec
    cases = oracle_sample(family, 1, seed)
    lin = {}
    for name, (n, k, codes, absmax, _, A, B, _) in zip(synth.PROJ_NAMES, cases):
        lin[name] = odec.Linear(n, k, A=A, B=B, codes=codes, absmax=absmax)
    layer = odec.Layer(H=family.heads, KV=family.kv_heads, d=family.head_dim,
                       g1=np.ones(family.hidden), g2=np.ones(family.hidden), lin=lin)
    rng = np.random.default_rng(seed + tokens)
    h0 = odec.bits_f64(synth.normal_bf16(rng, (tokens, family.hidden), 1.0))
    dh = odec.bits_f64(synth.normal_bf16(rng, (tokens, family.hidden), 1.0))
    return ("decoder", layer, h0, dh)


def oracle_step(cases, threads):
    import oracle
    if isinstance(cases, tuple) and cases[0] == "decoder":
        # forward, its recompute in the backward visit, then the backward
        from oracle import decoder as odec
        _, layer, h0, dh = cases
        odec.layer_forward(layer, h0)
        odec.layer_backward(layer, odec.layer_forward(layer, h0), dh)
        return
    for n, k, codes, absmax, X, A, B, dY in cases:
        if absmax is None:
            oracle.lora_fwd_bf16w(codes, X, A, B, 32.0, n_threads=threads)
        else:
            oracle.lora_fwd(codes, absmax, n, k, X, A, B, 32.0, n_threads=threads)
    for n, k, codes, absmax, X, A, B, dY in reversed(cases):
        if absmax is None:
            oracle.lora_bwd_bf16w(codes, X, A, B, dY, 32.0, n_threads=threads)
        else:
            oracle.lora_bwd(codes, absmax, n, k, X, A, B, dY, 32.0, n_threads=threads)


def _sample(family, tokens, base="nf4", model="projections"):
    if model == "decoder":
        return oracle_decoder_sample(family, tokens)
    return oracle_sample(family, tokens, base=base)


def calibrate_tokens(family, target_s, threads, base="nf4", model="projections"):
    """Largest sample (in tokens) whose oracle step stays near target_s."""
    cases = _sample(family, 1, base, model)
    t = time.perf_counter()
    oracle_step(cases, threads)
    one = time.perf_counter() - t
    cases = _sample(family, 2, base, model)
    t = time.perf_counter()
    oracle_step(cases, threads)
    two = time.perf_counter() - t
    per_token = max(two - one, 1e-3)
    fixed = max(one - per_token, 0.0)
    return max(1, min(512, int((target_s - fixed) / per_token)))


def cpu_baseline(args, family):
    """The oracle, as it stands, on the host cores over a bounded sample of
    the workload: `tokens` tokens through one layer, fwd + bwd, scaled to
    tokens/s for the workload's layer count."""
    import oracle
    oracle.build()
    threads = os.cpu_count() or 1
    tokens = calibrate_tokens(family, 2.0, threads, args.base, args.model)
    cases = _sample(family, tokens, args.base, args.model)
    times = []
    t_end = time.perf_counter() + 15.0
    while time.perf_counter() < t_end or len(times) < 2:
        t = time.perf_counter()
        oracle_step(cases, threads)
        times.append(time.perf_counter() - t)
        if len(times) >= 8:
            break
    per_layer = statistics.median(times)
    value = tokens / (per_layer * args.layers)
    return {"value": round(value, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{tokens} tokens x 1 layer of {family.name} ("
                      + ("decoder layer: fwd, recomputed fwd, bwd" if args.model == "decoder"
                         else "7 projections, fwd+bwd")
                      + f", median of {len(times)} runs); one layer x {args.layers}, "
                      + ("extrapolated" if args.layers > 1 or tokens < args.seq else "measured"),
            "extrapolated": args.layers > 1 or tokens < args.seq}


def run_reference(args, ws, rank):
    import oracle
    from host_streamed_nf4_b200 import synth
    if rank != 0:
        return None
    oracle.build()
    family = synth.FAMILIES[args.family]
    threads = os.cpu_count() or 1
    tokens = calibrate_tokens(family, args.ref_seconds, threads, args.base, args.model)
    cases = _sample(family, tokens, args.base, args.model)
    for _ in range(args.warmup):
        oracle_step(cases, threads)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(cases, threads)
    dt = (time.perf_counter() - t) / args.steps
    value = tokens / (dt * args.layers)
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * args.layers * 1e3 * (args.seq / tokens), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": args.workload + ("-decoder" if args.model == "decoder" else ""),
                       "model": args.model, "family": args.family, "layers": args.layers,
                       "tokens": args.seq, "batch": 1, "mode": "cpu-oracle",
                       "base": args.base},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": threads,
                             "kind": "oracle",
                             "sample": f"{tokens} tokens x 1 layer per step; one layer x "
                                       f"{args.layers}, "
                                       + ("extrapolated" if args.layers > 1 or tokens < args.seq
                                          else "measured")},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    ws, rank, local = dist_setup(args)
    if args.impl == "reference":
        out = run_reference(args, ws, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    out = run_ours(args, ws, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
