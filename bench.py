"""Benchmark of the KDA operator on B200: prefill tokens/s and decode steps/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  Two timed loops, one per entry point of the
library, because the headline metric is a pair:

* prefill (``value``): kda_chunk_fwd over the prefill workload -- B=4, H=16,
  T=4096, dk=dv=128, chunk 64, bf16 q/k/v/gates, fp32 state -- K timed steps;
  value = tokens of all ranks / max-over-ranks time.
* decode (``decode``): kda_decode_step over the decode workload -- 256
  sequences x 32 heads, fp32 dk=dv=128 states (537 MB) updated in place, fresh
  bf16 q/k/v/gates per step.

Inputs are seeded synthetic tensors resident in HBM before timing; every
timed working set (336 MB prefill inputs, 537 MB decode state) is larger than
the 126 MB L2, so no flush is inserted.  Timing: CUDA events on the launching
stream, W warm-up steps, barrier + synchronize around the K timed steps, max
over ranks.  ``e2e`` repeats the prefill metric through the public call with
the inputs copied from pinned host memory and the outputs read back inside
the timed region.  ``roofline`` compares algorithmic HBM bytes per launch
with the measured copy bandwidth in MEASURED_PEAKS.json.  ``cpu_baseline``
times the fp64 CPU oracle on a bounded sample of the same workload.

Multi-GPU: the operator shards over (sequence, head) with no exchange, so
each rank runs its own full workload ("scaling": "weak") and no collective is
used on the data path.
"""
from __future__ import annotations

import argparse
import faulthandler
import json
import os
import statistics
import sys
import threading
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "KDA prefill tokens/s & decode steps/s on 1 B200; % of tensor/HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- helpers
def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def prefill_bytes(B, T, H, d, gate_bytes=2, io_bytes=2):
    """Algorithmic HBM bytes of one prefill call: q, k, v, log_alpha read, o
    written (d values per token-head each), beta read, S0 read, S_T written."""
    per_token_head = 4 * d * io_bytes + d * gate_bytes + gate_bytes
    return B * T * H * per_token_head + 2 * B * H * d * d * 4


def prefill_flops(B, T, H, d, C=64):
    """Algorithmic flops: 6 d^2 + C (3 dk + 2 dv) per token-head (triangular
    halves of the C x C products)."""
    return B * T * H * (6 * d * d + C * (3 * d + 2 * d))


def decode_bytes(N, H, d, gate_bytes=2, io_bytes=2):
    """Per decode step: the fp32 state read and written once, q, k, v,
    log_alpha read, o written, beta read."""
    return N * H * (2 * d * d * 4 + 4 * d * io_bytes + d * gate_bytes + gate_bytes)


class ClockSampler:
    """SM clock and throttle-reason sampling during a timed region.

    Samples NVML every 5 ms on a background thread (dense enough for timed
    regions of a few ms); without NVML the summary reports "unsampled".
    """

    # NVML clocks-event-reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self._nvml = None
        self._h = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        self._nvml = pynvml
        try:
            # torch reports the PCI location as integers; NVML wants the
            # "domain:bus:device.function" string as bytes
            p = torch.cuda.get_device_properties(self.cuda_index)
            bus = f"{int(p.pci_domain_id):08x}:{int(p.pci_bus_id):02x}:{int(p.pci_device_id):02x}.0".encode()
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = self.cuda_index
            if vis:
                ids = [x.strip() for x in vis.split(",") if x.strip()]
                if idx < len(ids) and ids[idx].isdigit():
                    idx = int(ids[idx])
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        nv = self._nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = get_reasons(self._h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        try:
            self._h = self._handle()
            self.max_mhz = self._nvml.nvmlDeviceGetMaxClockInfo(self._h, self._nvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
            time.sleep(0.02)  # first samples before the timed region starts
        except Exception:
            self._t = None
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0,
                    "source": "nvml"}
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(x for x, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml"}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed(fn, steps, warmup, world, stream):
    """K timed calls of fn bracketed by barrier + synchronize; returns the
    max-over-ranks elapsed seconds (CUDA events on `stream`)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1) / 1e3, world)


# ----------------------------------------------------------------- oracle baseline
def oracle_baseline(w, budget_s: float = 12.0):
    """fp64 oracle on a bounded sample of the prefill workload: whole 4096-token
    sequences of as many (batch row, head) pairs as fit in the time budget,
    run in parallel over all host cores.  Returns tokens/s of the full-head
    workload (token-heads/s divided by H)."""
    import numpy as np
    import oracle
    from gated_delta_rule_110_b200 import inputs as gen
    cores = os.cpu_count() or 1
    oracle.build()
    # a single batch row's worth of inputs on the host
    x = gen.make_inputs(1, w.T, w.H, w.dk, w.dv, dtype=w.dtype, gate=w.gate, seed=w.seed)
    heads = 1
    elapsed = 0.0
    while True:
        hs = min(heads, w.H)
        sub = {kk: x[kk][:, :, :hs] for kk in ("q", "k", "v", "log_alpha", "beta")}
        S0 = x["S0"][:, :hs]
        t0 = time.perf_counter()
        oracle.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"], S0, n_threads=cores)
        elapsed = time.perf_counter() - t0
        if elapsed * 2 > budget_s or hs == w.H:
            break
        heads *= 2
    token_heads = w.T * hs
    return {"value": token_heads / elapsed / w.H, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{hs} head(s) x {w.T} tokens of the prefill workload, fp64, OpenMP over heads; "
                      f"tokens/s = token-heads/s / {w.H}", "seconds": elapsed}


# ----------------------------------------------------------------- arms
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from gated_delta_rule_110_b200 import inputs as gen
    w = gen.workload("prefill")
    vals = []
    for _ in range(args.warmup):
        oracle_baseline(w, budget_s=2.0)
    for _ in range(args.steps):
        vals.append(oracle_baseline(w, budget_s=min(20.0, 120.0 / max(args.steps, 1))))
    v = statistics.median(b["value"] for b in vals)
    cb = dict(vals[-1])
    cb["value"] = v
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill B4 H16 T4096 dk=dv=128 C64 (bounded sample per step)"},
        "cpu_baseline": cb,
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


PROFILE_DIR = ROOT / "profiles"
KERNEL_SOURCES = ("gated_delta_rule_110_b200/csrc/kda_prefill.cuh", "gated_delta_rule_110_b200/csrc/kda_ptx.cuh",
                  "gated_delta_rule_110_b200/csrc/kda_recurrent.cuh", "gated_delta_rule_110_b200/csrc/kda_api.cu",
                  "gated_delta_rule_110_b200/csrc/kda_epilogue.cuh")


def kernel_sources_hash() -> str:
    """sha256 (16 hex digits) of the kernel sources the ncu captures describe."""
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        h.update((ROOT / rel).read_bytes())
    return h.hexdigest()[:16]


def profiled_counters():
    """Per-launch DRAM traffic and tensor-pipe activity recorded from ncu
    captures in profiles/*.md (lines "counter <workload> <name> <value>"),
    valid only while the kernel sources still hash to the value the summary
    was taken at (line "kernel_sources_sha <hex>")."""
    import re
    out = {}
    cur = kernel_sources_hash()
    for f in sorted(PROFILE_DIR.glob("*.md")):
        text = f.read_text()
        m = re.search(r"^kernel_sources_sha (\w+)", text, re.M)
        if not m or m.group(1) != cur:
            continue
        for wl, name, val in re.findall(r"^counter (\w+) (\w+) ([0-9.eE+-]+)", text, re.M):
            out.setdefault(wl, {})[name] = float(val)
    return out


def cpu_model() -> str:
    try:
        for line in Path("/proc/cpuinfo").read_text().splitlines():
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# The layer legs' decay-gate parameters: Mamba's A range with step sizes
# dt in [1e-3, 1e-2], so that chunk decays stay in the factorised range as in
# the plain workloads (the default dt range up to 0.1 sends some chunks of
# the fastest channels to the exact path).
LAYER_DT_RANGE = (1e-3, 1e-2)


def prefill_leg(kda, gen, wname, steps, warmup, world, rank, local, stream, peaks, peak_src, counters,
                gated=False, layer=False):
    """Times kda_chunk_fwd (kda_chunk_fwd_gated with ``gated``: the output
    RMSNorm and sigmoid gate, placed by the library; kda_chunk_fwd_layer with
    ``layer``: raw q, k and the gate projection in, L2 norm and decay gate in
    the kernel, plus the output epilogue) on one workload; returns its JSON
    object."""
    w = gen.workload(wname)
    if layer:
        x = gen.make_layer_inputs(w.B, w.T, w.H, w.dk, w.dv, seqlens=w.seqlens, seed=w.seed + rank, device="cuda",
                                  dt_range=LAYER_DT_RANGE)
    else:
        x = gen.workload_inputs(w, device="cuda", seed_offset=rank)
    cu = x["cu_seqlens"]
    n_seqs = 0 if cu is None else cu.numel() - 1
    N = w.B if cu is None else n_seqs
    shape = kda.make_shape(w.B, w.T, w.H, w.dk, w.dv, 64, n_seqs, kda.KDA_BF16, kda.KDA_BF16)
    ws = torch.empty(max(kda.kda_chunk_fwd_workspace_size(shape), 1), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(x["v"])
    S_T = torch.empty_like(x["S0"])
    if layer:
        gate, nw = gen.output_gate_inputs(x["v"].shape, seed=w.seed + 100 + rank, device="cuda")

        def fn():
            kda.kda_chunk_fwd_layer(x["q"], x["k"], x["v"], x["f"], x["A_log"], x["dt_bias"], x["beta"], x["S0"], cu,
                                    out_gate=gate, norm_weight=nw, eps=1e-5, o=o, S_T=S_T, workspace=ws)
    elif gated:
        gate, nw = gen.output_gate_inputs(x["v"].shape, seed=w.seed + 100 + rank, device="cuda")

        def fn():
            kda.kda_chunk_fwd_gated(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], gate, nw, x["S0"], cu,
                                    eps=1e-5, o=o, S_T=S_T, workspace=ws)
    else:
        def fn():
            kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], cu, o=o, S_T=S_T,
                              workspace=ws)

    label = wname + (" layer" if layer else " gated" if gated else "")
    progress(f"{label}: timing {steps} calls")
    with ClockSampler(local) as clk:
        t = timed(fn, steps, warmup, world, stream)
    err = kda.kda_check_device_error()
    if err != 0:
        raise RuntimeError(f"device error {err} during {label}")
    tokens = w.B * w.T
    ms = t / steps * 1e3
    nbytes = prefill_bytes(tokens, 1, w.H, w.dk) - 2 * tokens * w.H * w.dk * w.dk * 4 + 2 * N * w.H * w.dk * w.dk * 4
    if gated or layer:
        nbytes += tokens * w.H * w.dv * 2 + w.dv * 4  # the gate read, the norm weight
    flops = prefill_flops(tokens, 1, w.H, w.dk)
    gbs = nbytes / (ms / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    c = counters.get(wname + ("_layer" if layer else "_gated" if gated else ""), {})
    traffic = c.get("dram_bytes")
    progress(f"{label}: {ms:.3f} ms/call, {gbs:.0f} GB/s")
    out = {
        "value": tokens * world * steps / t, "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
        "config": {"workload": f"{wname} {w.B}x{w.T} tokens H{w.H} dk=dv={w.dk} C64, bf16 q/k/v/gates, fp32 state"
                               + (", then per-head RMSNorm + sigmoid output gate (bf16 gate; fused into the prefill kernel "
                                  "where its transform CTAs bound the call, else a separate pass over o)" if gated else "")
                               + (": raw q, k and decay-gate projection f in (L2 norm of q, k and log alpha = "
                                  "-exp(A_log) softplus(f + dt_bias) computed in the kernel; A ~ U(1,16), "
                                  "dt ~ logU(1e-3, 1e-2)), per-head RMSNorm + sigmoid output gate out" if layer else ""),
                   "sequences": N, "tokens": tokens, "H": w.H,
                   "l2": f"inputs larger than L2 (no flush): {tokens * w.H * w.dk * 8 / 1e6:.0f} MB read per call"},
        "roofline": {"kernel": "kda_prefill_kernel (one cooperative launch per call)", "bound": "hbm",
                     "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                     "traffic": traffic, "algorithmic_bytes_per_launch": nbytes, "peak_source": peak_src,
                     "tensor": {"achieved_tflops": flops / (ms / 1e3) / 1e12, "peak_tflops": float(peaks["bf16_tflops"]),
                                "frac": flops / (ms / 1e3) / 1e12 / float(peaks["bf16_tflops"]),
                                "pipe_active_pct_ncu": c.get("tensor_pipe_pct")}},
        "clocks": clk.summary(),
    }
    del x, ws, o, S_T
    if gated or layer:
        del gate, nw
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    world, rank, local = dist_setup()
    import gated_delta_rule_110_b200 as kda
    from gated_delta_rule_110_b200 import inputs as gen
    kda.load_library()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()
    counters = profiled_counters()
    launches = 0

    # ---------------- prefill (the headline line)
    pre = prefill_leg(kda, gen, "prefill", args.steps, args.warmup, world, rank, local, stream, peaks, peak_src,
                      counters)
    launches += args.steps
    w = gen.workload("prefill")
    x = gen.workload_inputs(w, device="cuda", seed_offset=rank)
    B, T, H, d = w.B, w.T, w.H, w.dk
    shape = kda.make_shape(B, T, H, d, d, 64, 0, kda.KDA_BF16, kda.KDA_BF16)
    ws = torch.empty(kda.kda_chunk_fwd_workspace_size(shape), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(x["v"])
    S_T = torch.empty_like(x["S0"])
    tokens_per_step = B * T

    # ---------------- e2e: pinned host inputs -> device -> call -> host
    hx = {kk: x[kk].cpu().pin_memory() for kk in ("q", "k", "v", "log_alpha", "beta", "S0")}
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hS = torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory()
    dx = {kk: torch.empty_like(x[kk]) for kk in hx}
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = ho.numel() * ho.element_size() + hS.numel() * hS.element_size()

    def e2e_step():
        for kk in hx:
            dx[kk].copy_(hx[kk], non_blocking=True)
        kda.kda_chunk_fwd(dx["q"], dx["k"], dx["v"], dx["log_alpha"], dx["beta"], dx["S0"], o=o, S_T=S_T,
                          workspace=ws)
        ho.copy_(o, non_blocking=True)
        hS.copy_(S_T, non_blocking=True)

    progress("e2e: timing")
    e2e_steps = max(3, min(args.steps, 10))
    t_e2e = timed(e2e_step, e2e_steps, max(1, min(args.warmup, 3)), world, stream)
    launches += e2e_steps
    e2e_value = tokens_per_step * world * e2e_steps / t_e2e
    del dx, hx, x, ws, o, S_T
    torch.cuda.empty_cache()

    # ---------------- varlen and long-context prefill
    var = prefill_leg(kda, gen, "varlen", args.steps, args.warmup, world, rank, local, stream, peaks, peak_src,
                      counters)
    launches += args.steps
    long_steps = max(3, min(args.steps, 5))
    lng = prefill_leg(kda, gen, "long", long_steps, args.warmup, world, rank, local, stream, peaks, peak_src,
                      counters)
    launches += long_steps
    gtd = prefill_leg(kda, gen, "prefill", args.steps, args.warmup, world, rank, local, stream, peaks, peak_src,
                      counters, gated=True)
    launches += args.steps
    vgt = prefill_leg(kda, gen, "varlen", args.steps, args.warmup, world, rank, local, stream, peaks, peak_src,
                      counters, gated=True)
    launches += args.steps
    lgt = prefill_leg(kda, gen, "long", long_steps, args.warmup, world, rank, local, stream, peaks, peak_src,
                      counters, gated=True)
    launches += 2 * long_steps  # the prefill kernel and the separate epilogue pass
    ply = prefill_leg(kda, gen, "prefill", args.steps, args.warmup, world, rank, local, stream, peaks, peak_src,
                      counters, layer=True)
    launches += args.steps
    lly = prefill_leg(kda, gen, "long", long_steps, args.warmup, world, rank, local, stream, peaks, peak_src,
                      counters, layer=True)
    launches += 2 * long_steps

    # ---------------- decode
    progress("decode: setup")
    wd = gen.workload("decode")
    Nd, Hd = wd.B, wd.H
    S = gen.decode_state(Nd, Hd, d, d, device="cuda", seed=wd.seed + rank)
    n_inputs = 8  # distinct per-step inputs cycled through (each 8 MB, far below the 537 MB state)
    dins = [gen.decode_step_inputs(Nd, Hd, d, d, s, device="cuda", seed=wd.seed + rank) for s in range(n_inputs)]
    od = torch.empty((Nd, Hd, d), dtype=torch.bfloat16, device="cuda")
    counter = [0]

    def decode():
        xi = dins[counter[0] % n_inputs]
        counter[0] += 1
        kda.kda_decode_step(xi["q"], xi["k"], xi["v"], xi["log_alpha"], xi["beta"], S, o=od)

    dec_steps = args.decode_steps
    with ClockSampler(local) as clk_d:
        t_dec = timed(decode, dec_steps, max(args.warmup, 3), world, stream)
    launches += dec_steps
    err = kda.kda_check_device_error()
    if err != 0:
        raise RuntimeError(f"device error {err} during decode")
    dec_ms = t_dec / dec_steps * 1e3
    dec_bytes = decode_bytes(Nd, Hd, d)
    dec_gbs = dec_bytes / (dec_ms / 1e3) / 1e9
    peak_hbm = float(peaks["hbm_gbs"])
    progress(f"decode: {dec_ms:.3f} ms/step")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        progress("cpu baseline")
        cpu = oracle_baseline(w)
        cpu["cpu_model"] = cpu_model()

    if rank == 0:
        line = {
            "metric": METRIC, "value": pre["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": pre["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(pre["config"], B=B, T=T, chunk=64,
                           parallelism=f"weak x{world}: each rank its own workload, no collective"),
            "roofline": pre["roofline"],
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps},
            "gpu_launches": launches,
            "clocks": pre["clocks"],
            "varlen": var,
            "long": lng,
            "prefill_gated": gtd,
            "varlen_gated": vgt,
            "long_gated": lgt,
            "prefill_layer": ply,
            "long_layer": lly,
            "decode": {"value": world * dec_steps / t_dec, "unit": "steps/s", "ms_per_step": dec_ms,
                       "steps": dec_steps,
                       "config": {"workload": "decode 256 seqs x H32 dk=dv=128, fp32 state 537 MB in place, "
                                              "bf16 q/k/v/gates", "N": Nd, "H": Hd, "dk": d, "dv": d},
                       "roofline": {"kernel": "kda_decode_kernel", "bound": "hbm", "achieved": dec_gbs,
                                    "peak": peak_hbm, "unit": "GB/s", "frac": dec_gbs / peak_hbm,
                                    "traffic": counters.get("decode", {}).get("dram_bytes"),
                                    "algorithmic_bytes_per_launch": dec_bytes, "peak_source": peak_src},
                       "clocks": clk_d.summary()},
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_profile(args):
    """One leg alone, for profilers: --profile NAME runs W + K calls of that
    workload's entry point and prints the CUDA-event time per call (no JSON)."""
    import gated_delta_rule_110_b200 as kda
    from gated_delta_rule_110_b200 import inputs as gen
    torch.cuda.set_device(0)
    kda.load_library()
    stream = torch.cuda.current_stream()
    w = gen.workload("prefill" if args.profile.startswith("gated") or args.profile == "layer" else args.profile)
    if args.profile == "decode":
        S = gen.decode_state(w.B, w.H, w.dk, w.dv, device="cuda", seed=w.seed)
        xs = gen.decode_step_inputs(w.B, w.H, w.dk, w.dv, 0, device="cuda", seed=w.seed)
        od = torch.empty((w.B, w.H, w.dv), dtype=torch.bfloat16, device="cuda")

        def fn():
            kda.kda_decode_step(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["beta"], S, o=od)
    else:
        if args.profile == "layer":
            x = gen.make_layer_inputs(w.B, w.T, w.H, w.dk, w.dv, seed=w.seed, device="cuda", dt_range=LAYER_DT_RANGE)
        else:
            x = gen.workload_inputs(w, device="cuda")
        n_seqs = 0 if x["cu_seqlens"] is None else x["cu_seqlens"].numel() - 1
        shape = kda.make_shape(w.B, w.T, w.H, w.dk, w.dv, 64, n_seqs, kda.KDA_BF16, kda.KDA_BF16)
        ws = torch.empty(max(kda.kda_chunk_fwd_workspace_size(shape), 1), dtype=torch.uint8, device="cuda")
        o = torch.empty_like(x["v"])
        S_T = torch.empty_like(x["S0"])

        if args.profile.startswith("gated") or args.profile == "layer":
            gate, nw = gen.output_gate_inputs(x["v"].shape, seed=w.seed + 100, device="cuda")
            mode = "separate" if args.profile == "gated_separate" else "fused"

        def fn():
            if args.profile == "layer":
                kda.kda_chunk_fwd_layer(x["q"], x["k"], x["v"], x["f"], x["A_log"], x["dt_bias"], x["beta"], x["S0"],
                                        out_gate=gate, norm_weight=nw, eps=1e-5, o=o, S_T=S_T, workspace=ws)
            elif args.profile.startswith("gated"):
                kda.kda_chunk_fwd_gated(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], gate, nw, x["S0"],
                                        x["cu_seqlens"], eps=1e-5, o=o, S_T=S_T, workspace=ws, gate_mode=mode)
            else:
                kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], x["cu_seqlens"], o=o,
                                  S_T=S_T, workspace=ws)
    t = timed(fn, args.steps, args.warmup, 1, stream)
    err = kda.kda_check_device_error()
    print(f"{args.profile}: {t / args.steps * 1e6:.1f} us per call over {args.steps} calls, device status {err}",
          flush=True)
    return 0 if err == 0 else 1


def progress(msg: str):
    print(f"[bench] {msg}", file=sys.stderr, flush=True)


def main():
    faulthandler.enable()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=("prefill", "varlen", "long", "decode", "gated", "gated_separate", "layer"),
                    default=None,
                    help="time one workload's entry point alone (for ncu); prints no JSON line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.profile:
        return run_profile(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
