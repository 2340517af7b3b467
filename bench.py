#!/usr/bin/env python
"""Benchmark of the routed MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill]
                    [--impl ours|reference] [--no-extras]

Workload (default "decode"): the 384-expert layer (hidden 4096, top-8,
expert intermediate 2048, bf16 weights ~19 GB, router logits biased by a
Zipf(1.1) prior over a seeded expert permutation) run once at each decode
batch 1, 2, 4, 8, 16, 64; one "step" is the six forwards (95 tokens), each a
full pass of route -> permute -> expert FFN -> combine. "prefill" runs one
4096-token chunk per step. Inputs are seeded synthetic tensors already in HBM;
L2 is flushed (a 256 MiB write) before every forward, outside the timed
events. Time is device time from CUDA events on the launching stream, summed
over the K timed steps, max over ranks.

With N > 1 (torchrun) every rank holds its own replica of the layer and
processes its own tokens: there is no collective in the data path
("replicas", weak scaling); value = tokens of all ranks / max rank time.

Extras (rank 0, N = 1): the dominant kernel's roofline (gate/up GEMM, HBM bytes
per launch over its event-timed duration), per-batch and prefill breakdowns,
the end-to-end number through the public API with host buffers, and the CPU
oracle timed on a bounded sample as a baseline.

--impl reference times the CPU oracle (the correctness reference of this
repository; the pages this follows publish no runnable code) on the host
cores, on the same workload definition, one bounded sample per step.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s (decode B=1..64, prefill 4096) and % of HBM / tensor-pipe roofline"
H, E, K, I = 4096, 384, 8, 2048
DECODE_BATCHES = [1, 2, 4, 8, 16, 64]
ZIPF_S = 1.1
SEED = 0
EXPERT_BYTES = 2 * (2 * I * H + H * I)  # bf16 gate/up + down per expert


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# --------------------------------------------------------------- traffic --
# DRAM bytes per launch of the dominant kernel come from an ncu capture whose
# summary sits under profiles/ with a hash of the kernel's sources at capture
# time; they are reported only while the sources still hash the same.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_decode_sweep.txt")
KERNEL_SOURCES = [os.path.join(ROOT, "mixture_experts_layer_24_b200", "csrc", f)
                  for f in ("ffn_decode.cu", "common.cuh", "tile.cuh", "internal.h")]


def kernel_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(workload):
    """(bytes per launch, source note) from the committed capture, or (None, why)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, "no capture"
    kv = {}
    for line in open(TRAFFIC_FILE):
        if ":" in line and not line.lstrip().startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("workload") != workload:
        return None, "capture is of another workload"
    if kv.get("sources_sha256") != kernel_sources_sha256():
        return None, "kernel changed since the capture"
    try:
        return float(kv["dram_bytes_per_launch"]), TRAFFIC_FILE[len(ROOT) + 1:]
    except (KeyError, ValueError):
        return None, "capture file incomplete"


# ------------------------------------------------------------------ dist --

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world, backend):
    if world > 1:
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=600))


def dist_barrier(world):
    if world > 1:
        torch.distributed.barrier()


def dist_max(world, v, device):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def dist_sum(world, v, device):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """SM clock and clock-event reasons while the timed region runs.

    A thread polls NVML (reads only) about every millisecond, so a timed region
    of a few milliseconds still gets samples; the device is found by its PCI
    bus id. Without NVML it falls back to `nvidia-smi -lms 20`."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.thread = None
        self.samples = []
        self.smax = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            props = torch.cuda.get_device_properties(self.index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop_flag = threading.Event()
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((sm, [n for n, b in bits.items() if r & b]))
                    except Exception:
                        pass
                    time.sleep(0.001)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.source = "nvml"
            return
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
        except Exception:
            self.proc = None

    def window(self):
        """Drops the samples taken so far (NVML): the record covers only what follows."""
        self.samples = []

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            sm = [x for x, _ in self.samples]
            reasons = set(n for _, rs in self.samples for n in rs)
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.smax,
                    "reasons": sorted(reasons), "samples": len(sm), "source": "nvml, 1 ms polling"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
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
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi -lms 20"}


# ----------------------------------------------------------------- layer --

def build_layer(device, wdtype=0):
    import mixture_experts_layer_24_b200 as M
    layer = M.MoeLayer(H, E, K, I, wdtype=wdtype, device=device)
    keep = []
    for e in range(E):
        g, d = synth.expert_weights(e, H, I, seed=SEED, device=device)
        layer.register(e, g, d)
        keep.append((g, d))
    wr = synth.router_weight(E, H, seed=SEED, device=device)
    bias = synth.zipf_logit_bias(E, ZIPF_S, seed=SEED).to(device)
    torch.cuda.synchronize(device)
    return layer, wr, bias, keep


def touched_experts(layer, x, wr, bias):
    idx, _ = layer.route(x, wr, bias)
    return int(torch.unique(idx).numel())


_GRAPHS = {}


def graph_for(layer, x, wr, bias):
    """One CUDA graph per input tensor: the whole forward (route, permute, FFN,
    combine) replays as one launch of the captured kernels."""
    key = (id(layer), x.data_ptr(), x.shape[0])
    if key not in _GRAPHS:
        _GRAPHS[key] = layer.capture(x, wr, bias)
    return _GRAPHS[key][0]


def time_forwards(layer, xs, wr, bias, flush, stream, steps, graphs=False):
    """Device ms of `steps` passes over xs (one forward each), L2 flushed before each.
    Inputs are made on the default stream: `stream` (a torch stream, which does
    not wait for the default stream by itself) is made to wait for them first."""
    stream.wait_stream(torch.cuda.current_stream())
    gs = [graph_for(layer, x, wr, bias) for x in xs] if graphs else None
    pairs = []
    with torch.cuda.stream(stream):
        for _ in range(steps):
            for i, x in enumerate(xs):
                flush.fill_(1)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                if graphs:
                    gs[i].replay()
                else:
                    layer.forward(x, wr, bias, stream=stream)
                b.record(stream)
                pairs.append((a, b))
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in pairs)


# --------------------------------------------------------- cpu baseline --

_EXPERT_CACHE = ({}, {})  # host copies of generated experts, reused across samples
_ROUTER_CACHE = {}

def oracle_sample(n_tokens, first_token, threads, budget_s):
    """Times the CPU oracle on up to n_tokens tokens of the workload (stopping
    once budget_s is spent); returns (tokens, seconds, description)."""
    done, secs = 0, 0.0
    while done < n_tokens and secs < budget_s:
        secs += oracle_batch(1, first_token + done, threads)
        done += 1
    return done, secs


def oracle_batch(b, first_token, threads):
    """Seconds of CPU time the oracle takes for one forward of the b tokens
    first_token .. first_token + b - 1 (the expert weights it needs are drawn
    before the clock starts and kept for later batches)."""
    import oracle
    if "router" not in _ROUTER_CACHE:
        _ROUTER_CACHE["router"] = (synth.router_weight(E, H, seed=SEED).numpy(),
                                   synth.zipf_logit_bias(E, ZIPF_S, seed=SEED).numpy())
    wr, bias = _ROUTER_CACHE["router"]
    gu, dn = _EXPERT_CACHE
    x = synth.tokens(b, H, seed=SEED, first_token=first_token)
    xu = oracle.as_u16(x)
    _, idx, _ = oracle.route(xu, wr, bias, K, threads)
    for e in np.unique(idx):
        if int(e) not in gu:
            g, d = synth.expert_weights(int(e), H, I, seed=SEED)
            gu[int(e)], dn[int(e)] = oracle.as_u16(g), oracle.as_u16(d)
    t0 = time.perf_counter()
    oracle.forward(xu, wr, bias, K, E, gu, dn, threads=threads)
    return time.perf_counter() - t0


def workload_config(workload, batches, world):
    """The config object of the JSON line (both arms)."""
    return {"workload": workload, "hidden": H, "experts": E, "top_k": K, "intermediate": I,
            "batches": batches, "zipf_s": ZIPF_S, "weights": "bf16, seeded N(0,0.02)",
            "l2": "flushed (256 MiB write) before every forward, outside the timed events",
            "parallelism": f"replicas x{world}"}


def sweep_inputs(workload, rank):
    """(batches, first token of each batch): the same tokens in both arms."""
    batches = DECODE_BATCHES if workload == "decode" else [4096]
    tok_base = 100000 * rank  # each replica gets its own tokens
    return batches, [tok_base + 1000 * i for i in range(len(batches))]


# ------------------------------------------------------------- reference --

REF_STEP_BUDGET_S = 8.0


def run_reference(args):
    """The CPU oracle on the same workload: each step walks the decode sweep's
    batches (the same tokens as our arm, batch by batch in the same order) until
    REF_STEP_BUDGET_S of oracle time is spent; the next step resumes where it
    stopped, so over the run the whole sweep is covered. Warm-up steps run one
    batch-1 forward each (they also draw the expert weights)."""
    world, rank, local = dist_env()
    if world > 1 and rank != 0:
        return 0
    threads = os.cpu_count() or 1
    workload = "decode_sweep_bf16" if args.workload == "decode" else "prefill4096_bf16"
    batches, firsts = sweep_inputs(args.workload, 0)
    for _ in range(args.warmup):
        oracle_batch(1, firsts[0], threads)
    tok, secs, nb = 0, 0.0, 0
    cursor = 0  # next batch of the sweep
    for _ in range(args.steps):
        step_s = 0.0
        while True:
            i = cursor % len(batches)
            b = batches[i]
            if args.workload != "decode":
                b = min(b, 8)  # a 4096-token chunk is hours of oracle time: time a bounded slice of it
            dt = oracle_batch(b, firsts[i], threads)
            step_s += dt
            tok += b
            nb += 1
            cursor += 1
            if step_s >= REF_STEP_BUDGET_S:
                break
        secs += step_s
    v = tok / secs
    sample = (f"{tok} tokens in {nb} batches of the sweep {batches} (the same tokens as the GPU arm, batch by "
              f"batch, resuming across steps; {REF_STEP_BUDGET_S:.0f} s of oracle time per step), fp32 plain C "
              f"oracle with OpenMP")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": workload_config(workload, batches, world),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ours --

def run_ours(args):
    import mixture_experts_layer_24_b200 as M
    from mixture_experts_layer_24_b200 import build as B
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    if rank == 0:
        B.build()
    dist_barrier(world)
    M.lib()

    layer, wr, bias, keep = build_layer(device)
    stream = torch.cuda.Stream(device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    batches, firsts = sweep_inputs(args.workload, rank)
    workload = "decode_sweep_bf16" if args.workload == "decode" else "prefill4096_bf16"
    xs = [synth.tokens(b, H, seed=SEED, device=device, first_token=f) for b, f in zip(batches, firsts)]
    layer.workspace(16384 if (world == 1 and not args.no_extras) else max(batches))  # no allocation while timing
    tokens_per_step = sum(batches)

    use_graphs = not args.eager
    clocks = ClockSampler(local)
    clocks.start()  # polling from here; the record is reset when the timed region starts
    # warm-up (also captures the graphs)
    launches0 = layer.launches()
    time_forwards(layer, xs, wr, bias, flush, stream, 1, graphs=False)
    per_forward_launches = (layer.launches() - launches0) / len(xs)
    time_forwards(layer, xs, wr, bias, flush, stream, max(args.warmup, 0), graphs=use_graphs)
    status = layer.status()
    if status:
        raise SystemExit(f"device status {status} after warm-up")

    dist_barrier(world)
    torch.cuda.synchronize()
    clocks.window()
    ms = time_forwards(layer, xs, wr, bias, flush, stream, args.steps, graphs=use_graphs)
    torch.cuda.synchronize()
    clk = clocks.stop()
    launches = int(round(per_forward_launches * len(xs) * args.steps))
    dist_barrier(world)
    ms_max = dist_max(world, ms, device)
    total_tokens = dist_sum(world, tokens_per_step * args.steps, device)
    value = total_tokens / (ms_max / 1000.0)

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(workload, batches, world),
            "launch": "CUDA graph per batch (kernels chained with programmatic dependent launch)"
            if use_graphs else "eager (kernels chained with programmatic dependent launch)",
            "gpu_launches": launches, "gpu_launches_per_step": launches / max(args.steps, 1), "clocks": clk}

    if world == 1 and not args.no_extras:
        args.workload_name = workload
        line.update(extras(layer, wr, bias, xs, batches, flush, stream, args, device, keep))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    layer.close()
    return 0


def extras(layer, wr, bias, xs, batches, flush, stream, args, device, keep):
    import mixture_experts_layer_24_b200 as M
    hbm, tf_burst, tf_sust, peak_kind = peaks()
    out = {}
    # --- per-kernel device time (events inside the library, same stream) ---
    steps = max(3, args.steps)
    M.moe_profile_enable(layer.ctx, True)
    M.moe_profile_read(layer.ctx, reset=True)
    time_forwards(layer, xs, wr, bias, flush, stream, steps)
    prof = M.moe_profile_read(layer.ctx, reset=True)
    M.moe_profile_enable(layer.ctx, False)
    touched = [touched_experts(layer, x, wr, bias) for x in xs]
    gu_bytes = sum(t * 2 * I * H * 2 + b * K * H * 2 + b * K * I * 2 for t, b in zip(touched, batches))
    dn_bytes = sum(t * H * I * 2 + b * K * I * 2 + b * K * H * 4 for t, b in zip(touched, batches))
    gu_ms, gu_n = prof["gate_up"]
    dn_ms, dn_n = prof["down"]
    fu_ms, fu_n = prof["ffn_fused"]
    if fu_n:
        # decode batches run both GEMMs in one launch: its bytes are gate/up + down
        dom_bytes, dom_ms, dom_n = gu_bytes + dn_bytes, fu_ms, fu_n
        dom_name = "ffn fused gate/up + SwiGLU + down x weight (tcgen05, one launch)"
    else:
        dom_bytes, dom_ms, dom_n = gu_bytes, gu_ms, gu_n
        dom_name = "ffn gate/up GEMM + SwiGLU (tcgen05)"
    per_launch_bytes = dom_bytes / len(batches)
    achieved = (dom_bytes * steps) / (dom_ms / 1000.0) / 1e9
    traffic, traffic_src = measured_traffic(args.workload_name)
    out["roofline"] = {"bound": "hbm", "kernel": dom_name, "achieved": achieved,
                       "peak": hbm, "unit": "GB/s", "frac": achieved / hbm, "traffic": traffic,
                       "traffic_source": traffic_src,
                       "peak_source": f"{peak_kind} hbm_gbs",
                       "algorithmic_bytes_per_launch": per_launch_bytes,
                       "avg_launch_us": 1000.0 * dom_ms / max(dom_n, 1)}
    total_ms = sum(v[0] for v in prof.values())
    out["kernels"] = {k: {"ms_per_step": v[0] / steps, "launches_per_step": v[1] / steps,
                          "share": v[0] / total_ms if total_ms else 0.0} for k, v in prof.items() if v[1]}
    if "down" in out["kernels"]:
        out["kernels"]["down"]["achieved_GBps"] = (dn_bytes * steps) / (dn_ms / 1000.0) / 1e9 if dn_ms else None

    # --- per-batch / prefill breakdown ---
    def kernel_profile(x, reps):
        M.moe_profile_enable(layer.ctx, True)
        M.moe_profile_read(layer.ctx, reset=True)
        time_forwards(layer, [x], wr, bias, flush, stream, reps)
        pr = M.moe_profile_read(layer.ctx, reset=True)
        M.moe_profile_enable(layer.ctx, False)
        return {k: round(1000 * v[0] / reps, 2) for k, v in pr.items() if v[1]}

    br = {}
    use_graphs = not args.eager
    for b, x, t in zip(batches, xs, touched):
        time_forwards(layer, [x], wr, bias, flush, stream, 2, graphs=use_graphs)  # warm-up
        ms = time_forwards(layer, [x], wr, bias, flush, stream, 5, graphs=use_graphs) / 5
        ms_eager = time_forwards(layer, [x], wr, bias, flush, stream, 5) / 5
        nbytes = t * EXPERT_BYTES + E * H * 4 + b * H * 2 * 2
        br[f"B{b}"] = {"us_per_layer": 1000 * ms, "us_per_layer_eager": 1000 * ms_eager,
                       "tokens_per_s": b / (ms / 1000), "touched_experts": t,
                       "hbm_roofline_frac": (nbytes / (ms / 1000) / 1e9) / hbm,
                       "kernel_us": kernel_profile(x, 3)}
    if args.workload == "decode":
        for T in (512, 4096, 16384):
            x = synth.tokens(T, H, seed=SEED, device=device, first_token=500000)
            reps = 3 if T < 16384 else 2
            time_forwards(layer, [x], wr, bias, flush, stream, 1)  # warm-up
            ms = time_forwards(layer, [x], wr, bias, flush, stream, reps) / reps
            t = touched_experts(layer, x, wr, bias)
            flops = 2.0 * T * K * (2 * I * H + H * I) + 2.0 * T * E * H
            nbytes = t * EXPERT_BYTES + E * H * 4 + T * H * 4
            br[f"prefill{T}"] = {"us_per_layer": 1000 * ms, "tokens_per_s": T / (ms / 1000), "touched_experts": t,
                                 "kernel_us": kernel_profile(x, 2),
                                 "tensor_frac": (flops / (ms / 1000) / 1e12) / tf_burst,
                                 "hbm_frac": (nbytes / (ms / 1000) / 1e9) / hbm,
                                 "combined_roofline_frac": max(flops / (tf_burst * 1e12), nbytes / (hbm * 1e9)) /
                                 (ms / 1000)}
    out["breakdown"] = br

    if args.workload == "decode" and not args.quick:
        br.update(fp8_breakdown(keep, wr, bias, flush, stream, device, hbm))
        br.update(fp4_breakdown(keep, wr, bias, flush, stream, device, hbm))
        br.update(hotcold_breakdown(keep, wr, bias, flush, stream, device, hbm))

    # --- end to end through the public API, host buffers ---
    hx = [x.cpu().pin_memory() for x in xs]
    hout = [torch.empty_like(x, device="cpu").pin_memory() for x in xs]
    dx = [torch.empty_like(x) for x in xs]
    stream.wait_stream(torch.cuda.current_stream())
    pairs = []
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            for i in range(len(xs)):
                flush.fill_(1)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                dx[i].copy_(hx[i], non_blocking=True)
                y = layer.forward(dx[i], wr, bias, stream=stream)
                hout[i].copy_(y, non_blocking=True)
                b.record(stream)
                pairs.append((a, b))
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in pairs)
    io = sum(b * H * 2 for b in batches)
    out["e2e"] = {"value": sum(batches) * args.steps / (e2e_ms / 1000), "unit": "tokens/s",
                  "h2d_bytes_per_step": io, "d2h_bytes_per_step": io}

    # --- CPU oracle on a bounded sample ---
    threads = os.cpu_count() or 1
    n, secs = oracle_sample(64, 2000, threads, 15.0)
    out["cpu_baseline"] = {"value": n / secs, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                           "sample": f"{n} decode tokens (batch 1 each) through the whole layer, "
                                     f"{secs:.1f} s of CPU time, fp32 plain C oracle with OpenMP"}
    if layer.status():
        out["device_status"] = layer.status()
    return out


def run_profile_case(kind):
    """Small cases for ncu captures of the FFN kernels, three forwards each:
    "t64": the layer shape with 32 experts (1.6 GB of bf16 weights, all
    touched) and 64 tokens; "t1": 8 experts (top-8 of 8, all touched, 400 MB)
    and one token -- the per-launch shape of batch-1 decode; "p2048": 48
    experts and a 2048-token prefill chunk under the Zipf logit prior;
    "f64" / "f2048" / "f1": "t64" / "p2048" / "t1" with e4m3 experts; "m64" /
    "m2048" / "m1": with MXFP4 experts; "r4096": the router
    alone (384 experts, 4096 tokens, Zipf prior), three calls."""
    import mixture_experts_layer_24_b200 as M
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    if kind == "r4096":
        layer = M.MoeLayer(H, E, K, I, device=device)
        wr = synth.router_weight(E, H, seed=SEED, device=device)
        bias = synth.zipf_logit_bias(E, ZIPF_S, seed=SEED).to(device)
        x = synth.tokens(4096, H, seed=SEED, device=device)
        for _ in range(3):
            layer.route(x, wr, bias)
        torch.cuda.synchronize()
        st = layer.status()
        print(json.dumps({"profile_case": f"router E={E} H={H} K={K} T=4096", "status": st}))
        layer.close()
        return 1 if st else 0
    E_s, T_s = {"t64": (32, 64), "t1": (8, 1), "p2048": (48, 2048), "f64": (32, 64), "f2048": (48, 2048),
                "f1": (8, 1), "m64": (32, 64), "m2048": (48, 2048), "m1": (8, 1)}[kind]
    fp8 = kind in ("f64", "f2048", "f1")
    mx = kind in ("m64", "m2048", "m1")
    wd = M.MOE_FP8_E4M3_B128 if fp8 else (M.MOE_MXFP4 if mx else M.MOE_BF16)
    layer = M.MoeLayer(H, E_s, K, I, wdtype=wd, device=device)
    keep = []
    for e in range(E_s):
        g, d = synth.expert_weights(e, H, I, seed=SEED, device=device)
        if mx:
            w = quantize_expert_mx(M, g, d, device)
            del g, d
            layer.register(e, *w)
            keep.append(w)
        elif fp8:
            w = quantize_expert(M, g, d, device)
            del g, d
            layer.register(e, *w)
            keep.append(w)
        else:
            layer.register(e, g, d)
            keep.append((g, d))
    wr = synth.router_weight(E_s, H, seed=SEED, device=device)
    bias = synth.zipf_logit_bias(E_s, ZIPF_S, seed=SEED).to(device) if kind in ("p2048", "f2048", "m2048") else None
    x = synth.tokens(T_s, H, seed=SEED, device=device)
    for _ in range(3):
        layer.forward(x, wr, bias)
    torch.cuda.synchronize()
    st = layer.status()
    print(json.dumps({"profile_case": f"E={E_s} H={H} I={I} K={K} T={T_s} {'e4m3' if fp8 else ('mxfp4' if mx else 'bf16')}",
                      "status": st}))
    layer.close()
    return 1 if st else 0


def quantize_expert(M, g, d, device):
    """(codes_gu, codes_dn, scales_gu, scales_dn): e4m3 with 128x128 block
    scales, quantised on the GPU by the library's quantiser."""
    qg = torch.empty((2 * I, H), dtype=torch.uint8, device=device)
    sg = torch.empty((2 * I // 128, H // 128), dtype=torch.float32, device=device)
    qd = torch.empty((H, I), dtype=torch.uint8, device=device)
    sd = torch.empty((H // 128, I // 128), dtype=torch.float32, device=device)
    M.moe_quantize_e4m3(g, 2 * I, H, 128, qg, sg)
    M.moe_quantize_e4m3(d, H, I, 128, qd, sd)
    return qg, qd, sg, sd


def quantize_expert_mx(M, g, d, device):
    """(codes_gu, codes_dn, scales_gu, scales_dn): packed E2M1 codes and E8M0
    scales per 32 elements, quantised on the GPU by the library's MX quantiser."""
    qg = torch.empty((2 * I, H // 2), dtype=torch.uint8, device=device)
    sg = torch.empty((2 * I, H // 32), dtype=torch.uint8, device=device)
    qd = torch.empty((H, I // 2), dtype=torch.uint8, device=device)
    sd = torch.empty((H, I // 32), dtype=torch.uint8, device=device)
    M.moe_quantize_mx(g, 2 * I, H, 0, qg, sg)
    M.moe_quantize_mx(d, H, I, 0, qd, sd)
    return qg, qd, sg, sd


def layer_kernel_us(layer, x, wr, bias, flush, stream, reps):
    """Per-kernel device time (us per forward) of one layer's forwards, from the library's own events."""
    import mixture_experts_layer_24_b200 as M
    M.moe_profile_enable(layer.ctx, True)
    M.moe_profile_read(layer.ctx, reset=True)
    time_forwards(layer, [x], wr, bias, flush, stream, reps)
    pr = M.moe_profile_read(layer.ctx, reset=True)
    M.moe_profile_enable(layer.ctx, False)
    return {k: round(1000 * v[0] / reps, 2) for k, v in pr.items() if v[1]}


def fp8_breakdown(keep, wr, bias, flush, stream, device, hbm):
    """The same layer with e4m3 experts (128x128 block scales, quantised on the
    GPU from the bf16 weights): decode B=1, 8, 64 and a 4096-token chunk."""
    import mixture_experts_layer_24_b200 as M
    layer = M.MoeLayer(H, E, K, I, wdtype=M.MOE_FP8_E4M3_B128, device=device)
    qkeep = []
    for e in range(E):
        w = quantize_expert(M, keep[e][0], keep[e][1], device)
        layer.register(e, *w)
        qkeep.append(w)
    torch.cuda.synchronize()
    layer.workspace(4096)
    fp8_bytes = 3 * I * H + 2 * (2 * I // 128) * (H // 128) * 4 + 2 * (H // 128) * (I // 128) * 4
    out = {}
    for T in (1, 8, 64, 4096):
        x = synth.tokens(T, H, seed=SEED, device=device, first_token=600000)
        time_forwards(layer, [x], wr, bias, flush, stream, 2)
        reps = 5 if T < 4096 else 3
        ms = time_forwards(layer, [x], wr, bias, flush, stream, reps) / reps
        t = touched_experts(layer, x, wr, bias)
        nbytes = t * fp8_bytes + E * H * 4 + T * H * 4
        out[f"fp8_B{T}" if T < 4096 else "fp8_prefill4096"] = {
            "us_per_layer": 1000 * ms, "tokens_per_s": T / (ms / 1000), "touched_experts": t,
            "hbm_roofline_frac": (nbytes / (ms / 1000) / 1e9) / hbm,
            "kernel_us": layer_kernel_us(layer, x, wr, bias, flush, stream, 2)}
    if layer.status():
        out["fp8_device_status"] = layer.status()
    layer.close()
    del qkeep
    torch.cuda.empty_cache()
    return out


def fp4_breakdown(keep, wr, bias, flush, stream, device, hbm):
    """The same layer with MXFP4 experts (E2M1 codes and E8M0 scales per 32
    elements, quantised on the GPU from the bf16 weights by the MX quantiser):
    decode B=1, 8, 64 and a 4096-token chunk. Bytes per touched expert: the
    packed codes (3 I H / 2) and the scale bytes (3 I H / 32)."""
    import mixture_experts_layer_24_b200 as M
    layer = M.MoeLayer(H, E, K, I, wdtype=M.MOE_MXFP4, device=device)
    qkeep = []
    for e in range(E):
        w = quantize_expert_mx(M, keep[e][0], keep[e][1], device)
        layer.register(e, *w)
        qkeep.append(w)
    torch.cuda.synchronize()
    layer.workspace(4096)
    fp4_bytes = 3 * I * H // 2 + 3 * I * H // 32
    out = {}
    for T in (1, 8, 64, 4096):
        x = synth.tokens(T, H, seed=SEED, device=device, first_token=600000)
        time_forwards(layer, [x], wr, bias, flush, stream, 2)
        reps = 5 if T < 4096 else 3
        ms = time_forwards(layer, [x], wr, bias, flush, stream, reps) / reps
        t = touched_experts(layer, x, wr, bias)
        nbytes = t * fp4_bytes + E * H * 4 + T * H * 4
        out[f"fp4_B{T}" if T < 4096 else "fp4_prefill4096"] = {
            "us_per_layer": 1000 * ms, "tokens_per_s": T / (ms / 1000), "touched_experts": t,
            "hbm_roofline_frac": (nbytes / (ms / 1000) / 1e9) / hbm,
            "kernel_us": layer_kernel_us(layer, x, wr, bias, flush, stream, 2)}
    if layer.status():
        out["fp4_device_status"] = layer.status()
    layer.close()
    del qkeep
    torch.cuda.empty_cache()
    return out


def hotcold_breakdown(keep, wr, bias, flush, stream, device, hbm, n_hot=120, n_spare=32, n_cache_all=128):
    """Expert residency with the spare slots as an LRU cache of host-resident experts.

    "hot set": 120 of the 384 experts resident (greedy hot set from a seeded
    2048-token routing histogram), the other 264 in pinned host memory behind 32
    spare HBM slots. "all through the cache": every expert in pinned host
    memory behind 128 slots. Decode runs a stream of forwards over new tokens
    (so hits come from routing locality, not from repeating a batch): 4
    forwards fill the cache, the next 20 are timed. Bound per forward:
    max(HBM-read bytes / HBM, copied bytes / measured pinned H2D rate)."""
    import mixture_experts_layer_24_b200 as M
    probe = M.MoeLayer(H, E, K, I, device=device)
    for e in range(E):
        probe.register(e, *keep[e])
    hx = synth.tokens(2048, H, seed=SEED, device=device, first_token=700000)
    idx, _ = probe.route(hx, wr, bias)
    hist = torch.bincount(idx.reshape(-1).long(), minlength=E).cpu()
    hot = set(M.moe_plan_hot_set(hist, n_hot).tolist())
    probe.close()
    host = {e: tuple(t.cpu().pin_memory() for t in keep[e]) for e in range(E)}
    # pinned host -> HBM rate of the expert records the forwards stage: eight host experts (403 MB) copied back to
    # back, one copy per tensor as the staging does, after one warm-up pass; best of three
    cold_list = [e for e in range(E) if e not in hot][:8]
    scratch = [torch.empty_like(t, device=device) for t in host[cold_list[0]]]
    nbytes = sum(t.numel() * t.element_size() for e in cold_list for t in host[e])
    best_ms = None
    for rep in range(4):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for e in cold_list:
            for d, t in zip(scratch, host[e]):
                d.copy_(t, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        if rep:
            best_ms = a.elapsed_time(b) if best_ms is None else min(best_ms, a.elapsed_time(b))
    h2d_gbs = nbytes / (best_ms / 1000) / 1e9
    del scratch
    out = {"hotcold_h2d_GBps": h2d_gbs}

    def stream_of(layer, T, n_fill=4, n_time=20, base=610000):
        ms_tot, bound_tot, hits, routed, copied, touched_tot = 0.0, 0.0, 0, 0, 0, 0
        ms_nocopy = []  # forwards that copied nothing (every routed host expert was cached, or none routed)
        for i in range(n_fill + n_time):
            x = synth.tokens(T, H, seed=SEED, device=device, first_token=base + 1000 * i)
            ms = time_forwards(layer, [x], wr, bias, flush, stream, 1)
            if i < n_fill:
                continue
            st = layer.stats()
            ms_tot += ms
            if st["last_cold"] == 0:
                ms_nocopy.append(ms)
            hits += st["last_hits"]
            routed += st["last_routed_cold"]
            copied += st["last_cold"]
            touched_tot += st["last_touched"]
            hbm_bytes = st["last_touched"] * EXPERT_BYTES
            bound_tot += max(hbm_bytes / (hbm * 1e9), st["last_cold"] * EXPERT_BYTES / (h2d_gbs * 1e9))
        return {"us_per_layer": 1000 * ms_tot / n_time, "tokens_per_s": T * n_time / (ms_tot / 1000),
                "touched_experts_mean": touched_tot / n_time, "host_experts_routed_mean": routed / n_time,
                "copied_experts_mean": copied / n_time, "hit_rate": hits / routed if routed else None,
                "us_per_layer_no_copy": 1000 * statistics.median(ms_nocopy) if ms_nocopy else None,
                "forwards_no_copy": len(ms_nocopy),
                "roofline_frac": bound_tot / (ms_tot / 1000) if ms_tot > 0 else None,
                "sample": f"{n_time} forwards over new tokens after {n_fill} that fill the cache"}

    # ---- hot set + LRU cache of the rest
    layer = M.MoeLayer(H, E, K, I, n_spare_slots=n_spare, device=device)
    for e in range(E):
        if e in hot:
            layer.register(e, *keep[e])
        else:
            layer.register(e, *host[e], None, None, M.MOE_LOC_HOST_PINNED)
    for T in (1, 4):
        out[f"hotcold_B{T}"] = stream_of(layer, T)
    x = synth.tokens(4096, H, seed=SEED, device=device, first_token=610000)
    time_forwards(layer, [x], wr, bias, flush, stream, 1)
    reps = 3
    ms = time_forwards(layer, [x], wr, bias, flush, stream, reps) / reps
    st = layer.stats()
    cold, touched = st["last_cold"], st["last_touched"]
    bound_s = max((touched - cold) * EXPERT_BYTES / (hbm * 1e9), cold * EXPERT_BYTES / (h2d_gbs * 1e9))
    out["hotcold_prefill4096"] = {"us_per_layer": 1000 * ms, "tokens_per_s": 4096 / (ms / 1000),
                                  "touched_experts": touched, "cold_experts_staged": cold,
                                  "cold_bytes": cold * EXPERT_BYTES,
                                  "roofline_frac": bound_s / (ms / 1000) if ms > 0 else None}
    if layer.status():
        out["hotcold_device_status"] = layer.status()
    layer.close()

    # ---- every expert through a 128-slot cache
    layer = M.MoeLayer(H, E, K, I, n_spare_slots=n_cache_all, device=device)
    for e in range(E):
        layer.register(e, *host[e], None, None, M.MOE_LOC_HOST_PINNED)
    out["lru_all_B4"] = stream_of(layer, 4, n_fill=8)
    out["lru_all_B4"]["cache_slots"] = n_cache_all
    if layer.status():
        out["lru_all_device_status"] = layer.status()
    layer.close()
    del host
    return out


def run_ep(args):
    """Expert parallelism (--ep): experts split by range over the N ranks (384/N
    each), every rank routes its own tokens (the decode sweep, or a 4096-token
    chunk) and the pairs travel to the experts' GPUs and back by NCCL
    all-to-all (mixture_experts_layer_24_b200.ep). Per-rank work is fixed as N
    grows ("weak"); value = tokens of all ranks / max rank time. Each forward
    reads the per-expert counts on the host once (the all-to-all split sizes),
    so it is not graph-captured."""
    from mixture_experts_layer_24_b200 import build as B
    from mixture_experts_layer_24_b200 import ep
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    if rank == 0:
        B.build()
    dist_barrier(world)
    steps = ep.LibmoeSteps(H, E, K, I, rank, world, device=device)
    keep = []
    for e in range(steps.e0, steps.e0 + steps.E_loc):
        g, d = synth.expert_weights(e, H, I, seed=SEED, device=device)
        steps.register(e, g, d)
        keep.append((g, d))
    wr = synth.router_weight(E, H, seed=SEED, device=device)
    bias = synth.zipf_logit_bias(E, ZIPF_S, seed=SEED).to(device)
    comm = ep.TorchComm() if world > 1 else ep.LocalComm.group(1)[0]
    batches, firsts = sweep_inputs(args.workload, rank)
    xs = [synth.tokens(b, H, seed=SEED, device=device, first_token=f) for b, f in zip(batches, firsts)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    torch.cuda.synchronize()

    def one_pass():
        ms = 0.0
        for x in xs:
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            ep.ep_forward(steps, comm, x, wr, bias)
            b.record()
            b.synchronize()
            ms += a.elapsed_time(b)
        return ms

    for _ in range(args.warmup):
        one_pass()
    if steps.status():
        raise SystemExit("device status after warm-up")
    clocks = ClockSampler(local)
    clocks.start()
    dist_barrier(world)
    torch.cuda.synchronize()
    clocks.window()
    ms = sum(one_pass() for _ in range(args.steps))
    torch.cuda.synchronize()
    clk = clocks.stop()
    dist_barrier(world)
    ms_max = dist_max(world, ms, device)
    total_tokens = dist_sum(world, sum(batches) * args.steps, device)
    workload = "decode_sweep_bf16" if args.workload == "decode" else "prefill4096_bf16"
    cfg = workload_config(workload, batches, world)
    cfg["parallelism"] = f"ep{world} (experts split by range, NCCL all-to-all of pairs)"
    line = {"metric": METRIC, "value": total_tokens / (ms_max / 1000.0), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": cfg, "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)
    steps.close()
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill"])
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--eager", action="store_true", help="no CUDA graphs in the timed region")
    ap.add_argument("--quick", action="store_true", help="skip the FP8 and hot/cold breakdowns")
    ap.add_argument("--ep", action="store_true", help="expert parallelism over the ranks instead of replicas")
    ap.add_argument("--profile-case", nargs="?", const="t64", default=None, choices=["t64", "t1", "p2048", "f64", "f2048", "f1", "m64", "m2048", "m1", "r4096"],
                    help="small ncu case, 3 forwards, no timing: t64 = 32 experts x 64 tokens, t1 = 8 experts x 1 token")
    args = ap.parse_args()
    if args.profile_case:
        return run_profile_case(args.profile_case)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.ep:
        return run_ep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
