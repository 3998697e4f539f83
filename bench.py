#!/usr/bin/env python
"""Benchmark of the dropless top-k MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step = one pass of the whole layer over one batch: route (router logits,
fp32 softmax + top-k, routing metadata) -> dispatch -> grouped gate/up GEMM
with SwiGLU -> grouped down GEMM -> combine, each through the C ABI.
`value` = tokens/s of the whole job with inputs resident in HBM; `e2e` = the
same metric through moe_layer_fwd with the step's input copied from pinned
host memory and the output copied back inside the timed region.

Multi-GPU: the layer is run as independent replicas, one process per GPU
(launched by torch.distributed.run); there is no data-path collective.
`value` = tokens processed by all ranks / max-over-ranks device time.

`--impl reference` times the CPU oracle (test infrastructure) on the host
cores on a bounded sample of the same workload; it is the only other place
besides the cpu_baseline leg where this script runs the oracle.
"""
from __future__ import annotations

import argparse
import datetime
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

import torch  # noqa: E402

from dropless_top_mixture_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MoE-layer tokens/s and grouped-GEMM TFLOP/s (% of peak) on 1 B200; dispatch GB/s"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "olmoe_1b7b"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------- ranks

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=300))


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    """Max of a per-rank scalar over all ranks (every rank calls it)."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons, stamped on arrival."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        try:
            uuid = torch.cuda.get_device_properties(device_index).uuid
            sel = f"GPU-{uuid}"
        except Exception:
            sel = str(device_index)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.th = threading.Thread(target=self._read, daemon=True)
        self.th.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.monotonic(), line.strip()))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def window(self, t0: float, t1: float):
        return [s for (t, s) in self.samples if t0 <= t <= t1]

    @staticmethod
    def summarize(lines):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 8:
                continue
            try:
                sm.append(float(p[0]))
                smax.append(float(p[1]))
            except ValueError:
                continue
            for nm, val in zip(names, p[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- helpers

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def file_hash(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(f"{kernel}/{workload}")
    if not ent:
        return None
    src = os.path.join(ROOT, "dropless_top_mixture_b200", "csrc", ent["source"])
    if not os.path.exists(src) or file_hash(src) != ent["source_sha"]:
        return None
    return ent["dram_bytes_per_launch"]


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


# ---------------------------------------------------------------- CPU oracle arm

def oracle_sample(w, inp_cpu, S: int):
    """Run the CPU oracle on the first S tokens of the workload; returns
    seconds. Routing of the sample, then the per-token SwiGLU mixture."""
    from oracle import moe_oracle as O
    x = inp_cpu["x"][:S]
    t0 = time.perf_counter()
    if w.logits == "router":
        lg = O.router_logits(x, inp_cpu["Wr"])
    else:
        lg = inp_cpu["logits"][:S].numpy()
    idx, gate, _ = O.route(lg, w.k)
    O.routing_metadata(idx, w.E)
    O.moe_layer_tokens(x, list(range(S)), idx, gate, inp_cpu["W1"], inp_cpu["W3"], inp_cpu["W2"])
    return time.perf_counter() - t0


def cpu_baseline(w, inp_cpu, target_s: float = 12.0):
    S = 64
    dt = oracle_sample(w, inp_cpu, S)
    if dt < target_s / 4 and S < w.T:
        S = int(min(w.T, max(S + 1, S * target_s / max(dt, 1e-3))))
        dt = oracle_sample(w, inp_cpu, S)
    return {"value": S / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"first {S} of {w.T} tokens of {w.name}: router logits, top-k, routing "
                      f"metadata and the per-token SwiGLU mixture in float64 ({dt:.1f} s)"}


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inp = make_inputs(w, "cpu")
    S = args.ref_tokens
    for _ in range(args.warmup):
        oracle_sample(w, inp, S)
    times = [oracle_sample(w, inp, S) for _ in range(args.steps)]
    tot = sum(times)
    value = S * args.steps / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_of(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: first {S} of {w.T} tokens of {w.name}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, world):
    return {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "k": w.k, "F": w.F,
            "routing": {"router": "logits = x·Wrᵀ", "normal": "logits ~ N(0,1)",
                        "zipf": "logits ~ N(0,1) + ln Zipf(1.1)"}[w.logits],
            "global_batch": w.T * world, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (no flush)"}


# ---------------------------------------------------------------- GPU arm

def run_ours(args):
    rank, world, local = dist_env()
    dist_init(world, "nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from dropless_top_mixture_b200 import moe

    w = WORKLOADS[args.workload]
    inp = make_inputs(w, dev)
    T, d, E, k, F, R = w.T, w.d, w.E, w.k, w.F, w.R
    dt = w.torch_dtype
    i32 = dict(dtype=torch.int32, device=dev)
    use_router = w.logits == "router"
    x = inp["x"]
    Wr = inp.get("Wr")
    logits = inp.get("logits")
    W1, W3, W2 = inp["W1"], inp["W3"], inp["W2"]
    rt = moe.Route(idx=torch.empty((T, k), **i32), gate=torch.empty((T, k), dtype=torch.float32, device=dev),
                   counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
                   slot=torch.empty((T, k), **i32), tile_offsets=torch.empty(E + 1, **i32))
    rws = torch.empty(moe.lib.moe_route_workspace_size(T, E, int(use_router)), dtype=torch.uint8, device=dev)
    Xe = torch.empty((R, d), dtype=dt, device=dev)
    H = torch.empty((R, F), dtype=dt, device=dev)
    Ye = torch.empty((R, d), dtype=dt, device=dev)
    out = torch.empty((T, d), dtype=dt, device=dev)
    kernels_per_step = (4 if use_router else 3) + 4

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        if use_router:
            moe.moe_route(k, x=x, Wr=Wr, out=rt, workspace=rws)
        else:
            moe.moe_route(k, logits=logits, out=rt, workspace=rws)
        if ev is not None:
            ev[1].record()
        moe.moe_dispatch(x, rt.slot, out=Xe)
        if ev is not None:
            ev[2].record()
        moe.moe_grouped_gate_up(Xe, W1, W3, rt.offsets, H=H)
        if ev is not None:
            ev[3].record()
        moe.moe_grouped_down(H, W2, rt.offsets, Ye=Ye)
        if ev is not None:
            ev[4].record()
        moe.moe_combine(Ye, rt.slot, rt.gate, out=out)
        if ev is not None:
            ev[5].record()

    sampler = ClockSampler(local) if (rank == 0 and not args.no_clocks) else None
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if moe.moe_get_status() != 0:
        raise RuntimeError("device status word set during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    w0 = time.monotonic()
    start.record()
    for i in range(args.steps):
        step(evs[i])
    end.record()
    torch.cuda.synchronize(dev)
    w1 = time.monotonic()
    barrier(world)
    ms_local = start.elapsed_time(end)
    ms_total = max_over_ranks(ms_local, world, dev)
    ms_step = ms_total / args.steps
    value = T * world * args.steps / (ms_total / 1e3)

    parts = ["route", "dispatch", "gate_up", "down", "combine"]
    per = {p: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j, p in enumerate(parts)}

    # clocks: the timed window; if it held too few samples, keep running
    # untimed steps of the same workload while sampling
    extra_s = 0.0
    if sampler is not None:
        lines = sampler.window(w0, w1)
        if len(lines) < 10:
            t_ext0 = time.monotonic()
            while time.monotonic() - t_ext0 < 1.0:
                for _ in range(20):
                    step()
                torch.cuda.synchronize(dev)
            extra_s = time.monotonic() - t_ext0
            lines = sampler.window(w0, time.monotonic())
        clocks = ClockSampler.summarize(lines)
        if clocks is not None and extra_s:
            clocks["note"] = f"timed window plus {extra_s:.1f} s of untimed steps of the same workload"
    else:
        clocks = None

    # end to end through the public call with host buffers
    e2e = None
    if not args.no_e2e:
        x_h = x.cpu().pin_memory()
        lg_h = logits.cpu().pin_memory() if logits is not None else None
        out_h = torch.empty((T, d), dtype=dt).pin_memory()
        x_d = torch.empty_like(x)
        lg_d = torch.empty_like(logits) if logits is not None else None
        lo = moe.moe_layer_fwd(x, k, W1, W3, W2, logits=logits, Wr=Wr)

        def e2e_step():
            x_d.copy_(x_h, non_blocking=True)
            if lg_d is not None:
                lg_d.copy_(lg_h, non_blocking=True)
            moe.moe_layer_fwd(x_d, k, W1, W3, W2, logits=lg_d, Wr=Wr, out=lo)
            out_h.copy_(lo.out, non_blocking=True)

        for _ in range(args.warmup):
            e2e_step()
        barrier(world)
        torch.cuda.synchronize(dev)
        s2 = torch.cuda.Event(enable_timing=True)
        e2 = torch.cuda.Event(enable_timing=True)
        s2.record()
        for _ in range(args.steps):
            e2e_step()
        e2.record()
        torch.cuda.synchronize(dev)
        barrier(world)
        ms_e2e = max_over_ranks(s2.elapsed_time(e2), world, dev)
        h2d = x.numel() * x.element_size() + (logits.numel() * 4 if logits is not None else 0)
        e2e = {"value": T * world * args.steps / (ms_e2e / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": out.numel() * out.element_size()}

    if moe.moe_get_status() != 0:
        raise RuntimeError("device status word set during the timed region")
    if sampler is not None:
        sampler.stop()

    if rank != 0:
        return 0

    peaks, peak_src = measured_peaks()
    es = w.esize
    gemm1_flops = 4.0 * R * d * F
    gemm2_flops = 2.0 * R * d * F
    tf_gate_up = gemm1_flops / (per["gate_up"] / 1e3) / 1e12
    tf_down = gemm2_flops / (per["down"] / 1e3) / 1e12
    tf_ffn = (gemm1_flops + gemm2_flops) / ((per["gate_up"] + per["down"]) / 1e3) / 1e12
    peak_tf = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    disp_bytes = T * d * es + R * d * es + R * 4
    comb_bytes = R * d * es + T * d * es + R * 8
    hbm = peaks["hbm_gbs"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if dt == torch.bfloat16 else "f32",
        "data": "synthetic", "config": config_of(w, world),
        "roofline": {"kernel": "grouped gate_up GEMM + SwiGLU (tcgen05)", "bound": "tensor",
                     "achieved": tf_gate_up, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": tf_gate_up / peak_tf,
                     "peak_source": f"{peak_src} bf16 sustained (kernel timed inside a long step)",
                     "algorithmic_per_launch": f"{gemm1_flops:.4g} flop = 4*R*d*F",
                     "traffic": recorded_traffic("gate_up", w.name)},
        "breakdown_ms": per,
        "grouped_gemm": {"gate_up_tflops": tf_gate_up, "down_tflops": tf_down,
                         "ffn_tflops": tf_ffn, "ffn_frac_of_peak": tf_ffn / peak_tf},
        "hbm": {"dispatch_gbs": disp_bytes / (per["dispatch"] / 1e3) / 1e9,
                "combine_gbs": comb_bytes / (per["combine"] / 1e3) / 1e9,
                "dispatch_frac": disp_bytes / (per["dispatch"] / 1e3) / 1e9 / hbm,
                "combine_frac": comb_bytes / (per["combine"] / 1e3) / 1e9 / hbm,
                "peak_gbs": hbm},
        "e2e": e2e, "gpu_launches": kernels_per_step * args.steps, "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        inp_cpu = {kk: v.cpu() for kk, v in inp.items()}
        line["cpu_baseline"] = cpu_baseline(w, inp_cpu)
    else:
        line["cpu_baseline"] = None
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=64,
                    help="tokens per step of the CPU-oracle reference arm")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true",
                    help="skip nvidia-smi clock sampling (for runs under a profiler)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps; the line reports it
    if args.impl == "reference":
        return run_reference(args)
    rc = run_ours(args)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
