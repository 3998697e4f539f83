#!/usr/bin/env python
"""Benchmark of the dropless top-k MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--also NAMES] [--impl ours|reference]

One step = one pass of the whole layer over one batch: route (router logits,
fp32 softmax + top-k, routing metadata) -> dispatch (recording each row's
gate) -> grouped gate/up GEMM with SwiGLU -> grouped down GEMM with the gates
in its epilogue -> combine, each through the C ABI (the sequence
moe_layer_fwd runs; with --backward the gates stay in the combine, since the
router backward reads the expert rows unscaled).
The default workload is the 128-expert layer of the expert-count sweep
(T=8192, d=4096, E=128, top-4, ffn 2048, bf16, logits ~ N(0,1)), the
configuration the layer's targets are stated on; the OLMoE-shaped layer
(router from x·Wrᵀ) is timed the same way in the same run and reported
under "also".
`value` = tokens/s of the whole job with inputs resident in HBM, timed over
one replay of the K steps captured in a CUDA graph (the same library calls,
with CUDA events between the parts captured too, which give the breakdown);
eager steps with --no-graph (their time is always reported as well);
`e2e` = the same metric through moe_layer_fwd with the step's input copied
from pinned host memory and the output copied back inside the timed region.
`cpu_baseline` / `cpu_baseline_one_thread` = the CPU oracle on a bounded
sample of the workload, on the host's BLAS threads / on one thread.

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
DEFAULT_WORKLOAD = "sweep_e128"
ALSO_WORKLOAD = "olmoe_1b7b"
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

def oracle_sample(w, inp_cpu, S: int, backward: bool = False):
    """Run the CPU oracle on the first S tokens of the workload; returns
    seconds. Routing of the sample, then the per-token SwiGLU mixture (the
    MXFP8 oracle for the MXFP8 workload; plus the input gradient of those
    tokens when the step includes the backward)."""
    from oracle import moe_oracle as O
    x = inp_cpu["x"][:S]
    t0 = time.perf_counter()
    if w.logits == "router":
        lg = O.router_logits(x, inp_cpu["Wr"])
    else:
        lg = inp_cpu["logits"][:S].numpy()
    if w.mxfp8:
        O.mxfp8_layer(x, w.k, inp_cpu["W1"], inp_cpu["W3"], inp_cpu["W2"], lg)
        if backward:
            # the float64 input gradient of the sample (the oracle's MXFP8
            # backward re-quantises whole expert weights per call, minutes
            # per expert on the host, so it is not what the sample times)
            O.moe_layer_bwd_sampled(x, inp_cpu["dOut"][:S], w.k, inp_cpu["W1"], inp_cpu["W3"],
                                    inp_cpu["W2"], lg, list(range(S)), [])
        return time.perf_counter() - t0
    idx, gate, _ = O.route(lg, w.k)
    O.routing_metadata(idx, w.E)
    O.moe_layer_tokens(x, list(range(S)), idx, gate, inp_cpu["W1"], inp_cpu["W3"], inp_cpu["W2"])
    if backward:
        O.moe_layer_bwd_sampled(x, inp_cpu["dOut"][:S], w.k, inp_cpu["W1"], inp_cpu["W3"],
                                inp_cpu["W2"], lg, list(range(S)), [])
    return time.perf_counter() - t0


def cpu_baseline(w, inp_cpu, target_s: float = 15.0, backward: bool = False, threads=None):
    """The oracle as it stands on a bounded sample of the workload, on the
    host's cores (BLAS and OpenMP threads as configured) or, with
    ``threads``, limited to that many threads."""
    import contextlib
    lim = contextlib.nullcontext()
    if threads is not None:
        from threadpoolctl import threadpool_limits
        lim = threadpool_limits(limits=threads)
    with lim:
        # the MXFP8 oracle quantises each routed expert's whole weights
        # (seconds per expert on the host), so its sample is a couple of tokens
        S = 2 if w.mxfp8 else (16 if backward else 64)
        if threads == 1 and not w.mxfp8:
            S = max(4, S // 4)
        dt = oracle_sample(w, inp_cpu, S, backward)
        if dt < target_s / 2 and S < w.T:
            S = int(min(w.T, max(S + 1, S * target_s / max(dt, 1e-3))))
            dt = oracle_sample(w, inp_cpu, S, backward)
        cores = threads if threads is not None else blas_threads()
    what = ("router logits, top-k, routing metadata and the per-token "
            + ("MXFP8 SwiGLU mixture" if w.mxfp8 else "SwiGLU mixture")
            + ((" plus the float64 input gradient of those tokens (no weight gradients)"
                if w.mxfp8 else " plus the input gradient of those tokens (no weight gradients)")
               if backward else "")
            + " in float64")
    return {"value": S / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"first {S} of {w.T} tokens of {w.name}: {what} ({dt:.1f} s)"}


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    if args.backward and not w.backward:
        w = w.scaled(name=w.name, backward=True)  # adds the upstream gradient dOut
    inp = make_inputs(w, "cpu")
    S = args.ref_tokens
    for _ in range(args.warmup):
        oracle_sample(w, inp, S, args.backward)
    times = [oracle_sample(w, inp, S, args.backward) for _ in range(args.steps)]
    tot = sum(times)
    value = S * args.steps / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_of(w, world, args.backward),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: first {S} of {w.T} tokens of {w.name}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, world, backward=False):
    return {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "k": w.k, "F": w.F,
            "pass": "forward + backward" if backward else "forward",
            "precision": "MXFP8 (E4M3, UE8M0 block scales)" if w.mxfp8 else w.dtype,
            "routing": {"router": "logits = x·Wrᵀ", "normal": "logits ~ N(0,1)",
                        "zipf": "logits ~ N(0,1) + ln Zipf(1.1)"}[w.logits],
            "global_batch": w.T * world, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (no flush)"}


# ---------------------------------------------------------------- GPU arm

def _steps(moe, w, inp, dev, backward):
    """Buffers and the step of one workload. Returns (parts, step,
    kernels_per_step, work) where work[part] = (flop, algorithmic bytes)."""
    T, d, E, k, F, R = w.T, w.d, w.E, w.k, w.F, w.R
    dt = w.torch_dtype
    es = w.esize
    i32 = dict(dtype=torch.int32, device=dev)
    use_router = w.logits == "router"
    x, Wr, logits = inp["x"], inp.get("Wr"), inp.get("logits")
    W1, W3, W2 = inp["W1"], inp["W3"], inp["W2"]
    rt = moe.Route(idx=torch.empty((T, k), **i32),
                   gate=torch.empty((T, k), dtype=torch.float32, device=dev),
                   counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
                   slot=torch.empty((T, k), **i32), tile_offsets=torch.empty(E + 1, **i32))
    if use_router and backward:
        rt.logits = torch.empty((T, E), dtype=torch.float32, device=dev)  # kept for the router bwd
    rws = torch.empty(moe.lib.moe_route_workspace_size(T, E, int(use_router)), dtype=torch.uint8,
                      device=dev)
    out = torch.empty((T, d), dtype=torch.bfloat16 if w.mxfp8 else dt, device=dev)
    Ye = torch.empty((R, d), dtype=torch.bfloat16 if w.mxfp8 else dt, device=dev)

    def route():
        if use_router:
            moe.moe_route(k, x=x, Wr=Wr, out=rt, workspace=rws)
        else:
            moe.moe_route(k, logits=logits, out=rt, workspace=rws)

    if w.mxfp8:
        mw = moe.mxfp8_quantize_weights(W1, W3, W2)  # offline, outside the timed region
        Xq = torch.empty((R, d), dtype=torch.uint8, device=dev)
        Xs = torch.empty((R, d // 32), dtype=torch.uint8, device=dev)
        Hq = torch.empty((R, F), dtype=torch.uint8, device=dev)
        # activation scales in the tile-packed layout the GEMMs copy
        Xsp = torch.empty(moe.lib.mxfp8_act_scales_packed_size(E, R, d), dtype=torch.uint8,
                          device=dev)
        Hsp = torch.empty(moe.lib.mxfp8_act_scales_packed_size(E, R, F), dtype=torch.uint8,
                          device=dev)

        def mx_dispatch():
            moe.moe_dispatch_mxfp8(x, rt.slot, Xq, Xs)
            moe.mxfp8_pack_act_scales(Xs, rt.offsets, E, Xsp)

        A = torch.empty((R, F), dtype=torch.bfloat16, device=dev) if backward else None
        B = torch.empty((R, F), dtype=torch.bfloat16, device=dev) if backward else None
        fns = [("route", route),
               ("dispatch", mx_dispatch),
               ("gate_up", lambda: moe.moe_grouped_gate_up_mxfp8(Xq, Xsp, mw, rt.offsets, Hq, Hsp,
                                                                 packed=True, A=A, B=B)),
               ("down", lambda: moe.moe_grouped_down_mxfp8(Hq, Hsp, mw, rt.offsets, Ye,
                                                           packed=True)),
               ("combine", lambda: moe.moe_combine(Ye, rt.slot, rt.gate, out=out))]
        sx, sw, sh = 1 + 1 / 32, 1 + 1 / 32, 1 + 1 / 32
        if backward:
            # the backward weights, re-quantised along F (W1, W3) and d (W2):
            # once per weight update, outside the timed region like mw
            wb = moe.mxfp8_quantize_weights_bwd(W1, W3, W2)
            dOut = inp["dOut"]
            u8 = dict(dtype=torch.uint8, device=dev)
            bf = dict(dtype=torch.bfloat16, device=dev)
            dYe = torch.empty((R, d), **bf)
            dYq, dYs = torch.empty((R, d), **u8), torch.empty((R, d // 32), **u8)
            dYsp = torch.empty(moe.lib.mxfp8_act_scales_packed_size(E, R, d), **u8)
            dH = torch.empty((R, F), **bf)
            dA, dB = torch.empty((R, F), **bf), torch.empty((R, F), **bf)
            dq, ds = torch.empty((R, 2 * F), **u8), torch.empty((R, 2 * F // 32), **u8)
            dsp = torch.empty(moe.lib.mxfp8_act_scales_packed_size(E, R, 2 * F), **u8)
            dXe, Xd = torch.empty((R, d), **bf), torch.empty((R, d), **bf)
            Hs, Hd = torch.empty((R, F // 32), **u8), torch.empty((R, F), **bf)
            dx = torch.empty((T, d), **bf)
            dW = (torch.empty((E, F, d), **bf), torch.empty((E, F, d), **bf),
                  torch.empty((E, d, F), **bf))

            def bwd_dispatch():
                moe.moe_dispatch(dOut, rt.slot, gate=rt.gate, out=dYe)
                moe.mxfp8_quantize(dYe, q=dYq, scales=dYs)
                moe.mxfp8_pack_act_scales(dYs, rt.offsets, E, dYsp)

            def bwd_swiglu():
                moe.moe_swiglu_bwd_mxfp8(dH, A, B, dA, dB, dq, ds)
                moe.mxfp8_pack_act_scales(ds, rt.offsets, E, dsp)

            def bwd_dequant():
                moe.mxfp8_dequantize(Xq, Xs, out=Xd)
                moe.mxfp8_unpack_act_scales(Hsp, rt.offsets, E, R, F, Hs)
                moe.mxfp8_dequantize(Hq, Hs, out=Hd)

            aux = torch.empty(1, dtype=torch.float32, device=dev)
            aux_ws = torch.empty(moe.lib.moe_aux_loss_workspace_size(T, E), **u8)
            rg = moe.RouterGrads(dgate=torch.empty((T, k), dtype=torch.float32, device=dev),
                                 dlogits=torch.empty((T, E), dtype=torch.float32, device=dev))
            fns += [("bwd_dispatch", bwd_dispatch),
                    ("bwd_dH", lambda: moe.moe_grouped_mxfp8_gemm(dYq, dYsp, wb.W2tq, wb.Ps2t,
                                                                  rt.offsets, dH)),
                    ("bwd_swiglu", bwd_swiglu),
                    ("bwd_dX", lambda: moe.moe_grouped_mxfp8_gemm(dq, dsp, wb.W13tq, wb.Ps13t,
                                                                  rt.offsets, dXe)),
                    ("bwd_combine", lambda: moe.moe_combine(dXe, rt.slot, None, out=dx)),
                    ("bwd_dequant", bwd_dequant),
                    ("bwd_dW", lambda: moe.moe_grouped_swiglu_wgrad(Xd, dA, dB, dYe, Hd,
                                                                    rt.offsets, out=dW)),
                    ("aux_loss", lambda: moe.moe_aux_loss(logits, rt.counts, out=aux,
                                                          workspace=aux_ws)),
                    ("router_bwd", lambda: moe.moe_router_bwd(
                        dOut, Ye, rt.slot, rt.idx, logits, rt.counts, aux_coef=0.01,
                        dgate=rg.dgate, dlogits=rg.dlogits))]
    else:
        Xe = torch.empty((R, d), dtype=dt, device=dev)
        H = torch.empty((R, F), dtype=dt, device=dev)
        A = torch.empty((R, F), dtype=dt, device=dev) if backward else None
        B = torch.empty((R, F), dtype=dt, device=dev) if backward else None

        def gate_up():
            if backward:
                moe.moe_grouped_gate_up_save(Xe, W1, W3, rt.offsets, H, A, B)
            else:
                moe.moe_grouped_gate_up(Xe, W1, W3, rt.offsets, H=H)

        if backward:
            # the router backward reads Ye unscaled: gates in the combine
            fns = [("route", route),
                   ("dispatch", lambda: moe.moe_dispatch(x, rt.slot, out=Xe)),
                   ("gate_up", gate_up),
                   ("down", lambda: moe.moe_grouped_down(H, W2, rt.offsets, Ye=Ye)),
                   ("combine", lambda: moe.moe_combine(Ye, rt.slot, rt.gate, out=out))]
        else:
            # as moe_layer_fwd runs it: the gates in the down GEMM's epilogue
            row_gate = torch.empty(R, dtype=torch.float32, device=dev)
            fns = [("route", route),
                   ("dispatch", lambda: moe.moe_dispatch_gate(x, rt.slot, rt.gate, out=Xe,
                                                              row_gate=row_gate)),
                   ("gate_up", gate_up),
                   ("down", lambda: moe.moe_grouped_down_gated(H, W2, rt.offsets, row_gate,
                                                               Ye=Ye)),
                   ("combine", lambda: moe.moe_combine(Ye, rt.slot, None, out=out))]
        sx, sw, sh = es, es, es
        if backward:
            dOut = inp["dOut"]
            dYe = torch.empty((R, d), dtype=dt, device=dev)
            grads = moe.ExpertGrads(dXe=torch.empty((R, d), dtype=dt, device=dev),
                                    dW1=torch.empty((E, F, d), dtype=dt, device=dev),
                                    dW3=torch.empty((E, F, d), dtype=dt, device=dev),
                                    dW2=torch.empty((E, d, F), dtype=dt, device=dev),
                                    dA=torch.empty((R, F), dtype=dt, device=dev),
                                    dB=torch.empty((R, F), dtype=dt, device=dev))
            dx = torch.empty((T, d), dtype=dt, device=dev)
            fns += [("bwd_dispatch", lambda: moe.moe_dispatch(dOut, rt.slot, gate=rt.gate, out=dYe)),
                    ("bwd_gemms", lambda: moe.moe_grouped_swiglu_bwd(Xe, A, B, H, dYe, W1, W3, W2,
                                                                     rt.offsets, out=grads)),
                    ("bwd_combine", lambda: moe.moe_combine(grads.dXe, rt.slot, None, out=dx))]
            # router backward: the load-balancing loss (coefficient 0.01, the
            # OLMoE default), the gates through the softmax, and the router
            # GEMM when the logits come from x and Wr
            lg_src = rt.logits if use_router else logits
            aux = torch.empty(1, dtype=torch.float32, device=dev)
            aux_ws = torch.empty(moe.lib.moe_aux_loss_workspace_size(T, E), dtype=torch.uint8,
                                 device=dev)
            rg = moe.RouterGrads(dgate=torch.empty((T, k), dtype=torch.float32, device=dev),
                                 dlogits=torch.empty((T, E), dtype=torch.float32, device=dev))
            fns += [("aux_loss", lambda: moe.moe_aux_loss(lg_src, rt.counts, out=aux,
                                                          workspace=aux_ws)),
                    ("router_bwd", lambda: moe.moe_router_bwd(
                        dOut, Ye, rt.slot, rt.idx, lg_src, rt.counts, aux_coef=0.01,
                        dgate=rg.dgate, dlogits=rg.dlogits))]
            if use_router:
                dWr = torch.empty((E, d), dtype=dt, device=dev)
                lin_ws = torch.empty(moe.lib.moe_router_linear_bwd_workspace_size(T, d, E),
                                     dtype=torch.uint8, device=dev)
                fns += [("router_linear_bwd", lambda: moe.moe_router_linear_bwd(
                    rg.dlogits, x, Wr, dx=dx, dWr=dWr, workspace=lin_ws))]

    def step(ev=None):
        for j, (_, fn) in enumerate(fns):
            if ev is not None:
                ev[j].record()
            fn()
        if ev is not None:
            ev[len(fns)].record()

    step()
    torch.cuda.synchronize(dev)
    e_act = int((rt.counts > 0).sum().item())
    wbytes = e_act * F * d * sw
    # the bf16/fp32 forward alone carries the gates from the dispatch (which
    # records them per row) through the down epilogue, not to the combine
    gated = not backward and not w.mxfp8
    work = {
        "route": (0.0, T * (d * es if use_router else E * 4) + R * 12),
        "dispatch": (0.0, T * d * es + R * d * sx + R * 4 + (R * 8 if gated else 0)),
        "gate_up": (4.0 * R * d * F, R * d * sx + 2 * wbytes + R * F * sh),
        "down": (2.0 * R * d * F, R * F * sh + wbytes + R * d * 2 + (R * 4 if gated else 0)),
        "combine": (0.0, R * d * 2 + T * d * 2 + (R * 4 if gated else R * 8)),
    }
    if backward and w.mxfp8:
        q8 = 1 + 1 / 32  # an E4M3 code and its share of a scale byte
        wq = e_act * F * d * q8
        work["bwd_dispatch"] = (0.0, T * d * 2 + R * d * 2 + R * 8 + R * d * 2 + R * d * q8)
        work["bwd_dH"] = (2.0 * R * d * F, R * d * q8 + wq + R * F * 2)
        work["bwd_swiglu"] = (0.0, 3 * R * F * 2 + 2 * R * F * 2 + 2 * R * F * q8)
        work["bwd_dX"] = (4.0 * R * d * F, 2 * R * F * q8 + 2 * wq + R * d * 2)
        work["bwd_combine"] = (0.0, R * d * 2 + T * d * 2 + R * 4)
        work["bwd_dequant"] = (0.0, R * (d + F) * q8 + R * (d + F) * 2)
        work["bwd_dW"] = (6.0 * R * d * F, 3 * e_act * F * d * 2 + R * (3 * d + 3 * F) * 2)
        work["aux_loss"] = (0.0, T * E * 4 + E * 4)
        work["router_bwd"] = (0.0, T * d * 2 + R * d * 2 + 2 * T * E * 4 + 3 * R * 4)
    elif backward:
        work["bwd_dispatch"] = (0.0, T * d * es + R * d * es + R * 8)
        work["bwd_gemms"] = (12.0 * R * d * F, 6 * wbytes + R * (5 * d + 5 * F) * es)
        work["bwd_combine"] = (0.0, R * d * es + T * d * es + R * 4)
        work["aux_loss"] = (0.0, T * E * 4 + E * 4)
        work["router_bwd"] = (0.0, T * d * es + R * d * es + 2 * T * E * 4 + 3 * R * 4)
        # dx += dlogits Wr and dWr = dlogits^T x: two T x E x d products
        work["router_linear_bwd"] = (4.0 * T * E * d, T * E * 4 + E * d * es + 3 * T * d * es
                                     + E * d * es)
    # backward: bf16 dispatch 1 + GEMMs 5 + combine 1; MXFP8 dispatch,
    # quantise, pack 3 + dH 1 + SwiGLU, pack 2 + dX 1 + combine 1 +
    # dequantise, unpack, dequantise 3 + dW 3; then the aux loss 2 (partial
    # sums, final sum) and the router backward 2 (gate gradients, softmax
    # backward), + 4 for the router GEMM backward (dlogits to bf16, dx, dWr
    # chunk partials, their ordered sum; the bf16 router workloads)
    bwd_kernels = (14 if w.mxfp8 else 7) + 2 + 2 + (4 if use_router else 0)
    # route: (tensor-core logits, fixed-order refinement) + top-k, scan,
    # finalize
    kernels = ((5 if use_router else 3) + (5 if w.mxfp8 else 4)
               + (bwd_kernels if backward else 0))
    return [n for n, _ in fns], step, kernels, work, e_act


def _workload(name, args):
    w = WORKLOADS[name]
    if args.shrink > 1:
        # the same shape per expert (T and E divided together) on a smaller
        # problem, for profiler captures that must stay small
        w = w.scaled(name=f"{w.name}/shrink{args.shrink}", T=max(1, w.T // args.shrink),
                     E=max(w.k, w.E // args.shrink))
    if args.backward and not w.mxfp8 and w.dtype != "bf16":
        raise SystemExit("--backward runs on the bf16 and MXFP8 workloads")
    if args.backward and not w.backward:
        w = w.scaled(name=w.name, backward=True)  # adds the upstream gradient dOut
    return w


def _measure(moe, w, args, rank, world, local, dev, full: bool):
    """Warm up, time K steps of workload ``w`` (graph replay, else eager) and,
    when ``full``, the clocks and the end-to-end run. Returns the raw
    figures; the caller turns them into the JSON line."""
    backward = bool(args.backward)
    inp = make_inputs(w, dev)
    parts, step, kernels_per_step, work, e_act = _steps(moe, w, inp, dev, backward)

    sampler = ClockSampler(local) if (full and rank == 0 and not args.no_clocks) else None
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if moe.moe_get_status() != 0:
        raise RuntimeError("device status word set during warm-up")

    # Timed region: the K steps captured once in a CUDA graph, with CUDA events
    # between the parts of every step captured too (external events become
    # event-record nodes), and the graph replayed once after an untimed warm
    # replay. The library's calls are stream-ordered launches with no host
    # synchronisation or allocation, so a replay runs exactly the eager
    # launches without the per-call host overhead, and the part times come
    # from the timed region itself. K eager steps follow (ms_per_step_eager);
    # with --no-graph, or if any rank fails to capture, they are the timed
    # region.
    def make_events():
        return [[torch.cuda.Event(enable_timing=True, external=True)
                 for _ in range(len(parts) + 1)] for _ in range(args.steps)]

    evs = make_events()
    graph, ms_graph = None, None
    if not args.no_graph:
        graph = _capture_step(lambda: [step(evs[i]) for i in range(args.steps)], dev)
        if max_over_ranks(0.0 if graph is not None else 1.0, world, dev) > 0:
            graph = None
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    per = None
    w0 = w1 = None
    if graph is not None:
        graph.replay()  # untimed: the K captured steps once more
        torch.cuda.synchronize(dev)
        barrier(world)
        torch.cuda.synchronize(dev)
        w0 = time.monotonic()
        start.record()
        graph.replay()
        end.record()
        torch.cuda.synchronize(dev)
        w1 = time.monotonic()
        barrier(world)
        ms_graph = max_over_ranks(start.elapsed_time(end), world, dev)
        per = {p: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
               for j, p in enumerate(parts)}
        del graph

    evs_e = make_events()
    barrier(world)
    torch.cuda.synchronize(dev)
    e0 = time.monotonic()
    start.record()
    for i in range(args.steps):
        step(evs_e[i])
    end.record()
    torch.cuda.synchronize(dev)
    e1 = time.monotonic()
    barrier(world)
    ms_eager = max_over_ranks(start.elapsed_time(end), world, dev)
    if ms_graph is None:
        ms_total, launch = ms_eager, "eager (one host call per library entry)"
        w0, w1 = e0, e1
        per = {p: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs_e)
               for j, p in enumerate(parts)}
    else:
        ms_total = ms_graph
        launch = "CUDA graph of the K steps (same library calls), replayed once"

    # clocks: the timed window; if it held too few samples, keep running
    # untimed steps of the same workload while sampling
    clocks = None
    if sampler is not None:
        lines = sampler.window(w0, w1)
        extra_s = 0.0
        if len(lines) < 10:
            t_ext0 = time.monotonic()
            while time.monotonic() - t_ext0 < 1.0:
                for _ in range(5):
                    step()
                torch.cuda.synchronize(dev)
            extra_s = time.monotonic() - t_ext0
            lines = sampler.window(w0, time.monotonic())
        clocks = ClockSampler.summarize(lines)
        if clocks is not None and extra_s:
            clocks["note"] = f"timed window plus {extra_s:.1f} s of untimed steps of the same workload"

    # end to end through the public layer calls with host buffers
    e2e = None
    if full and not args.no_e2e:
        e2e = _e2e(moe, w, inp, dev, world, args, backward)

    if moe.moe_get_status() != 0:
        raise RuntimeError("device status word set during the timed region")
    if sampler is not None:
        sampler.stop()
    inp_cpu = ({kk: v.cpu() for kk, v in inp.items()}
               if full and rank == 0 and world == 1 and not args.no_cpu_baseline else None)
    return dict(parts=parts, per=per, work=work, e_act=e_act, ms_total=ms_total,
                ms_eager=ms_eager, launch=launch, clocks=clocks, e2e=e2e,
                kernels_per_step=kernels_per_step, inp_cpu=inp_cpu)


def _rates(w, m):
    """Per-part rates, the roofline of the dominant GEMM and the HBM
    fractions of dispatch and combine."""
    parts, per, work = m["parts"], m["per"], m["work"]
    peaks, peak_src = measured_peaks()
    hbm = peaks["hbm_gbs"]
    bf16_tf = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    peak_tf = bf16_tf * (2.0 if w.mxfp8 else 1.0)
    tf_src = (f"{peak_src} bf16 sustained x 2 (dense FP8/BF16 nominal ratio 4.5/2.25)" if w.mxfp8
              else f"{peak_src} bf16 sustained (kernel timed inside a long step)")
    rates = {}
    for p in parts:
        flop, byts = work[p]
        t = per[p] / 1e3
        rates[p] = {"ms": per[p], "gbs": byts / t / 1e9}
        if flop:
            rates[p]["tflops"] = flop / t / 1e12
            rates[p]["intensity_flop_per_byte"] = flop / byts
    gemm_parts = [p for p in parts if work[p][0] > 0]
    dom = max(gemm_parts, key=lambda p: per[p])
    flop, byts = work[dom]
    roof_tf, roof_src = peak_tf, tf_src
    if dom == "bwd_dW":  # bf16 GEMMs inside the MXFP8 backward
        roof_tf = bf16_tf
        roof_src = f"{peak_src} bf16 sustained (kernel timed inside a long step)"
    ridge = roof_tf * 1e12 / (hbm * 1e9)
    if flop / byts >= ridge:
        roof = {"bound": "tensor", "achieved": rates[dom]["tflops"], "peak": roof_tf,
                "unit": "TFLOP/s", "frac": rates[dom]["tflops"] / roof_tf,
                "peak_source": roof_src, "algorithmic_per_launch": f"{flop:.4g} flop"}
    else:
        roof = {"bound": "hbm", "achieved": rates[dom]["gbs"], "peak": hbm, "unit": "GB/s",
                "frac": rates[dom]["gbs"] / hbm, "peak_source": f"{peak_src} HBM copy bandwidth",
                "algorithmic_per_launch": f"{byts:.4g} bytes (operands once, outputs once)"}
    roof["kernel"] = {"gate_up": "grouped gate_up GEMM + SwiGLU (tcgen05)",
                      "down": "grouped down GEMM (tcgen05)",
                      "bwd_gemms": "grouped backward GEMMs dH/dX/dW (tcgen05)",
                      "bwd_dH": "MXFP8 grouped dH GEMM (tcgen05 block-scaled)",
                      "bwd_dX": "MXFP8 grouped dX GEMM (tcgen05 block-scaled)",
                      "bwd_dW": "bf16 weight-gradient GEMMs (tcgen05)",
                      "router_linear_bwd": "router GEMM backward (CUDA cores)"}[dom]
    roof["ridge_flop_per_byte"] = ridge
    roof["traffic"] = recorded_traffic(dom, w.name)
    ffn_t = (per["gate_up"] + per["down"]) / 1e3
    ffn_tf = (work["gate_up"][0] + work["down"][0]) / ffn_t / 1e12
    grouped = {"ffn_tflops": ffn_tf, "ffn_frac_of_peak": ffn_tf / peak_tf,
               "peak_tflops": peak_tf, "experts_with_rows": m["e_act"]}
    hbm_fr = {"dispatch_frac": rates["dispatch"]["gbs"] / hbm,
              "combine_frac": rates["combine"]["gbs"] / hbm, "peak_gbs": hbm}
    return rates, roof, grouped, hbm_fr


def run_ours(args):
    rank, world, local = dist_env()
    dist_init(world, "nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from dropless_top_mixture_b200 import moe

    w = _workload(args.workload, args)
    backward = bool(args.backward)
    m = _measure(moe, w, args, rank, world, local, dev, full=True)
    # a second workload, device-timed only (the same step, K and W)
    also = {}
    for name in ([] if args.also in ("", "none") else args.also.split(",")):
        if name == args.workload:
            continue
        wa = _workload(name, args)
        ma = _measure(moe, wa, args, rank, world, local, dev, full=False)
        also[wa.name] = (wa, ma)
    if rank != 0:
        return 0

    ms_step = m["ms_total"] / args.steps
    value = w.T * world * args.steps / (m["ms_total"] / 1e3)
    rates, roof, grouped, hbm_fr = _rates(w, m)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if w.mxfp8 else ("bf16" if w.dtype == "bf16" else "f32"),
        "data": "synthetic", "config": config_of(w, world, backward), "roofline": roof,
        "breakdown": rates, "grouped_gemm": grouped, "hbm": hbm_fr,
        "e2e": m["e2e"], "gpu_launches": m["kernels_per_step"] * args.steps,
        "clocks": m["clocks"], "launch": m["launch"],
        "ms_per_step_eager": m["ms_eager"] / args.steps,
    }
    if also:
        line["also"] = {}
        for name, (wa, ma) in also.items():
            ra, rfa, ga, ha = _rates(wa, ma)
            line["also"][name] = {
                "value": wa.T * world * args.steps / (ma["ms_total"] / 1e3), "unit": UNIT,
                "ms_per_step": ma["ms_total"] / args.steps, "config": config_of(wa, world, backward),
                "roofline": rfa, "breakdown": ra, "grouped_gemm": ga, "hbm": ha,
                "gpu_launches": ma["kernels_per_step"] * args.steps, "launch": ma["launch"],
                "note": "device-timed like the headline, in the same run; no e2e or CPU baseline"}
            line["gpu_launches"] += ma["kernels_per_step"] * args.steps
            line["gpu_launches_note"] = ("headline steps plus the steps of the workloads under "
                                         "'also', each timed in its own region")
    if m["inp_cpu"] is not None:
        line["cpu_baseline"] = cpu_baseline(w, m["inp_cpu"], backward=backward)
        line["cpu_baseline_one_thread"] = cpu_baseline(w, m["inp_cpu"], backward=backward,
                                                       threads=1)
    else:
        line["cpu_baseline"] = None
    print(json.dumps(line), flush=True)
    return 0


def _capture_step(step, dev):
    """`step` captured in a CUDA graph (after a warm call on the capture
    stream), or None if capture is not possible here."""
    try:
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            step()
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        torch.cuda.synchronize(dev)
        return g
    except RuntimeError as ex:
        print(f"bench: CUDA graph capture failed ({ex}); timing eager steps", file=sys.stderr)
        return None


def _e2e(moe, w, inp, dev, world, args, backward):
    """Same metric through the public layer calls, with the step's inputs
    copied from pinned host memory and its result copied back, per step."""
    T, k = w.T, w.k
    x, Wr, logits = inp["x"], inp.get("Wr"), inp.get("logits")
    W1, W3, W2 = inp["W1"], inp["W3"], inp["W2"]
    x_h = x.cpu().pin_memory()
    lg_h = logits.cpu().pin_memory() if logits is not None else None
    x_d = torch.empty_like(x)
    lg_d = torch.empty_like(logits) if logits is not None else None
    h2d = x.numel() * x.element_size() + (logits.numel() * 4 if logits is not None else 0)
    if args.e2e_chunks <= 0:
        wbytes = 3 * w.E * w.F * w.d * (1 if w.mxfp8 else x.element_size())
        args.e2e_chunks = moe.choose_chunks(T, w.d, x.element_size(), wbytes)
    if w.mxfp8 and backward:
        dO_h = inp["dOut"].cpu().pin_memory()
        dO_d = torch.empty_like(inp["dOut"])
        h2d += dO_d.numel() * dO_d.element_size()
        mw = moe.mxfp8_quantize_weights(W1, W3, W2)
        wb = moe.mxfp8_quantize_weights_bwd(W1, W3, W2)
        lo = moe.moe_layer_fwd_mxfp8(x, k, mw, logits=logits, Wr=Wr, save=True)
        gr = moe.moe_layer_bwd_mxfp8(lo, inp["dOut"], k, wb)
        res = gr.dx

        def run():
            dO_d.copy_(dO_h, non_blocking=True)
            moe.moe_layer_fwd_mxfp8(x_d, k, mw, logits=lg_d, Wr=Wr, out=lo, save=True)
            moe.moe_layer_bwd_mxfp8(lo, dO_d, k, wb, out=gr)
    elif w.mxfp8:
        # token slices whose copies overlap the compute (moe_layer_fwd_mxfp8_host)
        mw = moe.mxfp8_quantize_weights(W1, W3, W2)
        hlm = moe.HostLayerMxfp8(T, w.d, w.E, w.F, k, dev, logits_given=logits is not None,
                                 chunks=args.e2e_chunks)
        res = hlm.res.out
    elif backward:
        dO_h = inp["dOut"].cpu().pin_memory()
        dO_d = torch.empty_like(inp["dOut"])
        h2d += dO_d.numel() * dO_d.element_size()
        lo = moe.moe_layer_fwd(x, k, W1, W3, W2, logits=logits, Wr=Wr, save=True)
        gr = moe.moe_layer_bwd(lo, inp["dOut"], k, W1, W3, W2)
        res = gr.dx

        def run():
            dO_d.copy_(dO_h, non_blocking=True)
            moe.moe_layer_fwd(x_d, k, W1, W3, W2, logits=lg_d, Wr=Wr, out=lo, save=True)
            moe.moe_layer_bwd(lo, dO_d, k, W1, W3, W2, out=gr)
    else:
        # token slices whose copies overlap the compute (moe_layer_fwd_host)
        hl = moe.HostLayer(T, w.d, w.E, w.F, k, x.dtype, dev, logits_given=logits is not None,
                           chunks=args.e2e_chunks)
        res = hl.res.out
    res_h = torch.empty(res.shape, dtype=res.dtype).pin_memory()

    if w.mxfp8 and not backward:
        def e2e_step():
            hlm(x_h, mw, logits_host=lg_h, Wr=Wr, out_host=res_h)
    elif not backward:
        def e2e_step():
            hl(x_h, W1, W3, W2, logits_host=lg_h, Wr=Wr, out_host=res_h)
    else:
        def e2e_step():
            x_d.copy_(x_h, non_blocking=True)
            if lg_d is not None:
                lg_d.copy_(lg_h, non_blocking=True)
            run()
            res_h.copy_(res, non_blocking=True)

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
    r = {"value": T * world * args.steps / (ms_e2e / 1e3), "unit": UNIT,
         "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": res.numel() * res.element_size()}
    if not backward:
        r["pipeline_chunks"] = args.e2e_chunks
    return r


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--also", default=ALSO_WORKLOAD,
                    help="comma-separated workloads also timed (device only) into the 'also' key; "
                         "'none' to skip")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=64,
                    help="tokens per step of the CPU-oracle reference arm")
    ap.add_argument("--backward", action="store_true",
                    help="time forward + backward (bf16 workloads; the fine-grained workload's pass)")
    ap.add_argument("--shrink", type=int, default=1,
                    help="divide T and E by this factor (profiling a small case of the same shape)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager steps instead of replays of one captured step")
    ap.add_argument("--e2e-chunks", type=int, default=0,
                    help="token slices of the host-buffer forward (copies overlap compute); "
                         "0 = chosen from the copy and weight-streaming times (moe.choose_chunks)")
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
