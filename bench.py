#!/usr/bin/env python
"""MoE layer forward+backward throughput on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload dsv3] [--impl moe|reference]

One step = one forward + one backward of the whole layer (router GEMM, top-k
gating, histogram/scan, stable scatter + dispatch, grouped gate/up GEMM with
SwiGLU, grouped down GEMM with the gate multiply, combine; reverse-combine,
dgrad with the SwiGLU backward and router-gate gradient, router backward,
dgrad gate/up, reverse-dispatch, wgrad) over one batch of synthetic tokens.

* value: tokens/s over all ranks, inputs resident in HBM, CUDA-event timed on
  the launch stream, max over ranks.  The expert weights (>= 22 GB) exceed
  L2 and are streamed every step, so no explicit L2 flush is needed.
* e2e: the same steps through the C ABI from pinned HOST buffers: X and dY
  copied in, Y and dX copied out, inside the timed region.
* roofline: the kernel with the largest share of the timed region, its
  algorithmic bytes per launch / its CUDA-event duration, against the
  measured HBM copy bandwidth.
* cpu_baseline: the fp64 CPU oracle on a bounded sample of the workload.
* --impl reference: times that oracle alone, as the comparison arm.

Multi-GPU (torchrun, N > 1): N independent replicas of the single-GPU layer
(weak scaling, no data-path collective); only the timing is reduced (max).
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

import torch  # noqa: E402

from mixture_experts_layer_27_b200 import inputs as IN  # noqa: E402

METRIC = "MoE layer fwd+bwd tokens/s and TFLOP/s (% of B200 BF16/FP8 tensor peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


def measure_mxfp8_peak(dev, seconds: float = 2.0) -> dict:
    """Dense MXFP8 tensor throughput of this GPU: cuBLAS block-scaled E4M3 GEMM (torch._scaled_mm
    with one E8M0 scale per 1x32 block), 8192^3, 2 N^3 FLOPs per call.  Burst = best single call;
    sustained = back to back for `seconds`.  A measurement of the denominator only."""
    n = 8192
    try:
        g = torch.Generator(device=dev).manual_seed(0)
        a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
        bt = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
        one = torch.full((n * (n // 32),), 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)

        def f():
            return torch._scaled_mm(a, bt.t(), one, one, out_dtype=torch.bfloat16)

        for _ in range(3):
            f()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1) / 1e3)
        flop = 2.0 * n ** 3
        calls = max(1, int(seconds / best))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(calls):
            f()
        e1.record()
        torch.cuda.synchronize()
        sus = flop * calls / (e0.elapsed_time(e1) / 1e3) / 1e12
        del a, bt, one
        torch.cuda.empty_cache()
        return {"burst_tflops": flop / best / 1e12, "sustained_tflops": sus,
                "how": f"torch._scaled_mm e4m3 x e4m3, e8m0 1x32 scales, {n}^3: best of 10 and {calls} back to back"}
    except Exception as ex:  # this torch or cuBLAS may lack block-scaled fp8
        return {"unavailable": f"{type(ex).__name__}: {ex}"[:200]}


# the grouped GEMMs that run on block-scaled fp8 tensor cores in MXFP8 mode
MX_GEMMS = ("gemm_gateup_swiglu", "gemm_down_combw", "gemm_dgrad_down_swiglu_bwd", "gemm_dgrad_gateup")


def workload_config(w: IN.Workload) -> dict:
    if w.stream_M:
        routing = (f"{w.El} local experts of {w.E}, each receiving {w.local_tokens} tokens over the stream; "
                   f"{w.stream_M} minibatches x {w.T} tokens through a {w.ring_bytes >> 20} MiB ring")
        l2 = ("no flush: the step streams %.2f GB of tokens (X, dY, the dispatched rows and their "
              "activations) through HBM, far beyond the 126 MB L2" % (4 * w.tokens * w.d * 2 / 1e9))
    else:
        if w.local_tokens:
            routing = (f"{w.El} local experts of {w.E}, each receiving {w.local_tokens} tokens; one batch, "
                       "the dispatched rows held whole (no ring)")
        else:
            routing = "zipf(1.2) bias, hottest ~10x mean" if w.zipf else "near-uniform (W_r ~ N(0, 0.02^2))"
        l2 = ("no flush: expert weights (%.1f GB) exceed the 126 MB L2 and stream every step"
              % (3 * w.El * w.d * w.I * 2 / 1e9))
        if needs_flush(w):
            l2 = "L2 flushed (256 MB write) between timed steps; each step timed on its own"
    prec = "mxfp8" if w.mxfp8 else "bf16"
    return {"workload": f"{w.name}: T={w.tokens} d={w.d} E={w.E} top_k={w.k} I={w.I} {prec}, {routing}",
            "T": w.tokens, "d": w.d, "E": w.E, "top_k": w.k, "I": w.I, "precision": "mxfp8" if w.mxfp8 else "bf16",
            "seed": w.seed, "l2": l2, "parallelism": "replicas"}


def run_config(w: IN.Workload, args) -> dict:
    """The `config` of both arms' lines: the workload, the gradient dtype and how the GEMM pairs are
    launched (the ring-streamed layer always runs them as persistent pairs)."""
    cfg = dict(workload_config(w), wgrad_dtype="fp32" if args.wgrad_fp32 else "bf16",
               forward="persistent" if args.persistent or (w.stream_M and not w.mxfp8) else "launches")
    if w.mxfp8:  # the weight-gradient GEMMs: MXFP8 operands along the rows, or the bf16 operands
        cfg["wgrad_gemms"] = "mxfp8" if getattr(args, "mx_wgrad", False) else "bf16"
    return cfg


L2_BYTES = 126 << 20


def needs_flush(w: IN.Workload) -> bool:
    """Workloads whose weights and tokens fit in L2 flush it between timed steps."""
    return 3 * w.El * w.d * w.I * 2 + 2 * w.tokens * w.d * 2 < 2 * L2_BYTES


def local_rows(w: IN.Workload) -> int:
    return w.El * w.local_tokens if w.local_tokens else w.tokens * w.k


def algorithmic_flops(w: IN.Workload) -> dict:
    rows, dI = local_rows(w), w.d * w.I
    return {"gemm_gateup_swiglu": 4 * dI * rows, "gemm_down_combw": 2 * dI * rows,
            "gemm_dgrad_down_swiglu_bwd": 2 * dI * rows, "gemm_dgrad_gateup": 4 * dI * rows,
            "gemm_wgrad_gateup": 4 * dI * rows, "gemm_wgrad_down": 2 * dI * rows,
            "gemm_wgrad_gateup_mx": 4 * dI * rows, "gemm_wgrad_down_mx": 2 * dI * rows,
            "router_logits": 2 * w.tokens * w.d * w.E,
            "gemm_gateup_down_persistent": 6 * dI * rows,  # gate/up and down in one launch
            "gemm_dgrads_persistent": 6 * dI * rows,  # both dgrads in one launch
            # dW_r = X^T dl; the kernel issues it twice (the hi and lo bf16 terms of dl)
            "router_wgrad": 2 * w.tokens * w.d * w.E}


# ----------------------------------------------------------------------------
# algorithmic bytes per launch of each kernel (minimum HBM traffic of its job)
# rows = T*k routed assignments; weights of all local experts; bf16 = 2 bytes
# ----------------------------------------------------------------------------
def algorithmic_bytes(w: IN.Workload, wgrad_elem_bytes: int = 2, mx_wgrad: bool = False) -> dict:
    T, d, E, I, k, El = w.tokens, w.d, w.E, w.I, w.k, w.El
    rows = local_rows(w)
    # token rows a gather reads: every token once, or in an expert slice at most one per local row
    Tg = min(T, rows)
    W1 = El * d * I * 2  # one expert weight matrix family (gate, up or down), bytes
    G1 = El * d * I * wgrad_elem_bytes  # its gradient (bf16, or fp32 with --wgrad-fp32)
    if w.mxfp8:
        # fp8 operands carry one scale byte per 32 values; outputs stay bf16 (H, dA, dB also as fp8)
        Wq = El * d * I * 33 // 32
        return {
            "router_logits": T * d * 2 + d * E * 2 + T * E * 4,
            "topk_gating": T * E * 4 + rows * 8,
            # X once, then bf16 rows and fp8 along d; or (mx_wgrad) fp8 along d and along the rows
            "dispatch": Tg * d * 2 + (2 * rows * d * 33 // 32 if mx_wgrad else rows * d * 2 + rows * d * 33 // 32),
            "gemm_gateup_swiglu": 2 * Wq + rows * d * 33 // 32 + 2 * rows * I * 2 + rows * I * 33 // 32,
            "gemm_down_combw": Wq + rows * I * 33 // 32 + rows * d * 2,
            "combine": rows * d * 2 + T * d * 2,
            "reverse_combine": Tg * d * 2 + (2 * rows * d * 33 // 32 if mx_wgrad else rows * d * 2 + rows * d * 33 // 32),
            # dA, dB, Hg out in bf16 for the bf16 weight gradients, or (mx_wgrad) as fp8 along the rows
            "gemm_dgrad_down_swiglu_bwd": Wq + rows * d * 33 // 32 + 2 * rows * I * 2
            + (3 * rows * I * 33 // 32 if mx_wgrad else 3 * rows * I * 2) + 2 * rows * I * 33 // 32,
            "router_wgrad": T * d * 2 + T * k * 8 + d * E * 4,
            "gemm_dgrad_gateup": 2 * Wq + 2 * rows * I * 33 // 32 + rows * d * 2,
            "reverse_dispatch": rows * d * 2 + T * d * 2 + E * d * 2,
            "gemm_wgrad_gateup": rows * d * 2 + 2 * rows * I * 2 + 2 * G1,
            "gemm_wgrad_down": rows * I * 2 + rows * d * 2 + G1,
            # MXFP8 weight gradients: the two GEMMs on the operands quantised along the rows (by the
            # dispatch, the reverse-combine and the dgrad of W_down)
            "gemm_wgrad_gateup_mx": (rows * d + 2 * rows * I) * 33 // 32 + 2 * G1,
            "gemm_wgrad_down_mx": (rows * I + rows * d) * 33 // 32 + G1,
        }
    return {
        "router_logits": T * d * 2 + d * E * 2 + T * E * 4,
        "topk_gating": T * E * 4 + rows * 8,
        "dispatch": Tg * d * 2 + rows * d * 2,
        "gemm_gateup_swiglu": 2 * W1 + rows * d * 2 + 3 * rows * I * 2,
        "gemm_down_combw": W1 + rows * I * 2 + rows * d * 2,
        "combine": rows * d * 2 + T * d * 2,
        "reverse_combine": Tg * d * 2 + rows * d * 2,
        "gemm_dgrad_down_swiglu_bwd": W1 + rows * d * 2 + 2 * rows * I * 2 + 3 * rows * I * 2,
        "router_wgrad": T * d * 2 + T * k * 8 + d * E * 4,  # X once, dl and ids, dW_r
        "gemm_dgrad_gateup": 2 * W1 + 2 * rows * I * 2 + rows * d * 2,
        "reverse_dispatch": rows * d * 2 + T * d * 2 + E * d * 2,
        "gemm_wgrad_gateup": rows * d * 2 + 2 * rows * I * 2 + 2 * G1,
        "gemm_wgrad_down": rows * I * 2 + rows * d * 2 + G1,
        # gate/up and down in one launch: the weights, X_perm in, A and B (saved) and O' out;
        # H passes between two tiles of the launch and is not counted
        "gemm_gateup_down_persistent": 3 * W1 + rows * d * 2 + 2 * rows * I * 2 + rows * d * 2,
        # both dgrads in one launch: the weights, dY_perm, A and B in; dA, dB, Hg and dX_perm out
        # (dA, dB read back by the dgrad of gate/up within the launch are not counted again)
        "gemm_dgrads_persistent": 3 * W1 + rows * d * 2 + 2 * rows * I * 2 + 3 * rows * I * 2 + rows * d * 2,
    }


# DRAM bytes per launch measured by ncu (dram__bytes_read.sum + dram__bytes_write.sum) on a
# 16-expert case of the same expert shape, scaled to the workload by the experts processed.
# A figure is reported only while the GEMM sources still hash to the value they had
# when the counters were taken.
NCU_TRAFFIC = {
    ("gemm_dgrads_persistent", "dsv3"): ((1457.578752e6 + 0.988160e6) * 16, "c0eb420bbee705f6"),
    ("gemm_gateup_down_persistent", "dsv3"): ((1442.484480e6 + 5.134336e6) * 16, "c0eb420bbee705f6"),
    ("gemm_wgrad_gateup", "dsv3"): ((34.699264e6 + 875.961088e6) * 16, "c0eb420bbee705f6"),
}
GEMM_SOURCES = ("gemm.cu", "ptx.cuh", "moe_internal.cuh")


def gemm_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for n in GEMM_SOURCES:
        with open(os.path.join(ROOT, "mixture_experts_layer_27_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    t = NCU_TRAFFIC.get((kernel, workload))
    if t is None or t[1] != gemm_source_hash():
        return None
    return t[0]


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        try:
            self.dev = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.dev = str(device.index or 0)
        self.proc = None
        self.path = os.path.join("/tmp", f"moe_clocks_{os.getpid()}_{device.index or 0}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.dev)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = max((num(r[2]) for r in rows if num(r[2]) is not None), default=None)
        loaded = [r for r in rows if (num(r[3]) or 0) > 250] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(4) if r[5 + i].lower().startswith("active")})
        sm_load = [num(r[1]) for r in loaded if num(r[1]) is not None]
        return {"sm_mhz": statistics.median(sm_load) if sm_load else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max((num(r[3]) or 0) for r in rows)}


# ----------------------------------------------------------------------------
# CPU oracle on a bounded sample (the baseline and the reference arm)
#
# One sample step = the fp64 oracle's forward + backward of the layer restricted to a window of
# ORACLE_WINDOW consecutive local experts (every token routed, then those experts' assignments
# through the SwiGLU experts and back, their weight gradients, the router gradient of their
# tokens).  Its work in token units is the assignments it processed / top_k.  The rate is that
# work over the median measured step time: nothing is extrapolated, and both CPU figures
# (cpu_baseline and the reference arm) use this one sampler.
# ----------------------------------------------------------------------------
ORACLE_WINDOW = 8
CPU_BASELINE_STEPS = 8


def oracle_window(w: IN.Workload) -> tuple:
    """(first local expert index, number) of the sampled window: the middle of the local experts."""
    m = min(ORACLE_WINDOW, w.El)
    return (w.El - m) // 2, m


def oracle_sample(w: IN.Workload, x_cpu: dict) -> tuple:
    """(seconds, assignments) of one oracle fwd+bwd over the sampled expert window: the fp64
    layer, or for MXFP8 workloads the MXFP8 layer (weights rounded once, as the GPU path prepares
    them once per optimiser step, outside the timed step; weight gradients as the run has them)."""
    import numpy as np
    import oracle as O

    def f64(t):
        return t.float().numpy().astype(np.float64)

    e0, m = x_cpu["window"]
    X, Wr, dY = f64(x_cpu["X"]), f64(x_cpu["W_r"]), f64(x_cpu["dY"])
    b = None if x_cpu["bias"] is None else f64(x_cpu["bias"])
    Wg, Wu, Wd = (f64(x_cpu[n]) for n in ("W_gate", "W_up", "W_down"))
    first = w.first_local + e0
    if w.mxfp8 and "mx_layouts" not in x_cpu:
        x_cpu["mx_layouts"] = {first + e: O.mx_weight_layouts(Wg[e], Wu[e], Wd[e]) for e in range(m)}
    t0 = time.perf_counter()
    if w.mxfp8:
        lay = x_cpu["mx_layouts"]
        _, ctx = O.forward_mx(X, Wr, b, lambda e: Wg[e - first], lambda e: Wu[e - first], lambda e: Wd[e - first], w.k,
                              first_local=first, num_local=m, rounded=lay.__getitem__)
        O.backward_mx(ctx, dY, mx_wgrad=x_cpu.get("mx_wgrad", False))
    else:
        _, ctx = O.forward(X, Wr, b, lambda e: Wg[e - first], lambda e: Wu[e - first], lambda e: Wd[e - first], w.k,
                           first_local=first, num_local=m)
        O.backward(ctx, dY)
    dt = time.perf_counter() - t0
    return dt, int(ctx["sched"]["offsets"][-1])


def cpu_inputs(w: IN.Workload, mx_wgrad: bool = False) -> dict:
    """Host copies of the inputs the sample needs (CPU generator; same distributions)."""
    e0, m = oracle_window(w)
    x = {"mx_wgrad": mx_wgrad,
         "X": IN._normal((w.tokens, w.d), 1.0, IN._seed(w.seed, w.name, "X"), "cpu"),
         "W_r": IN._normal((w.d, w.E), 0.02, IN._seed(w.seed, w.name, "W_r"), "cpu"),
         "dY": IN._normal((w.tokens, w.d), 1.0, IN._seed(w.seed, w.name, "dY"), "cpu"), "window": (e0, m)}
    for n in ("W_gate", "W_up", "W_down"):
        x[n] = torch.stack([IN.expert_weights(w, n, w.first_local + e0 + e, "cpu") for e in range(m)])
    if w.zipf:
        x["bias"] = IN.zipf_bias(w, x["X"], x["W_r"])
    elif w.local_tokens:
        x["bias"] = IN.local_load_bias(w, x["X"], x["W_r"])
    else:
        x["bias"] = None
    return x


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_rate(w: IN.Workload, x_cpu: dict, steps: int) -> dict:
    """Times `steps` sample steps; the rate in tokens/s and the per-step times."""
    ts, asg = [], []
    for _ in range(steps):
        dt, a = oracle_sample(w, x_cpu)
        ts.append(dt)
        asg.append(a)
    e0, m = x_cpu["window"]
    med = statistics.median(ts)  # the median step: robust to a step disturbed by other host work
    return {"value": asg[0] / w.k / med, "seconds": ts, "assignments": asg[0],
            "sample": (f"fp64 numpy oracle{' (MXFP8 layer' + (', MX weight gradients' if x_cpu.get('mx_wgrad') else '') + ')' if w.mxfp8 else ''}, "
                       f"measured (no extrapolation): each step routes all {w.tokens} tokens and "
                       f"runs forward + backward of local experts {e0}..{e0 + m - 1} ({asg[0]} of the "
                       f"{w.tokens * w.k if w.El == w.E else 'local'} assignments, weight gradients included); "
                       f"rate = assignments / top_k / the median of {steps} measured steps "
                       f"({med:.2f} s; {min(ts):.2f}-{max(ts):.2f} s)")}


def cpu_baseline(w: IN.Workload, mx_wgrad: bool = False) -> dict:
    x = cpu_inputs(w, mx_wgrad)
    oracle_sample(w, x)  # first call: imports, BLAS start-up
    r = oracle_rate(w, x, CPU_BASELINE_STEPS)
    return {"value": r["value"], "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle", "sample": r["sample"]}


# ----------------------------------------------------------------------------
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(v: float, world: int, device="cuda") -> float:
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, seconds: float, world: int) -> float:
    """Whole-job rate: every rank's units over the slowest rank's time (weak scaling: each rank
    runs the layer on its own tokens, so the per-rank work is fixed as ranks are added)."""
    return units_per_rank * world / seconds


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def run_reference(args, w: IN.Workload, world: int, rank: int):
    if rank != 0:
        return
    x = cpu_inputs(w, args.mx_wgrad)
    if w.nvfp4:  # the NVFP4 oracle forward (its own start-up call inside)
        r = nv_oracle_rate(w, x, args.steps)
        value = r["value"]
        print(json.dumps({
            "metric": METRIC_NV, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": statistics.median(r["seconds"]) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": nv_config(w),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": r["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
            flush=True)
        return
    for _ in range(args.warmup):
        oracle_sample(w, x)
    r = oracle_rate(w, x, args.steps)
    value = r["value"]
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": statistics.median(r["seconds"]) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": run_config(w, args),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": r["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_moe(args, w: IN.Workload, world: int, rank: int, local: int):
    from mixture_experts_layer_27_b200 import binding as B

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    x = IN.make_inputs(w, device=dev)
    wdt = torch.float32 if args.wgrad_fp32 else torch.bfloat16
    if w.mxfp8 and w.stream_M:
        layer = B.MoEStreamMX(w.T, w.d, w.E, w.I, w.k, w.stream_M, w.ring_bytes, w.first_local, w.num_local,
                              device=dev, wgrad_dtype=wdt, mx_wgrad=args.mx_wgrad)
    elif w.mxfp8:
        layer = B.MoELayerMX(w.T, w.d, w.E, w.I, w.k, w.first_local, w.num_local, device=dev, wgrad_dtype=wdt,
                             mx_wgrad=args.mx_wgrad)
    elif w.stream_M:
        layer = B.MoEStream(w.T, w.d, w.E, w.I, w.k, w.stream_M, w.ring_bytes, w.first_local, w.num_local,
                            device=dev, wgrad_dtype=wdt)
    else:
        layer = B.MoELayer(w.T, w.d, w.E, w.I, w.k, first_local_expert=w.first_local, num_local_experts=w.num_local,
                           device=dev, wgrad_dtype=wdt)
    NT = w.tokens
    Y = torch.empty(NT, w.d, dtype=torch.bfloat16, device=dev)
    grads = dict(dX=torch.empty(NT, w.d, dtype=torch.bfloat16, device=dev),
                 dW_gate=torch.empty_like(x["W_gate"], dtype=wdt), dW_up=torch.empty_like(x["W_up"], dtype=wdt),
                 dW_down=torch.empty_like(x["W_down"], dtype=wdt),
                 dW_r=torch.empty(w.d, w.E, dtype=torch.float32, device=dev))
    stream = torch.cuda.current_stream(dev)

    prep_ms = None
    fp8_peak = None
    if w.mxfp8:
        fp8_peak = measure_mxfp8_peak(dev)
        # quantised weights are prepared once per optimiser step, outside the layer step
        layer.prepare(x["W_gate"], x["W_up"], x["W_down"])
        pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        pa.record(stream)
        layer.prepare(x["W_gate"], x["W_up"], x["W_down"])
        pb.record(stream)
        torch.cuda.synchronize()
        prep_ms = pa.elapsed_time(pb)

        def step(X, dY, Yout, g):
            layer.forward(X, x["W_r"], x["bias"], Y=Yout)
            layer.backward(X, x["W_r"], dY, out=g)
    elif args.persistent:
        def step(X, dY, Yout, g):
            layer.forward(X, x["W_r"], x["bias"], x["W_gate"], x["W_up"], x["W_down"], Y=Yout, persistent=True)
            layer.backward(X, x["W_r"], x["W_gate"], x["W_up"], x["W_down"], dY, out=g, persistent=True)
    else:
        def step(X, dY, Yout, g):
            layer.forward(X, x["W_r"], x["bias"], x["W_gate"], x["W_up"], x["W_down"], Y=Yout)
            layer.backward(X, x["W_r"], x["W_gate"], x["W_up"], x["W_down"], dY, out=g)

    for _ in range(args.warmup):
        step(x["X"], x["dY"], Y, grads)
    torch.cuda.synchronize()
    st = layer.error()
    if st != B.MOE_OK:
        raise RuntimeError("device error during warm-up: " + B.status_string(st))

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if needs_flush(w) else None

    # ---------------- per-kernel durations: direct launches, the library's event pairs ----------------
    # (the same K steps as the timed region below, launched one by one so that every kernel is
    # bracketed by CUDA events on its stream; kernel durations do not depend on how it is launched)
    B.moe_profile_read()  # drop anything recorded so far
    B.moe_profile_enable(True)
    launches0 = B.moe_kernel_launches()
    barrier(world)
    torch.cuda.synchronize()
    for _ in range(args.steps):
        if flush is not None:
            flush.fill_(1)
        step(x["X"], x["dY"], Y, grads)
    torch.cuda.synchronize()
    launches_per_step = (B.moe_kernel_launches() - launches0) // args.steps
    B.moe_profile_enable(False)
    prof = B.moe_profile_read()
    st = layer.error()
    if st != B.MOE_OK:
        raise RuntimeError("device error in the per-kernel pass: " + B.status_string(st))

    # ---------------- one step as a CUDA graph ----------------
    # The layer only enqueues work (no host synchronisation, no allocation inside a call), so a
    # whole fwd+bwd step is captured once and replayed: no launch gaps between its kernels.
    graph, launch_mode = None, "cuda_graph"
    if not args.no_graph:
        try:
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                step(x["X"], x["dY"], Y, grads)
            stream.wait_stream(side)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step(x["X"], x["dY"], Y, grads)
            torch.cuda.synchronize()
        except Exception as ex:  # report and fall back to direct launches
            graph, launch_mode = None, f"direct (graph capture failed: {type(ex).__name__})"
    else:
        launch_mode = "direct"

    def run_step():
        if graph is not None:
            graph.replay()
        else:
            step(x["X"], x["dY"], Y, grads)

    for _ in range(2):
        run_step()
    torch.cuda.synchronize()

    # ---------------- device-resident timed region ----------------
    clocks = ClockSampler(dev)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    if flush is not None:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for a, b in evs:
            flush.fill_(1)
            a.record(stream)
            run_step()
            b.record(stream)
        torch.cuda.synchronize()
        t_local = sum(a.elapsed_time(b) for a, b in evs) / 1e3
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            run_step()
        e1.record(stream)
        torch.cuda.synchronize()
        t_local = e0.elapsed_time(e1) / 1e3
    barrier(world)
    clk = clocks.stop()
    launches = launches_per_step * args.steps  # graph replays launch the captured kernels
    st = layer.error()
    if st != B.MOE_OK:
        raise RuntimeError("device error in the timed region: " + B.status_string(st))
    t = max_over_ranks(t_local, world)

    # ---------------- end to end through host buffers ----------------
    hX = torch.empty(NT, w.d, dtype=torch.bfloat16, pin_memory=True)
    hdY = torch.empty_like(hX, pin_memory=True)
    hY = torch.empty_like(hX, pin_memory=True)
    hdX = torch.empty_like(hX, pin_memory=True)
    hX.copy_(x["X"].cpu())
    hdY.copy_(x["dY"].cpu())
    # Two sets of device inputs and outputs; set 0 is the one the graph above reads and writes
    # (the weight gradients, ctx and workspace are shared: steps run one after another on the
    # compute stream).  Each step's host copies run on two copy streams (in and out), so they
    # overlap the neighbouring steps' compute; every step's copies are inside the timed region.
    Xb, dYb, Yb = torch.empty_like(x["X"]), torch.empty_like(x["dY"]), torch.empty_like(Y)
    gb = dict(grads)
    gb["dX"] = torch.empty_like(grads["dX"])
    graph_b = None
    if graph is not None:
        try:
            graph_b = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_b):
                step(Xb, dYb, Yb, gb)
            torch.cuda.synchronize()
        except Exception:
            graph_b = None
    sets = [(x["X"], x["dY"], Y, grads, graph), (Xb, dYb, Yb, gb, graph_b)]
    cs_in, cs_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)  # host->device, device->host
    ev = {n: [torch.cuda.Event(), torch.cuda.Event()] for n in ("h2d", "comp", "d2h")}

    def e2e_run(n):
        cs_in.wait_stream(stream)
        cs_out.wait_stream(stream)
        for i in range(n):
            bi = i % 2
            Xi, dYi, Yi, gi, gr = sets[bi]
            with torch.cuda.stream(cs_in):
                if i >= 2:
                    cs_in.wait_event(ev["comp"][bi])  # step i-2 has finished reading this input set
                Xi.copy_(hX, non_blocking=True)
                dYi.copy_(hdY, non_blocking=True)
                ev["h2d"][bi].record(cs_in)
            stream.wait_event(ev["h2d"][bi])
            if i >= 2:
                stream.wait_event(ev["d2h"][bi])  # step i-2's outputs have left this output set
            if gr is not None:
                gr.replay()
            else:
                step(Xi, dYi, Yi, gi)
            ev["comp"][bi].record(stream)
            with torch.cuda.stream(cs_out):
                cs_out.wait_event(ev["comp"][bi])
                hY.copy_(Yi, non_blocking=True)
                hdX.copy_(gi["dX"], non_blocking=True)
                ev["d2h"][bi].record(cs_out)
        stream.wait_stream(cs_in)
        stream.wait_stream(cs_out)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier(world)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    e2e_run(args.steps)
    e3.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    t_e2e = max_over_ranks(e2.elapsed_time(e3) / 1e3, world)
    st = layer.error()
    if st != B.MOE_OK:
        raise RuntimeError("device error in the e2e region: " + B.status_string(st))

    if rank != 0:
        return
    tokens = NT * args.steps * world
    flops = w.model_flops() * args.steps * world
    value = job_throughput(NT * args.steps, t, world)
    tflops = flops / t / 1e12
    per_gpu_tflops = tflops / world
    algo = algorithmic_bytes(w, 4 if args.wgrad_fp32 else 2, args.mx_wgrad)
    traffic_key = w.name + ("+wgrad_fp32" if args.wgrad_fp32 else "")  # counters were taken with bf16 gradients
    aflops = algorithmic_flops(w)
    if w.El < w.E:
        # in an expert slice the router weight gradient contracts over the tokens with a local
        # assignment only; their number depends on the routing, so no figure is claimed for it
        algo.pop("router_wgrad", None)
        aflops.pop("router_wgrad", None)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    bf16 = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    fp8 = fp8_peak.get("sustained_tflops") if fp8_peak else None
    kern = {}
    for name, (ms, n) in sorted(prof.items(), key=lambda kv: -kv[1][0]):
        steps = args.steps
        e = {"ms_per_step": ms / steps, "launches_per_step": n / steps, "share": ms / (t * 1e3)}
        sec = ms / steps / 1e3  # the kernel's time in one step (all its launches)
        if name in algo:
            e["algorithmic_GB"] = algo[name] / 1e9
            e["achieved_GBs"] = algo[name] / sec / 1e9
        if name in aflops:
            e["achieved_TFLOPs"] = aflops[name] / sec / 1e12
            # the binding resource: the larger of the two times at peak (fp8 peak for MX GEMMs)
            on_fp8 = bool(fp8) and name in MX_GEMMS
            tpeak = fp8 if on_fp8 else bf16
            e["bound"] = "tensor" if aflops[name] / (tpeak * 1e12) > algo.get(name, 0) / (hbm * 1e9) else "hbm"
            if on_fp8:
                e["tensor_peak"] = "mxfp8"
        else:
            e["bound"] = "hbm"
        kern[name] = e
    top = max(kern.items(), key=lambda kv: kv[1]["share"])[0]
    if kern[top]["bound"] == "tensor" and kern[top].get("tensor_peak") == "mxfp8":
        ach = kern[top]["achieved_TFLOPs"]
        roof = {"kernel": top, "bound": "tensor", "achieved": ach, "peak": fp8, "unit": "TFLOP/s",
                "frac": ach / fp8, "traffic": ncu_traffic(top, traffic_key),
                "peak_source": "measured sustained MXFP8 cuBLAS GEMM in this run (" + fp8_peak["how"] + ")"}
    elif kern[top]["bound"] == "tensor":
        ach = kern[top]["achieved_TFLOPs"]
        roof = {"kernel": top, "bound": "tensor", "achieved": ach, "peak": bf16, "unit": "TFLOP/s",
                "frac": ach / bf16, "traffic": ncu_traffic(top, traffic_key),
                "peak_source": "measured sustained bf16 GEMM (MEASURED_PEAKS.json bf16_tflops_sustained)"
                if peak_kind == "measured" else "fallback 1.4 PFLOP/s sustained bf16 (no MEASURED_PEAKS.json)"}
    else:
        ach = kern[top].get("achieved_GBs")
        roof = {"kernel": top, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                "frac": (ach / hbm) if ach else None, "traffic": ncu_traffic(top, traffic_key),
                "peak_source": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, random-init weights)",
        "config": run_config(w, args),
        "tflops": tflops, "pct_of_bf16_peak": 100.0 * per_gpu_tflops / bf16,
        "peak_note": f"bf16 sustained {bf16} TFLOP/s ({peak_kind}); model FLOPs 18 d I T k + 6 T d E per step",
        "roofline": roof,
        "e2e": {"value": job_throughput(NT * args.steps, t_e2e, world), "unit": "tokens/s", "h2d_bytes_per_step": 2 * NT * w.d * 2,
                "d2h_bytes_per_step": 2 * NT * w.d * 2,
                "note": "X, dY copied in from pinned host memory and Y, dX copied back every step, on copy "
                        "streams with double-buffered device inputs and outputs so that a step's copies "
                        "overlap the neighbouring steps' compute; weights and their gradients stay in HBM; "
                        "the compute is launched as in the timed region"},
        "gpu_launches": int(launches),
        "launch": launch_mode,
        "clocks": clk,
        "kernels": kern,
    }
    if prep_ms is not None:
        line["prepare_weights_ms"] = prep_ms
        line["mxfp8_peak"] = fp8_peak
        if fp8:
            line["pct_of_mxfp8_peak"] = 100.0 * per_gpu_tflops / fp8
        wg = ("weight gradients on block-scaled fp8 too (operands quantised along each expert's rows)"
              if args.mx_wgrad else "weight gradients bf16")
        line["peak_note"] += ("; MXFP8: gate/up, down and both dgrads on block-scaled fp8 tensor cores, %s; "
                              "pct_of_mxfp8_peak against the sustained MXFP8 GEMM measured in this run" % wg)
        line["dtype"] = "mxfp8 (e4m3 + e8m0 scales)" + ("" if args.mx_wgrad else " / bf16 wgrad")
    if w.stream_M:
        pl = layer.plan()["plan"]
        line["stream_plan"] = {"macrobatches": int(pl[0]), "backward_chunks": int(pl[1]), "padded_rows": int(pl[2]),
                               "replayed_rows": int(pl[3]), "resident_rows": int(pl[4]), "ring_rows": int(pl[5])}
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.mx_wgrad)
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# NVFP4 layer (moe_fwd_nvfp4 + moe_bwd_nvfp4): a step is one forward + one backward
# ----------------------------------------------------------------------------
METRIC_NV = METRIC
NV_GEMMS = ("gemm_gateup_swiglu_nvfp4", "gemm_down_combw_nvfp4", "gemm_dgrad_down_swiglu_bwd_nvfp4",
            "gemm_dgrad_gateup_nvfp4")


def nv_algorithmic(w: IN.Workload) -> tuple:
    """(bytes, flops) per step of each kernel of the NVFP4 layer: E2M1 codes at 1/2 byte and one
    E4M3 scale per 16 values (9/16 byte per value); H, dA and dB in fp32 between the two passes
    of their quantisation; the router, combine, reverse dispatch and bf16 weight gradients as
    in the bf16 layer."""
    T, d, E, I, k, El = w.tokens, w.d, w.E, w.I, w.k, w.El
    rows = local_rows(w)
    Tg = min(T, rows)
    q = 9 / 16
    W = El * d * I * q  # one weight tensor in NVFP4
    by = algorithmic_bytes(w)
    fl = algorithmic_flops(w)
    by.update({"nvfp4_amax_scale": 2 * T * d * 2,  # X, then dY
               "dispatch": Tg * d * 2 + rows * d * (q + 2),  # codes and the bf16 rows
               "reverse_combine": Tg * d * 2 + rows * d * (q + 2),
               "gemm_gateup_swiglu_nvfp4": 2 * W + rows * d * q + rows * I * (4 + 2 * 2),  # H fp32, A, B bf16
               "nvfp4_quantize_h": rows * I * 4 + rows * I * q,
               "gemm_down_combw_nvfp4": W + rows * I * q + rows * d * 2,
               # dY codes, W_down, A and B in; Hg in bf16, dA and dB in fp32 and dg partials out
               "gemm_dgrad_down_swiglu_bwd_nvfp4": W + rows * d * q + rows * I * (2 * 2 + 2 + 2 * 4)
               + rows * (I // 128) * 4,
               # dA, dB in fp32 in; their codes and their bf16 copies (the weight gradients' operands) out
               "nvfp4_quantize_da_db": 2 * rows * I * (4 + q + 2),
               "gemm_dgrad_gateup_nvfp4": 2 * W + 2 * rows * I * q + rows * d * 2})
    fl.update({"gemm_gateup_swiglu_nvfp4": 4 * d * I * rows, "gemm_down_combw_nvfp4": 2 * d * I * rows,
               "gemm_dgrad_down_swiglu_bwd_nvfp4": 2 * d * I * rows, "gemm_dgrad_gateup_nvfp4": 4 * d * I * rows})
    return by, fl


def nv_config(w: IN.Workload) -> dict:
    cfg = dict(workload_config(w), precision="nvfp4", wgrad_dtype="bf16", wgrad_gemms="bf16")
    cfg["workload"] = cfg["workload"].replace(" bf16,", " nvfp4,")
    return cfg


def nv_oracle_rate(w: IN.Workload, x_cpu: dict, steps: int) -> dict:
    """The NVFP4 oracle forward + backward on the sampled expert window (all tokens routed), timed."""
    import numpy as np
    import oracle.nvfp4 as N

    def f64(t):
        return t.float().numpy().astype(np.float64)

    e0, m = x_cpu["window"]
    X, Wr, dY = f64(x_cpu["X"]), f64(x_cpu["W_r"]), f64(x_cpu["dY"])
    b = None if x_cpu["bias"] is None else f64(x_cpu["bias"])
    Wg, Wu, Wd = (f64(x_cpu[n]) for n in ("W_gate", "W_up", "W_down"))
    first = w.first_local + e0
    gs_w = N.nv_weight_scales(Wg, Wu, Wd)  # over the window's experts
    gs_b = N.nv_weight_scales_bwd(Wg, Wu, Wd)
    # weights rounded once, outside the timed step (the GPU path prepares them once per optimiser step)
    lay = {first + e: N.nv_weight_layouts(Wg[e], Wu[e], Wd[e], gs_w) for e in range(m)}
    lay_b = {first + e: N.nv_weight_layouts_bwd(Wg[e], Wu[e], Wd[e], gs_b) for e in range(m)}
    cg, cu, cd = (lambda e: Wg[e - first]), (lambda e: Wu[e - first]), (lambda e: Wd[e - first])

    def one():
        t0 = time.perf_counter()
        _, info = N.forward_nv(X, Wr, b, cg, cu, cd, w.k, first_local=first, num_local=m, gs_w=gs_w,
                               rounded=lay.__getitem__)
        N.backward_nv(info, X, Wr, cg, cu, cd, dY, gs_bwd=gs_b, rounded=lay_b.__getitem__)
        return time.perf_counter() - t0, int(info["sched"]["offsets"][-1])

    one()  # imports, BLAS start-up
    ts, asg = zip(*[one() for _ in range(steps)])
    med = statistics.median(ts)
    return {"value": asg[0] / w.k / med, "seconds": list(ts),
            "sample": (f"fp64 numpy NVFP4 oracle, measured: each step routes all {w.tokens} tokens and "
                       f"runs forward + backward of local experts {e0}..{e0 + m - 1} ({asg[0]} assignments; weights "
                       f"rounded once outside the step, global scales over the window); rate = assignments / "
                       f"top_k / the median of {steps} steps ({med:.2f} s)")}


def run_nvfp4(args, w: IN.Workload, world: int, rank: int, local: int):
    from mixture_experts_layer_27_b200 import binding as B

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    x = IN.make_inputs(w, device=dev)
    layer = B.MoELayerNVFP4(w.T, w.d, w.E, w.I, w.k, w.first_local, w.num_local, device=dev)
    El = w.El
    Wg, Wu, Wd = (x[n][w.first_local:w.first_local + El].contiguous() for n in ("W_gate", "W_up", "W_down"))
    NT = w.tokens
    Y = torch.empty(NT, w.d, dtype=torch.bfloat16, device=dev)
    grads = dict(dX=torch.empty(NT, w.d, dtype=torch.bfloat16, device=dev), dW_gate=torch.empty_like(Wg),
                 dW_up=torch.empty_like(Wu), dW_down=torch.empty_like(Wd),
                 dW_r=torch.empty(w.d, w.E, dtype=torch.float32, device=dev))
    stream = torch.cuda.current_stream(dev)
    fp8_peak = measure_mxfp8_peak(dev)
    layer.prepare(Wg, Wu, Wd)
    pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pa.record(stream)
    layer.prepare(Wg, Wu, Wd)  # once per optimiser step, outside the layer step
    pb.record(stream)
    torch.cuda.synchronize()
    prep_ms = pa.elapsed_time(pb)

    def step(X, dY, Yout, g):
        layer.forward(X, x["W_r"], x["bias"], Y=Yout)
        layer.backward(X, x["W_r"], dY, out=g)

    for _ in range(args.warmup):
        step(x["X"], x["dY"], Y, grads)
    torch.cuda.synchronize()
    if layer.error() != B.MOE_OK:
        raise RuntimeError("device error during warm-up")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if needs_flush(w) else None

    B.moe_profile_read()
    B.moe_profile_enable(True)
    launches0 = B.moe_kernel_launches()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        if flush is not None:
            flush.fill_(1)
        step(x["X"], x["dY"], Y, grads)
    torch.cuda.synchronize()
    launches_per_step = (B.moe_kernel_launches() - launches0) // args.steps
    B.moe_profile_enable(False)
    prof = B.moe_profile_read()

    graph, launch_mode = None, "cuda_graph"
    if not args.no_graph:
        try:
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                step(x["X"], x["dY"], Y, grads)
            stream.wait_stream(side)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step(x["X"], x["dY"], Y, grads)
            torch.cuda.synchronize()
        except Exception as ex:
            graph, launch_mode = None, f"direct (graph capture failed: {type(ex).__name__})"
    else:
        launch_mode = "direct"

    def run_step():
        if graph is not None:
            graph.replay()
        else:
            step(x["X"], x["dY"], Y, grads)

    for _ in range(2):
        run_step()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evs:
        if flush is not None:
            flush.fill_(1)
        a.record(stream)
        run_step()
        b.record(stream)
    torch.cuda.synchronize()
    t_local = sum(a.elapsed_time(b) for a, b in evs) / 1e3
    barrier(world)
    clk = clocks.stop()
    if layer.error() != B.MOE_OK:
        raise RuntimeError("device error in the timed region")
    t = max_over_ranks(t_local, world)

    # end to end: X, dY in from pinned host memory, Y, dX out, every step (in line on the compute stream)
    hX = torch.empty(NT, w.d, dtype=torch.bfloat16, pin_memory=True)
    hdY = torch.empty_like(hX, pin_memory=True)
    hY = torch.empty_like(hX, pin_memory=True)
    hdX = torch.empty_like(hX, pin_memory=True)
    hX.copy_(x["X"].cpu())
    hdY.copy_(x["dY"].cpu())
    Xd, dYd = torch.empty_like(x["X"]), torch.empty_like(x["dY"])
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e2.record(stream)
    for _ in range(args.steps):
        Xd.copy_(hX, non_blocking=True)
        dYd.copy_(hdY, non_blocking=True)
        step(Xd, dYd, Y, grads)
        hY.copy_(Y, non_blocking=True)
        hdX.copy_(grads["dX"], non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(e2.elapsed_time(e3) / 1e3, world)
    if rank != 0:
        return

    by, fl = nv_algorithmic(w)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fp8 = fp8_peak.get("sustained_tflops")
    fp4 = 2.0 * fp8 if fp8 else 2.0 * 2.0 * float(peaks.get("bf16_tflops_sustained",
                                                            FALLBACK_PEAKS["bf16_tflops_sustained"]))
    fp4_src = ("2 x the sustained MXFP8 cuBLAS GEMM measured in this run (the nominal dense fp4 : fp8 ratio, "
               "9 : 4.5 PFLOP/s)" if fp8 else "4 x the sustained bf16 peak (nominal fp4 : bf16 ratio)")
    kern = {}
    for name, (ms, n) in sorted(prof.items(), key=lambda kv: -kv[1][0]):
        sec = ms / args.steps / 1e3
        e = {"ms_per_step": ms / args.steps, "launches_per_step": n / args.steps, "share": ms / (t * 1e3)}
        if name in by:
            e["algorithmic_GB"] = by[name] / 1e9
            e["achieved_GBs"] = by[name] / sec / 1e9
        if name in fl:
            e["achieved_TFLOPs"] = fl[name] / sec / 1e12
            tpeak = fp4 if name in NV_GEMMS else float(peaks.get("bf16_tflops_sustained",
                                                                 FALLBACK_PEAKS["bf16_tflops_sustained"]))
            e["bound"] = "tensor" if fl[name] / (tpeak * 1e12) > by.get(name, 0) / (hbm * 1e9) else "hbm"
        else:
            e["bound"] = "hbm"
        kern[name] = e
    top = max(kern.items(), key=lambda kv: kv[1]["share"])[0]
    if kern[top]["bound"] == "tensor" and top in NV_GEMMS:
        ach = kern[top]["achieved_TFLOPs"]
        roof = {"kernel": top, "bound": "tensor", "achieved": ach, "peak": fp4, "unit": "TFLOP/s",
                "frac": ach / fp4, "traffic": ncu_traffic(top, w.name), "peak_source": fp4_src}
    elif kern[top]["bound"] == "tensor":  # a bf16 GEMM (the weight gradients, the router)
        bf16 = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        ach = kern[top]["achieved_TFLOPs"]
        roof = {"kernel": top, "bound": "tensor", "achieved": ach, "peak": bf16, "unit": "TFLOP/s",
                "frac": ach / bf16, "traffic": ncu_traffic(top, w.name),
                "peak_source": "measured sustained bf16 GEMM (MEASURED_PEAKS.json bf16_tflops_sustained)"
                if peak_kind == "measured" else "fallback 1.4 PFLOP/s sustained bf16 (no MEASURED_PEAKS.json)"}
    else:
        ach = kern[top].get("achieved_GBs")
        roof = {"kernel": top, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                "frac": (ach / hbm) if ach else None, "traffic": ncu_traffic(top, w.name),
                "peak_source": f"{peak_kind} HBM copy bandwidth" if peak_kind == "measured"
                else "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"}
    tflops = w.model_flops() * args.steps * world / t / 1e12
    line = {
        "metric": METRIC_NV, "value": job_throughput(NT * args.steps, t, world), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 + e4m3 per 16 + fp32 per tensor) / bf16 wgrad", "data": "synthetic (seeded, random-init weights)",
        "config": nv_config(w),
        "tflops": tflops, "pct_of_fp4_peak": 100.0 * tflops / world / fp4, "fp4_peak_tflops": fp4,
        "peak_note": ("model FLOPs 18 d I per assignment + 6 T d E per step; the four expert dgrad / forward "
                      "GEMMs on NVFP4, the weight gradients and the router on bf16; fp4 peak = " + fp4_src),
        "roofline": roof,
        "e2e": {"value": job_throughput(NT * args.steps, t_e2e, world), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * NT * w.d * 2, "d2h_bytes_per_step": 2 * NT * w.d * 2,
                "note": "X, dY copied in from pinned host memory and Y, dX copied back every step, in line on "
                        "the compute stream; prepared weights and the weight gradients stay in HBM"},
        "gpu_launches": int(launches_per_step * args.steps), "launch": launch_mode, "clocks": clk,
        "prepare_weights_ms": prep_ms, "mxfp8_peak": fp8_peak, "kernels": kern,
    }
    if world == 1 and not args.no_cpu_baseline:
        r = nv_oracle_rate(w, cpu_inputs(w), CPU_BASELINE_STEPS)
        line["cpu_baseline"] = {"value": r["value"], "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": r["sample"]}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="dsv3", choices=sorted(IN.WORKLOADS))
    ap.add_argument("--impl", default="moe", choices=["moe", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time direct launches instead of a CUDA graph of one step")
    ap.add_argument("--wgrad-fp32", action="store_true",
                    help="write the expert weight gradients as fp32 instead of bf16 (the weights' dtype)")
    ap.add_argument("--launches", action="store_true",
                    help="run every grouped GEMM as its own launch instead of the persistent pairs")
    ap.add_argument("--wgrad-gemms", choices=["mxfp8", "bf16"], default=None,
                    help="MXFP8 workloads: the weight-gradient GEMMs on MXFP8 (operands quantised along each "
                         "expert's rows; the default) or on the bf16 operands")
    ap.add_argument("--persistent", action="store_true",
                    help="require the persistent pairs (the default for bf16 one-batch workloads): the forward's "
                         "gate/up and down GEMMs, and the backward's two dgrads, each pair as one persistent launch")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = IN.WORKLOADS[args.workload]
    if args.wgrad_gemms and not w.mxfp8:
        ap.error("--wgrad-gemms applies to the MXFP8 workloads; %s is bf16" % w.name)
    args.mx_wgrad = w.mxfp8 and args.wgrad_gemms != "bf16"
    if args.launches and w.stream_M:
        ap.error("the ring-streamed layer always runs its GEMM pairs as persistent launches")
    if args.persistent and (w.mxfp8 or w.stream_M or args.launches):
        ap.error("--persistent runs the bf16 one-batch layer with persistent GEMM pairs; %s" %
                 ("--launches was given" if args.launches else "%s is %s" % (w.name, "MXFP8" if w.mxfp8 else "streamed")))
    # the persistent GEMM pairs (measured 1-3% faster on those GEMMs) wherever the layer has them
    args.persistent = not (args.launches or w.mxfp8 or w.stream_M)
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        (run_nvfp4 if w.nvfp4 else run_moe)(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
