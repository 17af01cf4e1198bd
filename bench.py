#!/usr/bin/env python
"""Throughput of the activation-sparse gated FFN forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one forward of the whole hot path (gate GEMM with the TwELL
epilogue, overflow routing, fused sparse up x down, dense-channel launches)
over one batch of the decode workload: d_model=4096, d_ff=14336, 8 tokens,
bf16, ReLU gate with bias -1.2816 (about 90 % zeros), tile capacity 32.
Inputs are seeded synthetic tensors already resident in HBM.  Three copies of
the weights (1.06 GB) and 16 input batches rotate between steps, so no step
finds its weights in the 126 MB L2.

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica
(the forward has no exchange step), the timed region is bracketed by a
barrier and synchronisation, and the max over ranks is reported.

--impl reference times the fp64 CPU oracle (tests' correctness reference) on
the host cores on the same workload; rank 0 alone runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse gated-FFN tokens/s and achieved HBM GB/s vs peak at 90%/99% sparsity"
UNIT = "tokens/s"
WORKLOAD = "decode_bf16"
TOKENS = 8
N_WEIGHT_SETS = 3
N_X_BATCHES = 16
TIMING_STRIDE = 8
PROFILE_DIR = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = {
    "gate": ["tc_gemm.cuh", "epilogues.cuh", "ptx.cuh"],
    "updown_rows": ["rows_mma.cuh", "ptx.cuh"],
}


# ------------------------------------------------------------ distributed
def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def aggregate(elapsed_ms: float, units: float, world: int):
    """Max elapsed time and total units over ranks (identity when world == 1)."""
    if world == 1:
        return elapsed_ms, units
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    u = torch.tensor([units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.idx, self.period = device_index, period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _reasons(self):
        try:
            return self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons())
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self._stop.set()
        self._t.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b]}


# ---------------------------------------------------------------- helpers
def load_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return json.load(open(p)), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        h.update(open(os.path.join(ROOT, "activation_sparse_gated_relu_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from a committed ncu summary, if the kernel's
    sources are unchanged since it was captured."""
    p = os.path.join(PROFILE_DIR, f"traffic_{kernel}_{workload}.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_hash") != source_hash(kernel):
        return None
    return d.get("dram_bytes_per_launch")


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_timing(inp, budget_s: float, steps: int = 0):
    """Time the fp64 oracle on the workload's token batch: operands decoded to
    fp64 once, then whole oracle forwards (gate, selection, TwELL pack, sparse
    up/down) until the budget is spent (or for `steps` forwards)."""
    import numpy as np
    import oracle
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    wl = inp.wl
    W = dict(W_up=f(inp.W_up), W_down=f(inp.W_down), W_gate=f(inp.W_gate), A=f(inp.A), B=f(inp.B),
             bias=f(inp.bias))
    xs = f(inp.x)
    n, tokens, t0 = 0, 0, time.perf_counter()
    while True:
        x = xs[(n * TOKENS) % xs.shape[0]:][:TOKENS]
        oracle.forward(np.ascontiguousarray(x), W["W_up"], W["W_down"], W_gate=W["W_gate"], A=W["A"],
                       B=W["B"], bias=W["bias"], dtype=wl.dtype, mode=wl.mode, act=wl.act,
                       threshold=wl.threshold, k=wl.k, C=wl.tile_capacity)
        n += 1
        tokens += x.shape[0]
        el = time.perf_counter() - t0
        if (steps and n >= steps) or (not steps and el >= budget_s):
            break
    return tokens / el, n, el


def config_dict(wl, T: int, sets: int = N_WEIGHT_SETS) -> dict:
    return {"workload": f"{wl.name}: d_model={wl.d_model} d_ff={wl.d_ff} tokens={T} {wl.dtype} "
                        f"{wl.act} gate bias={wl.bias} (~90% zeros) tile_capacity={wl.tile_capacity}",
            "tokens_per_step": T, "d_model": wl.d_model, "d_ff": wl.d_ff,
            "l2": f"inputs larger than L2: {sets} rotating weight copies "
                  f"({sets * 3 * wl.d_model * wl.d_ff * 2 / 1e9:.2f} GB) and {N_X_BATCHES} x batches",
            "parallelism": "replicas (one independent forward per GPU)"}


# ---------------------------------------------------------------- our arm
def run_ours(args) -> None:
    import numpy as np
    import torch

    import synth
    from activation_sparse_gated_relu_b200 import SFFN_OK, SparseFFN, load_library
    from activation_sparse_gated_relu_b200.build import build

    rank, local, world = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    if rank == 0:
        build()
    barrier(world)
    load_library()

    wl = synth.WORKLOADS[WORKLOAD]
    T = TOKENS
    inp = synth.make_inputs(wl, T=T * N_X_BATCHES)
    dev = lambda t: None if t is None else t.to("cuda")  # noqa: E731
    sets = []
    for s in range(args.weight_sets):
        ws = {k: dev(getattr(inp, k)) for k in ("W_gate", "W_up", "W_down", "bias")}
        ffn = SparseFFN(ws["W_up"], ws["W_down"], W_gate=ws["W_gate"], bias=ws["bias"],
                        tile_capacity=wl.tile_capacity, max_tokens=T)
        sets.append((ws, ffn))
    xall = dev(inp.x)
    xb = [xall[i * T:(i + 1) * T].contiguous() for i in range(N_X_BATCHES)]
    NS = args.weight_sets
    outs = [torch.empty((T, wl.d_model), dtype=torch.float32, device="cuda") for _ in range(NS)]
    stream = torch.cuda.current_stream()

    def step(i):
        sets[i % NS][1].forward(xb[i % N_X_BATCHES], outs[i % NS])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    for _, ffn in sets:
        assert ffn.read_status() == SFFN_OK
    launches_per_fwd = sets[0][1].stats().n_launches

    # ------------------------------------------------------- timed region
    # per-kernel events on every TIMING_STRIDE-th forward of each handle: enough
    # launches to average, few enough not to perturb the timed region
    for _, ffn in sets:
        ffn.timing_begin(args.steps // NS // TIMING_STRIDE + 2, TIMING_STRIDE)
    clocks = ClockSampler(torch.cuda.current_device())
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    elapsed = ev0.elapsed_time(ev1)
    kernels = {}
    for _, ffn in sets:
        for name, (ms, n) in ffn.timing_end().items():
            a = kernels.setdefault(name, [0.0, 0])
            a[0] += ms
            a[1] += n
    for _, ffn in sets:
        assert ffn.read_status() == SFFN_OK
    tot_ms, tot_units = aggregate(elapsed, float(T * args.steps), world)

    # ------------------------------------------------- algorithmic bytes
    # per x batch: union of kept neurons (from the forward's TwELL records)
    ffn0 = sets[0][1]
    unions, twell_bytes = [], []
    P, C = wl.d_ff // 128, wl.tile_capacity
    for b in range(N_X_BATCHES):
        ffn0.forward(xb[b], outs[0])
        tw = ffn0.twell(T)
        n = torch.minimum(tw["count"].long(), torch.tensor(C, device="cuda"))
        used = torch.arange(C, device="cuda")[None, None, :] < n[:, :, None]
        idx = tw["idx"].long()[used]
        unions.append(int(torch.unique(idx).numel()))
    union = float(np.mean(unions))
    d, F, es = wl.d_model, wl.d_ff, 2
    twell = T * P * (2 + C * (2 + es))
    nblk = math.ceil(T / 8)
    bytes_gate = F * d * es + T * d * es + twell + nblk * P * 16
    bytes_rows = union * 2 * d * es + T * d * es + T * d * 4 + twell + nblk * P * 16
    bytes_step = F * d * es + union * 2 * d * es + T * d * es + T * d * 4 + 2 * twell

    peaks, peak_src = load_peaks()
    per = {k: (v[0] / v[1] if v[1] else 0.0) for k, v in kernels.items()}
    dom = max(per, key=lambda k: kernels[k][0]) if per else None
    alg = {"gate": bytes_gate, "updown_rows": bytes_rows}
    roof = None
    if dom in alg:
        achieved = alg[dom] / (per[dom] * 1e-3) / 1e9
        traffic = profiled_traffic(dom, WORKLOAD)
        roof = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                "algorithmic_bytes": int(alg[dom]), "ms_per_launch": round(per[dom], 5),
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                else "fallback 6650 GB/s"}
    total_kernel_ms = sum(v[0] for v in kernels.values())
    kern_out = {k: {"ms_per_launch": round(per[k], 5), "launches": kernels[k][1],
                    "share": round(kernels[k][0] / total_kernel_ms, 4) if total_kernel_ms else None,
                    **({"achieved_gbs": round(alg[k] / (per[k] * 1e-3) / 1e9, 1),
                        "frac_of_hbm": round(alg[k] / (per[k] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
                       if k in alg and per[k] > 0 else {})}
                for k in kernels}

    # ------------------------------------------------------ end to end
    e2e = None
    e2e_steps = 0 if args.no_e2e else max(10, min(args.steps, 400))
    if e2e_steps:
        xh = [inp.x[i * T:(i + 1) * T].contiguous().pin_memory() for i in range(N_X_BATCHES)]
        oh = torch.empty((T, wl.d_model), dtype=torch.float32).pin_memory()
        for i in range(3):
            sets[i % NS][1].forward_host(xh[i % N_X_BATCHES], oh)
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(e2e_steps):
            sets[i % NS][1].forward_host(xh[i % N_X_BATCHES], oh)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms, e2e_units = aggregate(e0.elapsed_time(e1), float(T * e2e_steps), world)
        e2e = {"value": round(e2e_units / (e2e_ms * 1e-3), 1), "unit": UNIT,
               "h2d_bytes_per_step": T * wl.d_model * 2, "d2h_bytes_per_step": T * wl.d_model * 4,
               "api": "sffn_forward_host (pinned host x in, host y out, stream synchronised per step)"}

    # --------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_inp = synth.make_inputs(wl, T=T * 4)
        v, n, el = oracle_timing(cpu_inp, budget_s=args.cpu_budget)
        cpu = {"value": round(v, 3), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{n} fp64 oracle forwards of {T}-token batches of the same workload "
                         f"({el:.1f} s; operands decoded to fp64 once, before timing)"}

    if rank == 0:
        value = tot_units / (tot_ms * 1e-3)
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_ms / args.steps, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Gaussian x and N(0,1/fan_in) weights)",
            "config": config_dict(wl, T, NS),
            "hbm_gbs_step": round(bytes_step * args.steps * world / (tot_ms * 1e-3) / 1e9, 1),
            "hbm_frac_step": round(bytes_step * args.steps * world / (tot_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "union_active_neurons": union,
            "algorithmic_bytes_per_step": int(bytes_step),
            "roofline": roof,
            "kernels": kern_out,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_fwd * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    for _, ffn in sets:
        ffn.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------- reference arm
def run_reference(args) -> None:
    rank, _, world = dist_env()
    if rank != 0:
        return
    import synth
    wl = synth.WORKLOADS[WORKLOAD]
    T = TOKENS
    inp = synth.make_inputs(wl, T=T * 4)
    oracle_timing(inp, 0, steps=max(1, min(args.warmup, 3)))
    v, n, el = oracle_timing(inp, 0, steps=args.steps)
    cores = cpu_threads()
    line = {
        "metric": METRIC, "value": round(v, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(el / n * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl, T), "impl": "reference",
        "cpu_baseline": {"value": round(v, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n} fp64 oracle forwards of {T}-token batches (one per step)"},
        "e2e": {"value": round(v, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    ap.add_argument("--weight-sets", type=int, default=N_WEIGHT_SETS,
                    help="rotating weight copies (fewer only for small profiler captures)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
