#!/usr/bin/env python
"""Throughput of the activation-sparse gated FFN forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload decode_bf16|lopa_bf16|wina_bf16|prefill_bf16|tiny_fp32]

One step = one forward of the whole hot path over one batch of synthetic
tokens: gate GEMM with the TwELL epilogue (dense, low-rank or WINA top-k),
overflow routing, the sparse up x down of the non-overflow tokens and the
dense channel of the overflow tokens.  The default workload is decode:
d_model=4096, d_ff=14336, 8 tokens, bf16, ReLU gate with bias -1.2816 (about
90 % zeros), tile capacity 32.  The other workloads are the low-rank gate
(rank 512, 32 tokens), WINA top-k (k = 5018 of 14336, SiLU, 32 tokens),
sparse prefill (d_model=2048, d_ff=8192, 4096 tokens, ~99 % zeros with
heavy-tailed per-token activity, tile capacity 8) and a tiny fp32 case.
Inputs are seeded synthetic tensors already resident in HBM.  Several copies
of the weights rotate between steps, so that no step finds its weights in
the 126 MB L2.

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
DEFAULT_WORKLOAD = "decode_bf16"
# tokens per step, rotating weight copies, x batches, default timed steps
BENCH_SHAPES = {
    "decode_bf16": (8, 3, 16, 2000),
    "lopa_bf16": (32, 2, 16, 1000),
    "wina_bf16": (32, 2, 16, 1000),
    "prefill_bf16": (4096, 4, 3, 300),
    "tiny_fp32": (64, 1, 4, 1000),
    "wina_fullh_bf16": (32, 2, 16, 1000),
    "wina_input_bf16": (32, 2, 16, 1000),
    "gsi_bf16": (8, 12, 16, 2000),
    "moe_lopa_bf16": (8, 1, 16, 400),
    "train_prefill_bf16": (4096, 2, 3, 100),
}
SPARSITY = {
    "decode_bf16": "relu gate bias -1.2816 (~90% zeros)",
    "lopa_bf16": "low-rank gate r=512, relu, bias -1.2816 (~90% zeros)",
    "wina_bf16": "silu gate, WINA top-k k=5018 (65% dropped)",
    "prefill_bf16": "relu gate, heavy-tailed per-token nnz (mean ~99 dropped of 8192)",
    "tiny_fp32": "relu gate bias -1.2816 (~90% zeros)",
    "wina_fullh_bf16": "silu gate, WINA full-h top-k |a*u|*||w_down|| k=5018 (65% dropped)",
    "wina_input_bf16": "silu gate, orthogonal rotation V, input-side top-2048 of 4096, WINA top-k k=5018",
}
GSI_WORKLOADS = ("gsi_bf16",)
MOE_WORKLOADS = ("moe_lopa_bf16",)
TIMING_STRIDE = 8
REF_BUDGET_S = 90.0
PROFILE_DIR = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = {
    "gate": ["gate_rows.cuh", "rows_mma.cuh", "tc_gemm.cuh", "tc_gate_persist.cuh", "epilogues.cuh", "ptx.cuh"],
    "gate_lowrank_z": ["tc_gemm.cuh", "epilogues.cuh", "ptx.cuh"],
    "tile_h": ["tc_gemm.cuh", "epilogues.cuh", "ptx.cuh"],
    "fallback_h": ["tc_gemm.cuh", "epilogues.cuh", "ptx.cuh"],
    "down": ["tc_gemm.cuh", "epilogues.cuh", "ptx.cuh"],
    "updown_rows": ["rows_mma.cuh", "ptx.cuh"],
    "decode_fused": ["decode_fused.cuh", "rows_mma.cuh", "epilogues.cuh", "ptx.cuh"],
    "tile_fused": ["tile_fused.cuh", "tc_gemm.cuh", "epilogues.cuh", "ptx.cuh"],
    "router": ["simt.cuh", "ptx.cuh"],
    "wina_topk": ["simt.cuh", "ptx.cuh"],
    "gate_f32": ["simt.cuh", "epilogues.cuh", "ptx.cuh"],
    "rows_f32": ["simt.cuh", "ptx.cuh"],
    "fallback_f32": ["simt.cuh", "ptx.cuh"],
    "rotate_x": ["tc_gemm.cuh", "epilogues.cuh", "ptx.cuh"],
    "input_select": ["simt.cuh", "ptx.cuh"],
    "gsi_project": ["gsi.cuh", "ptx.cuh"],
    "gsi_resid": ["gsi.cuh", "ptx.cuh"],
    "gsi_out": ["gsi.cuh", "ptx.cuh"],
    "moe_route": ["moe.cuh", "ptx.cuh"],
    "moe_combine": ["moe.cuh", "ptx.cuh"],
    "bwd_index": ["backward.cuh", "simt.cuh", "ptx.cuh"],
    "bwd_token": ["backward.cuh", "epilogues.cuh", "ptx.cuh"],
    "bwd_neuron": ["backward.cuh", "ptx.cuh"],
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


def oracle_timing(inp, T: int, budget_s: float, steps: int = 0):
    """Time the fp64 oracle on T-token batches of the workload: operands
    decoded to fp64 once, then whole oracle forwards (gate, selection, TwELL
    pack, sparse up/down, dense channel) until the budget is spent (or for
    `steps` forwards)."""
    import numpy as np
    import oracle
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    wl = inp.wl
    W = dict(W_up=f(inp.W_up), W_down=f(inp.W_down), W_gate=f(inp.W_gate), A=f(inp.A), B=f(inp.B),
             bias=f(inp.bias), V=f(inp.V))
    xs = f(inp.x)
    n, tokens, t0 = 0, 0, time.perf_counter()
    while True:
        x = xs[(n * T) % xs.shape[0]:][:T]
        oracle.forward(np.ascontiguousarray(x), W["W_up"], W["W_down"], W_gate=W["W_gate"], A=W["A"],
                       B=W["B"], bias=W["bias"], dtype=wl.dtype, mode=wl.mode, act=wl.act,
                       threshold=wl.threshold, k=wl.k, C=wl.tile_capacity, input_k=wl.input_k, V=W["V"])
        n += 1
        tokens += x.shape[0]
        el = time.perf_counter() - t0
        if (steps and n >= steps) or (not steps and el >= budget_s):
            break
    return tokens / el, n, el


def weight_bytes(wl) -> int:
    es = 4 if wl.dtype == "fp32" else 2
    gate = (wl.d_model + wl.d_ff) * wl.rank if wl.rank else wl.d_ff * wl.d_model
    return (gate + 2 * wl.d_ff * wl.d_model) * es


def config_dict(wl, T: int, sets: int, x_batches: int) -> dict:
    return {"workload": f"{wl.name}: d_model={wl.d_model} d_ff={wl.d_ff} tokens={T} {wl.dtype} "
                        f"{SPARSITY.get(wl.name, '')} tile_capacity={wl.tile_capacity}",
            "tokens_per_step": T, "d_model": wl.d_model, "d_ff": wl.d_ff,
            "l2": f"inputs larger than L2: {sets} rotating weight copies "
                  f"({sets * weight_bytes(wl) / 1e9:.2f} GB) and {x_batches} x batches"
                  if sets * weight_bytes(wl) > 126e6 else
                  f"weights ({weight_bytes(wl) / 1e6:.1f} MB) are L2-resident: this workload is launch-bound",
            "parallelism": "replicas (one independent forward per GPU)"}


def kernel_work(wl, T: int, path: str, st: dict) -> dict:
    """Algorithmic HBM bytes and FLOPs of one launch of each kernel of the
    forward, from the workload's sizes and the realised sparsity of the batch
    (st: union = distinct kept neurons of the live tokens, nnz = their kept
    (token, neuron) pairs, n_overflow).  Bytes count what the method must
    move (weights read once, x, out, TwELL written and read); FLOPs exclude
    the dense work the method avoids and the dense channel's recomputed gate."""
    d, F, R = wl.d_model, wl.d_ff, wl.rank
    P, C = F // 128, wl.tile_capacity
    es = 4 if wl.dtype == "fp32" else 2
    twell = T * P * (2 + C * (2 + es))
    kmask = T * P * 16
    xb, yb = T * d * es, T * d * 4
    n_o, U, nnz = st["n_overflow"], st["union"], st["nnz"]
    fp32 = wl.dtype == "fp32"
    w = {}
    if wl.rotation != "none":
        w["rotate_x"] = {"bytes": d * d * es + 2 * xb, "flops": 2 * T * d * d}
    if wl.input_k:
        w["input_select"] = {"bytes": 2 * xb + d * 4, "flops": 0}
    g = "gate_f32" if fp32 else "gate"
    if R:
        w["gate_lowrank_z"] = {"bytes": d * R * es + xb + T * R * es, "flops": 2 * T * d * R}
        w[g] = {"bytes": R * F * es + T * R * es + twell + kmask, "flops": 2 * T * R * F}
    elif wl.mode == "wina_topk":
        w[g] = {"bytes": F * d * es + xb + T * F * (es + 4) + F * 4, "flops": 2 * T * d * F}
        w["wina_topk"] = {"bytes": T * F * (es + 4) + twell, "flops": 0}
    elif wl.mode == "wina_full_h":
        # g and u of every neuron: W_gate and W_up in full; v, score and h out
        w[g] = {"bytes": 2 * F * d * es + xb + T * F * (es + 8) + F * 4, "flops": 4 * T * d * F}
        w["wina_topk"] = {"bytes": T * F * (es + 8) + twell + T * F * 4, "flops": 0}
    else:
        w[g] = {"bytes": F * d * es + xb + twell + (0 if fp32 else kmask), "flops": 2 * T * d * F}
    sparse = {"bytes": U * 2 * d * es + xb + yb + twell, "flops": 4 * nnz * d}
    dense_in = 2 * F * d * es if n_o else 0      # W_gate and W_up, read once if any token overflows
    if fp32:
        w["router"] = {"bytes": T * 4, "flops": 0}
        w["rows_f32"] = sparse
        w["fallback_f32"] = {"bytes": dense_in + (F * d * es if n_o else 0), "flops": 4 * n_o * d * F}
    elif path == "rows":
        w["updown_rows"] = {"bytes": sparse["bytes"] + kmask, "flops": sparse["flops"]}
        if wl.mode != "wina_topk":
            w["fallback_h"] = {"bytes": dense_in + n_o * F * 4, "flops": 2 * n_o * d * F}
        w["down"] = {"bytes": (F * d * es + n_o * F * 4 + n_o * d * 4) if n_o else 0, "flops": 2 * n_o * F * d}
        # the single persistent launch (T <= 8): W_gate once, the W_up and
        # W_down rows of every token's kept neurons (an overflow token's too:
        # it has no separate dense channel), x in, y out, the TwELL records
        # and keep masks written once
        Ua, nnza = st.get("union_all", U), st.get("nnz_all", nnz)
        w["decode_fused"] = {"bytes": F * d * es + xb + Ua * 2 * d * es + yb + twell + kmask,
                             "flops": 2 * T * d * F + 4 * nnza * d}
    else:
        # the single tile launch (up to 32 tokens, threshold selection): the
        # gate's weights, the W_up and W_down rows of the kept neurons' union,
        # x in, y out, the TwELL records written
        if wl.mode == "relu_threshold":
            gw = (d * R + R * F) * es if R else F * d * es
            w["tile_fused"] = {"bytes": gw + U * 2 * d * es + xb + yb + twell,
                               "flops": (2 * T * (d * R + R * F) if R else 2 * T * d * F) + 4 * T * F * d}
        w["router"] = {"bytes": yb + 2 * n_o * d * es, "flops": 0}
        if wl.mode != "wina_full_h":
            w["tile_h"] = {"bytes": F * d * es + xb + twell + T * F * 4, "flops": 2 * T * d * F}
        if wl.mode == "relu_threshold":
            w["fallback_h"] = {"bytes": dense_in + n_o * F * 4, "flops": 2 * n_o * d * F}
        w["down"] = {"bytes": F * d * es + T * F * 4 + yb, "flops": 2 * T * F * d}
    return w


def step_work(wl, T: int, st: dict) -> tuple[int, int]:
    """Algorithmic bytes and FLOPs of one whole forward."""
    d, F, R = wl.d_model, wl.d_ff, wl.rank
    P, C = F // 128, wl.tile_capacity
    es = 4 if wl.dtype == "fp32" else 2
    twell = T * P * (2 + C * (2 + es))
    gate_w = (d * R + R * F) * es if R else F * d * es
    gate_f = 2 * T * (d * R + R * F) if R else 2 * T * d * F
    n_o = st["n_overflow"]
    byts = gate_w + st["union"] * 2 * d * es + T * d * es + T * d * 4 + 2 * twell
    if n_o:
        byts += 2 * F * d * es
    flops = gate_f + 4 * st["nnz"] * d + 4 * n_o * d * F
    if wl.mode == "wina_full_h":       # W_up read in full (not the union), u of every neuron
        byts += (F - st["union"]) * d * es
        flops += 2 * T * d * F - 2 * st["nnz"] * d
    if wl.rotation != "none":          # V read once per forward; x·V
        byts += d * d * es
        flops += 2 * T * d * d
    return int(byts), int(flops)


def roofline_of(work: dict, ms: float, peaks: dict, peak_src: str) -> dict:
    """Roofline of one kernel: bound = the resource whose ideal time for the
    kernel's algorithmic work is longer (HBM bytes at the copy peak, or bf16
    tensor FLOPs at the sustained GEMM peak, the kernel being timed inside a
    long run of steps)."""
    hbm, tc = peaks["hbm_gbs"], peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    t_hbm = work["bytes"] / (hbm * 1e9)
    t_tc = work["flops"] / (tc * 1e12)
    src = "measured" if peak_src == "measured" else "fallback"
    if t_tc > t_hbm:
        a = work["flops"] / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": round(a, 2), "peak": tc, "unit": "TFLOP/s",
                "frac": round(a / tc, 4), "algorithmic_flops": int(work["flops"]),
                "peak_source": f"{src} (bf16_tflops_sustained)"}
    a = work["bytes"] / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(a, 1), "peak": hbm, "unit": "GB/s", "frac": round(a / hbm, 4),
            "algorithmic_bytes": int(work["bytes"]), "peak_source": f"{src} (hbm_gbs)"}


# ---------------------------------------------------------------- our arm
def batch_sparsity(ffn, T: int, C: int) -> dict:
    """Realised sparsity of the last forward, from its TwELL records: the
    distinct kept neurons of the live (non-overflow) tokens, their kept pairs,
    the 8-token-block unions summed (rows the fused kernel gathers) and the
    overflow count."""
    import torch
    tw = ffn.twell(T)
    cnt = tw["count"].long()
    ovf = (cnt > C).any(dim=1)
    live = ~ovf
    n = torch.minimum(cnt, torch.tensor(C, device=cnt.device))
    used = (torch.arange(C, device=cnt.device)[None, None, :] < n[:, :, None]) & live[:, None, None]
    idx = tw["idx"].long()
    tok = torch.arange(T, device=cnt.device)[:, None, None].expand_as(idx)
    kept_idx, kept_tok = idx[used], tok[used]
    blocks = torch.zeros(((T + 7) // 8, ffn.d_ff), dtype=torch.bool, device=cnt.device)
    blocks[kept_tok // 8, kept_idx] = True
    st = {"union": int(torch.unique(kept_idx).numel()), "nnz": int(kept_idx.numel()),
          "block_rows": int(blocks.sum()), "n_overflow": int(ovf.sum())}
    # every token's full kept set (overflow tokens too), from the keep masks
    # of a ROWS-path forward: what the single launch streams
    st["union_all"], st["nnz_all"] = st["union"], st["nnz"]
    if ffn.stats().path == 1:
        km = ffn.keep_masks(T).to(torch.int64) & 0xFFFFFFFF
        bits = ((km[..., None] >> torch.arange(32, device=km.device)) & 1).bool()  # [T][P][4][32]
        st["nnz_all"] = int(bits.sum())
        st["union_all"] = int(bits.any(dim=0).sum())
    return st


def backward_work(wl, T: int, st: dict) -> dict:
    """Algorithmic bytes and FLOPs of the backward's kernels: the kept rows
    of W_gate, W_up and W_down read once, x and dy read, dx and the three dW
    arrays (fp32) written, three fp32 values per kept pair written and read;
    per kept pair 3 dot products and 2 updates of d in the token pass, 3
    updates of d in the neuron pass."""
    d, F = wl.d_model, wl.d_ff
    U, nnz = st.get("union_all", st["union"]), st.get("nnz_all", st["nnz"])
    return {
        "bwd_index": {"bytes": T * F // 8 * 3 + nnz * 8, "flops": 0},
        "bwd_token": {"bytes": U * 3 * d * 2 + T * d * (2 + 4 + 4) + nnz * 12, "flops": 10 * nnz * d},
        "bwd_neuron": {"bytes": 3 * F * d * 4 + F * 4 + nnz * 12, "flops": 6 * nnz * d},
    }


def measure(wl, T: int, NS: int, NXB: int, steps: int, warmup: int, world: int, traffic_key,
            train: bool = False) -> dict:
    """Time `steps` forwards of workload `wl` at T tokens (after `warmup`):
    NS rotating weight copies and NXB x batches resident in HBM, CUDA events
    around the whole region, barrier and max over ranks.  Returns the line's
    device-side fields (no e2e, no CPU baseline) plus the handles' objects
    for the caller's end-to-end pass."""
    import torch

    import synth
    from activation_sparse_gated_relu_b200 import SFFN_OK, SparseFFN

    inp = synth.make_inputs(wl, T=T * NXB)
    dev = lambda t: None if t is None else t.to("cuda")  # noqa: E731
    sets = []
    for s in range(NS):
        ws = {k: dev(getattr(inp, k)) for k in ("W_gate", "A", "B", "W_up", "W_down", "bias")}
        ffn = SparseFFN(ws["W_up"], ws["W_down"], W_gate=ws["W_gate"], A=ws["A"], B=ws["B"], bias=ws["bias"],
                        mode=wl.mode, act=wl.act, threshold=wl.threshold, k=wl.k,
                        tile_capacity=wl.tile_capacity, max_tokens=T, input_k=wl.input_k or 0,
                        V=dev(inp.V), backward=train)
        sets.append((ws, ffn))
    xall = dev(inp.x)
    xb = [xall[i * T:(i + 1) * T].contiguous() for i in range(NXB)]
    outs = [torch.empty((T, wl.d_model), dtype=torch.float32, device="cuda") for _ in range(NS)]
    stream = torch.cuda.current_stream()
    if train:   # one training step: the forward, then the backward for a fixed upstream gradient
        dys = dev(synth.upstream_grad(wl, T).contiguous())
        gbuf = {k: torch.empty(shape, dtype=torch.float32, device="cuda") for k, shape in (
            ("dx", (T, wl.d_model)), ("dW_gate", (wl.d_ff, wl.d_model)), ("dW_up", (wl.d_ff, wl.d_model)),
            ("dW_down", (wl.d_ff, wl.d_model)), ("d_bias", (wl.d_ff,)))}

    def step(i):
        f = sets[i % NS][1]
        f.forward(xb[i % NXB], outs[i % NS])
        if train:
            f.backward(xb[i % NXB], dys, **gbuf)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    for _, ffn in sets:
        assert ffn.read_status() == SFFN_OK
    launches_per_fwd = sets[0][1].stats().n_launches

    # ------------------------------------------------------- timed region
    # per-kernel events on every TIMING_STRIDE-th forward of each handle: enough
    # launches to average, few enough not to perturb the timed region
    for _, ffn in sets:   # (a training step records the forward and the backward)
        ffn.timing_begin((2 if train else 1) * (steps // NS // TIMING_STRIDE + 2), TIMING_STRIDE)
    clocks = ClockSampler(torch.cuda.current_device())
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    ev0.record(stream)
    for i in range(steps):
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
    tot_ms, tot_units = aggregate(elapsed, float(T * steps), world)

    # ---------------------------------- algorithmic work of the batches
    ffn0 = sets[0][1]
    sp = []
    for b in range(NXB):
        ffn0.forward(xb[b], outs[0])
        sp.append(batch_sparsity(ffn0, T, wl.tile_capacity))
    st = {k: sum(x[k] for x in sp) / len(sp) for k in sp[0]}
    path = "rows" if ffn0.stats().path == 1 else "tiles"
    works = kernel_work(wl, T, path, st)
    bytes_step, flops_step = step_work(wl, T, st)
    if train:
        bw = backward_work(wl, T, st)
        works.update(bw)
        bytes_step += sum(v["bytes"] for v in bw.values())
        flops_step += sum(v["flops"] for v in bw.values())

    peaks, peak_src = load_peaks()
    per = {k: (v[0] / v[1] if v[1] else 0.0) for k, v in kernels.items()}
    dom = max(per, key=lambda k: kernels[k][0]) if per else None
    # A forward that is one launch of one kernel: its average duration in the
    # timed region is the region's event time over the launches (consecutive
    # launches overlap prologue and tail by programmatic dependent launch; the
    # per-launch events, which break that overlap for the forwards they
    # bracket, are reported beside it as ms_per_launch_events)
    single = len(kernels) == 1 and launches_per_fwd == 1 and not train
    ms_dom = tot_ms / steps if single else per.get(dom, 0.0)
    roof = None
    if dom in works and ms_dom > 0:
        roof = roofline_of(works[dom], ms_dom, peaks, peak_src)
        traffic = profiled_traffic(dom, traffic_key) if traffic_key else None
        roof.update({"kernel": dom, "traffic": traffic, "ms_per_launch": round(ms_dom, 5)})
        if single:
            roof.update({"ms_per_launch_events": round(per[dom], 5),
                         "launch_time": "timed-region events / launches (one launch per forward)"})
    total_kernel_ms = sum(v[0] for v in kernels.values())
    kern_out = {}
    for k in kernels:
        e = {"ms_per_launch": round(per[k], 5), "launches": kernels[k][1],
             "share": round(kernels[k][0] / total_kernel_ms, 4) if total_kernel_ms else None}
        if k in works and per[k] > 0 and (works[k]["bytes"] or works[k]["flops"]):
            r = roofline_of(works[k], per[k], peaks, peak_src)
            e.update({"bound": r["bound"], "achieved": r["achieved"], "unit": r["unit"], "frac": r["frac"]})
        kern_out[k] = e
    step_s = tot_ms * 1e-3 / steps
    return {
        "value": round(tot_units / (tot_ms * 1e-3), 1), "ms_per_step": round(tot_ms / steps, 5),
        "steps": steps, "warmup": warmup,
        "hbm_gbs_step": round(bytes_step * world / step_s / 1e9, 1),
        "hbm_frac_step": round(bytes_step * world / step_s / 1e9 / peaks["hbm_gbs"], 4),
        "tflops_step": round(flops_step * world / step_s / 1e12, 2),
        "tensor_frac_step": round(flops_step * world / step_s / 1e12
                                  / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), 4),
        "sparsity": {k: round(v, 1) for k, v in st.items()},
        "path": path, "algorithmic_bytes_per_step": bytes_step, "algorithmic_flops_per_step": flops_step,
        "roofline": roof, "kernels": kern_out, "gpu_launches": launches_per_fwd * steps, "clocks": clk,
        "_sets": sets, "_inp": inp, "_NXB": NXB,
    }


def gsi_work(wl, T: int, n_slow: float, any_slow: float) -> dict:
    """Algorithmic bytes of the GSI forward's kernels (bf16 operands): the
    basis twice (V_k^T rows for g, V_k rows for r), the cached image M, W only
    when some token of the batch is slow (any_slow = the fraction of batches
    with one), x, g and y.  FLOPs: 2 k d_in per token twice, 2 k d_out per
    token and 2 d_in d_out per slow token."""
    di, do, k = wl.d_in, wl.d_out, wl.k
    xb = T * di * 2
    return {
        "gsi_project": {"bytes": k * di * 2 + xb + T * k * 4, "flops": 2 * T * k * di},
        "gsi_resid": {"bytes": di * k * 2 + xb + T * k * 4, "flops": 2 * T * k * di},
        "gsi_out": {"bytes": do * k * 2 + any_slow * do * di * 2 + T * k * 4 + T * do * 4,
                    "flops": 2 * T * k * do + 2 * n_slow * di * do},
    }


def measure_gsi(wl, T: int, NS: int, NXB: int, steps: int, warmup: int, world: int) -> dict:
    """The same protocol as `measure` for the gated subspace linear layer."""
    import torch

    import synth
    from activation_sparse_gated_relu_b200 import GsiLinear

    inp = synth.make_gsi_inputs(wl, T=T * NXB)
    Vk = inp.Vk.to("cuda")
    layers = []
    for s in range(NS):
        W = inp.W.to("cuda") if s == 0 else layers[0][0].clone()
        Vs = Vk if s == 0 else Vk.clone()
        layers.append((W, Vs, GsiLinear(W, Vs, wl.eps, max_tokens=T)))
    xall = inp.x.to("cuda")
    xb = [xall[i * T:(i + 1) * T].contiguous() for i in range(NXB)]
    outs = [torch.empty((T, wl.d_out), dtype=torch.float32, device="cuda") for _ in range(NS)]
    stream = torch.cuda.current_stream()

    def step(i):
        layers[i % NS][2].forward(xb[i % NXB], outs[i % NS])

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    for _, _, lay in layers:
        lay.timing_begin(steps // NS // TIMING_STRIDE + 2, TIMING_STRIDE)
    clocks = ClockSampler(torch.cuda.current_device())
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    ev0.record(stream)
    for i in range(steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    elapsed = ev0.elapsed_time(ev1)
    kernels = {}
    for _, _, lay in layers:
        for name, (ms, n) in lay.timing_end().items():
            a = kernels.setdefault(name, [0.0, 0])
            a[0] += ms
            a[1] += n
    tot_ms, tot_units = aggregate(elapsed, float(T * steps), world)
    slow = []
    for b in range(NXB):
        layers[0][2].forward(xb[b], outs[0])
        slow.append(layers[0][2].n_slow())
    n_slow = sum(slow) / NXB
    any_slow = sum(1 for v in slow if v) / NXB
    works = gsi_work(wl, T, n_slow, any_slow)
    for _, _, lay in layers:
        lay.close()
    peaks, peak_src = load_peaks()
    per = {k: (v[0] / v[1] if v[1] else 0.0) for k, v in kernels.items()}
    dom = max(per, key=lambda k: kernels[k][0]) if per else None
    roof = None
    if dom in works and per[dom] > 0:
        roof = roofline_of(works[dom], per[dom], peaks, peak_src)
        roof.update({"kernel": dom, "traffic": None, "ms_per_launch": round(per[dom], 5)})
    total_kernel_ms = sum(v[0] for v in kernels.values())
    kern_out = {}
    for k in kernels:
        e = {"ms_per_launch": round(per[k], 5), "launches": kernels[k][1],
             "share": round(kernels[k][0] / total_kernel_ms, 4) if total_kernel_ms else None}
        if k in works and per[k] > 0:
            r = roofline_of(works[k], per[k], peaks, peak_src)
            e.update({"bound": r["bound"], "achieved": r["achieved"], "unit": r["unit"], "frac": r["frac"]})
        kern_out[k] = e
    bytes_step = sum(w["bytes"] for w in works.values())
    step_s = tot_ms * 1e-3 / steps
    dense_bytes = wl.d_out * wl.d_in * 2
    return {
        "value": round(tot_units / (tot_ms * 1e-3), 1), "ms_per_step": round(tot_ms / steps, 5),
        "steps": steps, "warmup": warmup,
        "hbm_gbs_step": round(bytes_step * world / step_s / 1e9, 1),
        "hbm_frac_step": round(bytes_step * world / step_s / 1e9 / peaks["hbm_gbs"], 4),
        "algorithmic_bytes_per_step": int(bytes_step),
        "slow_tokens_per_step": n_slow, "batches_with_a_slow_token": any_slow,
        "weight_read_ratio_vs_dense": round(dense_bytes / bytes_step, 2),
        "roofline": roof, "kernels": kern_out, "gpu_launches": 3 * steps, "clocks": clk,
        "config": {"workload": f"{wl.name}: linear d_in={wl.d_in} -> d_out={wl.d_out}, basis k={wl.k}, "
                               f"eps={wl.eps}, tokens={T} bf16, residual ratio lognormal(median "
                               f"{wl.rho_med}, sigma {wl.rho_sigma})",
                   "tokens_per_step": T,
                   "l2": f"inputs larger than L2: {NS} rotating weight sets (each: W, V_k, M) and {NXB} x batches"},
        "dtype": "bf16", "unit": UNIT,
    }


def measure_moe(wl, T: int, NXB: int, steps: int, warmup: int, world: int) -> dict:
    """The same protocol as `measure` for the mixture of LoPA-gated experts
    (one weight set: the E experts' weights are far larger than L2)."""
    import torch

    import synth
    from activation_sparse_gated_relu_b200 import SFFN_OK, MoeFFN

    inp = synth.make_moe_inputs(wl, T=T * NXB)
    dev = lambda t: None if t is None else t.to("cuda")  # noqa: E731
    ex = [{k: dev(v) for k, v in e.items()} for e in inp.experts]
    moe = MoeFFN(dev(inp.W_r), ex, wl.top_k, threshold=wl.threshold, tile_capacity=wl.tile_capacity,
                 max_tokens=T)
    xall = dev(inp.x)
    xb = [xall[i * T:(i + 1) * T].contiguous() for i in range(NXB)]
    out = torch.empty((T, wl.d_model), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        moe.forward(xb[i % NXB], out)
    torch.cuda.synchronize()
    assert moe.read_status() == SFFN_OK
    moe.timing_begin(steps // TIMING_STRIDE + 2, TIMING_STRIDE)
    clocks = ClockSampler(torch.cuda.current_device())
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    ev0.record(stream)
    for i in range(steps):
        moe.forward(xb[i % NXB], out)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    elapsed = ev0.elapsed_time(ev1)
    kernels = {k: list(v) for k, v in moe.timing_end().items()}
    assert moe.read_status() == SFFN_OK
    tot_ms, tot_units = aggregate(elapsed, float(T * steps), world)
    # realised work: every expert reads its low-rank gate, then the W_up and
    # W_down rows its routed tokens keep (zero rows keep nothing)
    d, F, r, E = wl.d_model, wl.d_ff, wl.rank, wl.experts
    rows = []
    for b in range(NXB):
        moe.forward(xb[b], out)
        u = 0
        for e in range(E):
            tw = moe.expert_twell(e, T)
            n = torch.minimum(tw["count"].long(), torch.tensor(wl.tile_capacity, device="cuda"))
            used = torch.arange(wl.tile_capacity, device="cuda")[None, None, :] < n[:, :, None]
            u += int(torch.unique(tw["idx"].long()[used]).numel())
        rows.append(u)
    moe.close()
    union = sum(rows) / NXB
    bytes_step = E * d * 2 + E * (d * r + r * F) * 2 + union * 2 * d * 2 + T * d * 2 + T * d * 4
    peaks, peak_src = load_peaks()
    step_s = tot_ms * 1e-3 / steps
    per = {k: (v[0] / v[1] if v[1] else 0.0) for k, v in kernels.items()}
    total_kernel_ms = sum(v[0] for v in kernels.values())
    kern_out = {k: {"ms_per_launch": round(per[k], 5), "launches": kernels[k][1],
                    "share": round(kernels[k][0] / total_kernel_ms, 4) if total_kernel_ms else None}
                for k in kernels}
    dom = max(per, key=lambda k: kernels[k][0]) if per else None
    return {
        "value": round(tot_units / (tot_ms * 1e-3), 1), "ms_per_step": round(tot_ms / steps, 5),
        "steps": steps, "warmup": warmup,
        "hbm_gbs_step": round(bytes_step * world / step_s / 1e9, 1),
        "hbm_frac_step": round(bytes_step * world / step_s / 1e9 / peaks["hbm_gbs"], 4),
        "algorithmic_bytes_per_step": int(bytes_step), "expert_rows_kept_per_step": union,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(bytes_step / step_s / 1e9, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(bytes_step / step_s / 1e9 / peaks["hbm_gbs"], 4), "traffic": None,
                     "scope": "whole forward (router, every expert's kernels, combine)"},
        "kernels": kern_out, "clocks": clk,
        "config": {"workload": f"{wl.name}: {E} experts, top-{wl.top_k}, d_model={d} d_ff={F} rank={r} "
                               f"tokens={T} bf16, relu gate bias {wl.bias} (~90% zeros per expert)",
                   "tokens_per_step": T,
                   "l2": f"inputs larger than L2: {E} experts' weights ({E * (2 * F * d + d * r + r * F) * 2 / 1e9:.2f} GB)"},
        "dtype": "bf16", "unit": UNIT,
    }


# the other configurations, measured after the headline in the same default
# run: (workload, tokens per forward)
EXTRA_WORKLOADS = [("decode_bf16", 1), ("decode_bf16", 4), ("lopa_bf16", 32), ("wina_bf16", 32),
                   ("prefill_bf16", 4096), ("tiny_fp32", 64), ("wina_fullh_bf16", 32), ("wina_input_bf16", 32),
                   ("gsi_bf16", 8), ("moe_lopa_bf16", 8), ("train_prefill_bf16", 4096)]
EXTRA_MIN_STEPS = 200
EXTRA_MAX_S = 2.0


def run_ours(args) -> None:
    import torch

    import synth
    from activation_sparse_gated_relu_b200 import load_library
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

    if args.workload == "train_prefill_bf16":
        T = args.tokens or BENCH_SHAPES[args.workload][0]
        _, NSt, NXBt, _ = BENCH_SHAPES[args.workload]
        m = measure(synth.WORKLOADS["prefill_bf16"], T, NSt, NXBt, args.steps, args.warmup, world, None, train=True)
        for _, f in m.pop("_sets"):
            f.close()
        m.pop("_inp"), m.pop("_NXB")
        if rank == 0:
            line = {"metric": METRIC + " (training step: forward + sparse backward)", "value": m.pop("value"),
                    "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                    "ms_per_step": m.pop("ms_per_step"), "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                    "config": config_dict(synth.WORKLOADS["prefill_bf16"], T, NSt, NXBt)}
            m.pop("steps"), m.pop("warmup")
            line.update(m)
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if args.workload in GSI_WORKLOADS or args.workload in MOE_WORKLOADS:
        T, _, NXB, _ = BENCH_SHAPES[args.workload]
        T = args.tokens or T
        if args.workload in GSI_WORKLOADS:
            m = measure_gsi(synth.GSI_WORKLOADS[args.workload], T, args.weight_sets, NXB, args.steps,
                            args.warmup, world)
        else:
            m = measure_moe(synth.MOE_WORKLOADS[args.workload], T, NXB, args.steps, args.warmup, world)
        if rank == 0:
            line = {"metric": METRIC, "value": m.pop("value"), "unit": UNIT, "n_gpus": world,
                    "steps": args.steps, "warmup": args.warmup, "ms_per_step": m.pop("ms_per_step"),
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                    "data": "synthetic (seeded Gaussian or low-rank activations, N(0,1/fan_in) weights)",
                    "config": m.pop("config")}
            m.pop("steps"), m.pop("warmup"), m.pop("unit"), m.pop("dtype")
            line.update(m)
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    wl = synth.WORKLOADS[args.workload]
    T, _, NXB, _ = BENCH_SHAPES[args.workload]
    T = args.tokens or T
    NS = args.weight_sets
    # the committed captures are of the workload's own token count
    tkey = args.workload if T == BENCH_SHAPES[args.workload][0] else None
    m = measure(wl, T, NS, NXB, args.steps, args.warmup, world, tkey)
    sets, inp = m.pop("_sets"), m.pop("_inp")
    m.pop("_NXB")

    # ------------------------------------------------------ end to end
    e2e = None
    e2e_steps = 0 if args.no_e2e else max(10, min(args.steps, 400))
    if e2e_steps:
        xh = [inp.x[i * T:(i + 1) * T].contiguous().pin_memory() for i in range(NXB)]
        oh = torch.empty((T, wl.d_model), dtype=torch.float32).pin_memory()
        for i in range(3):
            sets[i % NS][1].forward_host(xh[i % NXB], oh)
        stream = torch.cuda.current_stream()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(e2e_steps):
            sets[i % NS][1].forward_host(xh[i % NXB], oh)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms, e2e_units = aggregate(e0.elapsed_time(e1), float(T * e2e_steps), world)
        es = 4 if wl.dtype == "fp32" else 2
        e2e = {"value": round(e2e_units / (e2e_ms * 1e-3), 1), "unit": UNIT,
               "h2d_bytes_per_step": T * wl.d_model * es, "d2h_bytes_per_step": T * wl.d_model * 4,
               "api": "sffn_forward_host (pinned host x in, host y out, stream synchronised per step)"}
    for _, ffn in sets:
        ffn.close()
    del sets
    torch.cuda.empty_cache()

    # --------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_inp = synth.make_inputs(wl, T=T * min(NXB, 4))
        v, n, el = oracle_timing(cpu_inp, T, budget_s=args.cpu_budget)
        cpu = {"value": round(v, 3), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{n} fp64 oracle forwards of {T}-token batches of the same workload "
                         f"({el:.1f} s; operands decoded to fp64 once, before timing)"}

    # ------------------------- the other configurations (one GPU only)
    workloads = None
    if world == 1 and not args.no_workloads and args.workload == DEFAULT_WORKLOAD and not args.tokens:
        workloads = {}
        for name, Tw in EXTRA_WORKLOADS:
            _, NSx, NXBx, _ = BENCH_SHAPES[name]
            if name in MOE_WORKLOADS:
                wlm = synth.MOE_WORKLOADS[name]
                probe = measure_moe(wlm, Tw, NXBx, 16, max(args.warmup, 3), world)
                ksteps = max(EXTRA_MIN_STEPS, min(2000, int(EXTRA_MAX_S / (probe["ms_per_step"] * 1e-3))))
                workloads[f"{name}@T={Tw}"] = measure_moe(wlm, Tw, NXBx, ksteps, max(args.warmup, 3), world)
                torch.cuda.empty_cache()
                continue
            if name in GSI_WORKLOADS:
                wlg = synth.GSI_WORKLOADS[name]
                probe = measure_gsi(wlg, Tw, NSx, NXBx, 24, max(args.warmup, 3), world)
                ksteps = max(EXTRA_MIN_STEPS, min(5000, int(EXTRA_MAX_S / (probe["ms_per_step"] * 1e-3))))
                ksteps -= ksteps % NSx
                workloads[f"{name}@T={Tw}"] = measure_gsi(wlg, Tw, NSx, NXBx, ksteps, max(args.warmup, 3), world)
                torch.cuda.empty_cache()
                continue
            train = name == "train_prefill_bf16"
            wlx = synth.WORKLOADS["prefill_bf16" if train else name]
            # a bounded run: at least EXTRA_MIN_STEPS forwards, about
            # EXTRA_MAX_S seconds at most, from a short probe of the step time
            probe = measure(wlx, Tw, NSx, NXBx, 10, max(args.warmup, 3), world, None, train=train)
            for _, f in probe.pop("_sets"):
                f.close()
            ksteps = max(EXTRA_MIN_STEPS, min(5000, int(EXTRA_MAX_S / (probe["ms_per_step"] * 1e-3))))
            ksteps -= ksteps % NSx
            key = name if Tw == BENCH_SHAPES[name][0] else None
            r = measure(wlx, Tw, NSx, NXBx, ksteps, max(args.warmup, 3), world, None if train else key, train=train)
            for _, f in r.pop("_sets"):
                f.close()
            r.pop("_inp"), r.pop("_NXB")
            torch.cuda.empty_cache()
            r["config"] = config_dict(wlx, Tw, NSx, NXBx)
            r["dtype"] = "f32" if wlx.dtype == "fp32" else "bf16"
            r["unit"] = UNIT
            workloads[f"{name}@T={Tw}"] = r

    if rank == 0:
        line = {
            "metric": METRIC, "value": m["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": m["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32" if wl.dtype == "fp32" else "bf16",
            "data": "synthetic (seeded Gaussian x and N(0,1/fan_in) weights)",
            "config": config_dict(wl, T, NS, NXB),
        }
        for k in ("hbm_gbs_step", "hbm_frac_step", "tflops_step", "tensor_frac_step", "sparsity", "path",
                  "algorithmic_bytes_per_step", "algorithmic_flops_per_step", "roofline", "kernels"):
            line[k] = m[k]
        line.update({"cpu_baseline": cpu, "e2e": e2e, "gpu_launches": m["gpu_launches"], "clocks": m["clocks"]})
        if workloads is not None:
            line["workloads"] = workloads
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------- reference arm
def run_reference(args) -> None:
    """The reference arm: the fp64 oracle on the host cores, one T-token
    forward of the workload per step.  The timed steps are capped so that the
    whole run stays within a few minutes (the rate does not depend on how
    many forwards are timed); the line says how many were."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    import synth
    if args.workload in GSI_WORKLOADS or args.workload in MOE_WORKLOADS:
        run_reference_other(args)
        return
    wl = synth.WORKLOADS[args.workload]
    T, _, NXB, _ = BENCH_SHAPES[args.workload]
    T = args.tokens or T
    inp = synth.make_inputs(wl, T=T * min(NXB, 4))
    _, nw, elw = oracle_timing(inp, T, 0, steps=max(1, min(args.warmup, 3)))
    per_fwd = elw / nw
    n_timed = max(1, min(args.steps, int(REF_BUDGET_S / max(per_fwd, 1e-6))))
    v, n, el = oracle_timing(inp, T, 0, steps=n_timed)
    cores = cpu_threads()
    sample = (f"{n} fp64 oracle forwards of {T}-token batches (one per step; {args.steps} steps asked, "
              f"capped at ~{REF_BUDGET_S:.0f} s of host time)")
    line = {
        "metric": METRIC, "value": round(v, 3), "unit": UNIT, "n_gpus": world, "steps": n,
        "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": round(el / n * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl, T, 1, min(NXB, 4)), "impl": "reference",
        "cpu_baseline": {"value": round(v, 3), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(v, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_other(args) -> None:
    """The reference arm for the GSI and MoE workloads: their fp64 oracles on
    the host, one forward of the workload's token batch per step."""
    import numpy as np

    import oracle.gsi
    import oracle.moe
    import synth
    T = args.tokens or BENCH_SHAPES[args.workload][0]
    if args.workload in GSI_WORKLOADS:
        wl = synth.GSI_WORKLOADS[args.workload]
        inp = synth.make_gsi_inputs(wl, T=T * 4)
        x, W, Vk = (t.double().numpy() for t in (inp.x, inp.W, inp.Vk))
        run = lambda xt: oracle.gsi.forward(xt, W, Vk, wl.eps, wl.dtype)  # noqa: E731
        desc = f"{wl.name}: d_in={wl.d_in} d_out={wl.d_out} k={wl.k} eps={wl.eps} tokens={T}"
    else:
        wl = synth.MOE_WORKLOADS[args.workload]
        inp = synth.make_moe_inputs(wl, T=T * 4)
        x = inp.x.double().numpy()
        Wr = inp.W_r.double().numpy()
        ex = [{k: (None if v is None else v.double().numpy()) for k, v in e.items()} for e in inp.experts]
        run = lambda xt: oracle.moe.forward(xt, Wr, ex, wl.top_k, threshold=wl.threshold,  # noqa: E731
                                            C=wl.tile_capacity)
        desc = f"{wl.name}: {wl.experts} experts top-{wl.top_k} d_model={wl.d_model} d_ff={wl.d_ff} tokens={T}"
    n, t0 = 0, time.perf_counter()
    while n < max(1, args.steps):
        run(np.ascontiguousarray(x[(n * T) % x.shape[0]:][:T]))
        n += 1
        if time.perf_counter() - t0 > REF_BUDGET_S:
            break
    el = time.perf_counter() - t0
    v = n * T / el
    line = {"metric": METRIC, "value": round(v, 3), "unit": UNIT, "n_gpus": 1, "steps": n,
            "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": round(el / n * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": desc}, "impl": "reference",
            "cpu_baseline": {"value": round(v, 3), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                             "sample": f"{n} fp64 oracle forwards of {T} tokens"},
            "e2e": {"value": round(v, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default: per workload)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(BENCH_SHAPES), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other configurations measured after the default workload")
    ap.add_argument("--weight-sets", type=int, default=None,
                    help="rotating weight copies (fewer only for small profiler captures)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--tokens", type=int, default=None,
                    help="tokens per forward instead of the workload's own (e.g. 1 or 4 for decode_bf16)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.tokens is not None and args.tokens < 1:
        ap.error("--tokens must be >= 1")
    _, sets, _, steps = BENCH_SHAPES[args.workload]
    if args.steps is None:
        args.steps = steps
    if args.weight_sets is None:
        args.weight_sets = sets
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
