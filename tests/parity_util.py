"""Helpers shared by the GPU parity tests: run the library and the oracle on
the same seeded inputs and compare TwELL records and outputs under the parity
rules (bit-exact TwELL where the gate arithmetic is exact, a decision band
around the selection boundary otherwise, relative max error on y)."""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

import oracle
import synth
from activation_sparse_gated_relu_b200 import SFFN_OK, SparseFFN

TOL = {"bf16": 2e-3, "fp32": 1e-5}


def to_dev(t: Optional[torch.Tensor]):
    return None if t is None else t.to("cuda").contiguous()


def make_ffn(inp: synth.Inputs, max_tokens: int, path: str = "auto", C: Optional[int] = None,
             debug_gate: bool = False, separate: bool = False, cooperative: bool = False,
             backward: bool = False) -> SparseFFN:
    wl = inp.wl
    return SparseFFN(to_dev(inp.W_up), to_dev(inp.W_down), W_gate=to_dev(inp.W_gate), A=to_dev(inp.A),
                     B=to_dev(inp.B), bias=to_dev(inp.bias), mode=wl.mode, act=wl.act,
                     threshold=wl.threshold, k=wl.k,
                     tile_capacity=wl.tile_capacity if C is None else C, max_tokens=max_tokens,
                     path=path, debug_gate=debug_gate, separate=separate, cooperative=cooperative,
                     input_k=wl.input_k or 0, V=to_dev(inp.V), backward=backward)


@dataclass
class GpuRun:
    y: np.ndarray
    count: np.ndarray
    idx: np.ndarray
    val: np.ndarray
    overflow: np.ndarray
    n_overflow: int
    path: int
    launches: int


def run_gpu(ffn: SparseFFN, x: torch.Tensor) -> GpuRun:
    xd = to_dev(x)
    T = xd.shape[0]
    out = torch.full((T, ffn.d_model), float("nan"), dtype=torch.float32, device="cuda")
    ffn.forward(xd, out)
    torch.cuda.synchronize()
    assert ffn.read_status() == SFFN_OK
    st = ffn.stats()
    tw = ffn.twell(T)
    return GpuRun(out.double().cpu().numpy(), tw["count"].cpu().numpy(), tw["idx"].cpu().numpy(),
                  tw["val"].double().cpu().numpy(),
                  (tw["overflow_epoch"].cpu().numpy().astype(np.int64) == st.epoch), st.n_overflow,
                  st.path, st.n_launches)


def rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    scale = np.abs(ref).max()
    return float(np.abs(y - ref).max() / (scale if scale > 0 else 1.0))


def ambiguous(res: oracle.OracleResult, mode: str, threshold: float, k: int, exact: bool) -> np.ndarray:
    """(t, j) whose selection may legitimately differ between fp32 device
    arithmetic and the fp64 oracle: within the band of the decision boundary."""
    if exact and mode == "relu_threshold":
        return np.zeros(res.keep.shape, dtype=bool)
    if mode == "relu_threshold":
        if np.all(res.a >= 0):  # ReLU: |a| > tau  <=>  g > tau
            return np.abs(res.g - threshold) <= res.band
        sig = 1.0 / (1.0 + np.exp(-res.g))
        slope = np.abs(sig * (1.0 + res.g * (1.0 - sig)))
        return np.abs(np.abs(res.a) - threshold) <= slope * res.band + np.ldexp(np.abs(res.a), -21)
    s = res.scores
    kth = np.sort(s, axis=1)[:, ::-1][:, max(k - 1, 0)][:, None] if k > 0 else np.full((s.shape[0], 1), np.inf)
    return np.abs(s - kth) <= res.band


def compare_twell(g: GpuRun, res: oracle.OracleResult, C: int, amb: np.ndarray, exact_vals: bool,
                  dtype: str) -> dict:
    """Check count/idx/val/overflow against the oracle; returns mismatch stats."""
    T, P = res.count.shape
    F = P * 128
    amb_tile = amb.reshape(T, P, 128).sum(-1)
    dc = np.abs(g.count.astype(np.int64) - res.count.astype(np.int64))
    assert np.all(dc <= amb_tile), "tile counts differ outside the decision band"
    # slots: ascending, in-tile, pads (-1, 0) beyond min(count, C)
    n = np.minimum(g.count, C).astype(np.int64)
    slot = np.arange(C)[None, None, :]
    used = slot < n[:, :, None]
    assert np.all(g.idx[~used] == -1), "pad indices are not -1"
    assert np.all(g.val[~used] == 0), "pad values are not +0"
    tile_of = np.where(used, g.idx // 128, -1)
    assert np.all(tile_of[used] == np.broadcast_to(np.arange(P)[None, :, None], used.shape)[used])
    dif = np.diff(np.where(used, g.idx, 1 << 20), axis=2)
    assert np.all((dif > 0) | ~used[:, :, 1:]), "indices not ascending"
    # kept sets (complete for tiles with count <= C)
    trunc = g.count > C
    tt, pp, ss = np.nonzero(used)
    jj = g.idx[tt, pp, ss].astype(np.int64)
    gkeep = np.zeros((T, F), dtype=bool)
    gval = np.zeros((T, F))
    gkeep[tt, jj] = True
    gval[tt, jj] = g.val[tt, pp, ss]
    trunc_f = np.repeat(trunc, 128, axis=1)
    mism = (gkeep != res.keep) & ~trunc_f
    assert not np.any(mism & ~amb), "kept sets differ outside the decision band"
    # truncated tiles: every listed neuron is kept by the oracle or ambiguous
    assert np.all(res.keep[tt, jj] | amb[tt, jj])
    both = gkeep & res.keep
    if exact_vals:
        assert np.array_equal(gval[both], res.v[both]), "TwELL values not bit-exact"
    else:
        # the device value may differ by the gate's accumulation error (at
        # most the band) plus one rounding of the stored format
        rtol = 2.0 ** -7 if dtype == "bf16" else 2.0 ** -22
        v = res.v[both]
        assert np.all(np.abs(gval[both] - v) <= rtol * np.abs(v) + 2 * res.band[both] + 1e-30), \
            "TwELL values differ"
    ovf_ref = res.overflow
    amb_tok = (amb_tile > 0).any(1)
    assert np.all((g.overflow == ovf_ref) | amb_tok), "overflow flags differ"
    assert np.array_equal(g.overflow, (g.count > C).any(1))
    assert g.n_overflow == int(g.overflow.sum())
    return {"mismatch": int(mism.sum()), "ambiguous": int(amb.sum()), "overflow": int(g.overflow.sum())}


def check(inp: synth.Inputs, T: Optional[int] = None, path: str = "auto", C: Optional[int] = None,
          res: Optional[oracle.OracleResult] = None, ffn: Optional[SparseFFN] = None,
          separate: bool = False) -> dict:
    wl = inp.wl
    x = inp.x if T is None else inp.x[:T]
    T = x.shape[0]
    C = wl.tile_capacity if C is None else C
    if res is None:
        res = oracle.forward(synth.to_f64(x), synth.to_f64(inp.W_up), synth.to_f64(inp.W_down),
                             W_gate=synth.to_f64(inp.W_gate), A=synth.to_f64(inp.A), B=synth.to_f64(inp.B),
                             bias=synth.to_f64(inp.bias), dtype=wl.dtype, mode=wl.mode, act=wl.act,
                             threshold=wl.threshold, k=wl.k, C=C, input_k=wl.input_k,
                             V=synth.to_f64(inp.V))
    own = ffn is None
    if own:
        ffn = make_ffn(inp, max_tokens=T, path=path, C=C, separate=separate)
    try:
        g = run_gpu(ffn, x)
    finally:
        if own:
            ffn.close()
    amb = ambiguous(res, wl.mode, wl.threshold, wl.k, wl.exact_grid)
    stats = compare_twell(g, res, C, amb, exact_vals=wl.exact_grid and wl.mode == "relu_threshold",
                          dtype=wl.dtype)
    err = rel_err(g.y, res.y)
    stats.update(err=err, path=g.path, launches=g.launches)
    assert np.all(np.isfinite(g.y)), "output not fully written"
    assert err <= TOL[wl.dtype], f"max|y - y_ref| / max|y_ref| = {err:.3e}"
    return stats
