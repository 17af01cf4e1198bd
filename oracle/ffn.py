"""Plain fp64 CPU definition of the activation-sparse gated FFN forward.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU
baseline use this module; the library's CUDA path never imports it and it
imports nothing from the library.  It is deliberately slow and literal: every
step is the definition written out in numpy float64, one function per step,
with no blocking, fusion or reordering beyond a library matmul used as a step.

Sources (web pages, cited by title and section):

* [LoPA] "Meta FAIR and Inria's LoPA Gating Hits 3.31x Real GPU Speedup for
  LLM Inference", section "How LoPA Gating Restructures FFN Computation":
  the gated FFN is gate projection -> activation -> elementwise multiply ->
  down projection; LoPA makes the gate low rank with rank ratio 1/8.
* [TwELL] "Sparser, Faster, Lighter Transformer Language Models" (news
  article), sections "稀疏不等於提速" (ReLU as sigma gives unstructured
  zeros), "TwELL 減掉轉換開銷" (tile-wise ELLPACK written in the gate
  epilogue; one pass fusing the up and down products so h is never stored),
  "Hybrid 應對非均勻稀疏" (highly active tokens routed whole to a dense
  tensor-core channel).
* [WINA] "大语言模型推理加速新突破：解读WINA框架的核心原理与实践价值",
  section 3.1 (score = |hidden value| x ||weight column||_2) and section 2
  (keep the top-K neurons per layer and token).

Readings where the pages are silent or garbled (the formulas of the gated FFN
were lost from the [TwELL] page):

1. y = W_down^T (sigma(g) ⊙ u) with g = W_gate x + b and u = W_up x, all
   weights stored neuron-major as [d_ff][d] (row j = neuron j).
2. Threshold selection keeps (t, j) iff |sigma(g_tj)| > tau (strict), tested
   on the unrounded fp64 activation; the per-neuron fp32 bias is added before
   sigma.
3. The stored TwELL value is v = round_bf16_RNE(a) (round_fp32(a) for fp32
   operands); the hidden value is h = v·u (0 where not kept); u and y are not
   rounded.
4. LoPA rank r = d/8; the intermediate z = x·A is rounded to the operand dtype
   (RNE) before z·B, the plainest point at which two GEMMs must round.
5. The WINA "hidden value" is the gate activation a = sigma(g) and the
   "weight column" is column j of the down projection in math form (row j of
   the neuron-major W_down): s_tj = |a_tj|·n_j with n_j = round_fp32(||row
   j||_2).  Exactly k neurons are kept per token; equal scores go to the
   smaller index.
6. TwELL: tiles of 128 consecutive neurons; per (token, tile) the true kept
   count (int16), then C slots holding the kept global neuron indices in
   ascending order (int16) and their values, padded with (-1, +0.0).  A token
   overflows iff some tile of it holds more than C kept neurons; the whole
   token then takes the dense channel.  y does not depend on C or routing.

Pins (tests/test_oracle_pins.py): exact-rational brute force on tiny inputs,
hand-worked fixtures in tests/golden/, the sparse == masked-dense invariant,
tau = 0 ReLU == textbook dense FFN, TwELL pack/unpack round trip, the A = I
low-rank reduction, WINA k = d_ff / k = 0 / equal-norm reductions, bf16
rounding against torch's RNE conversion and hand-derived bit patterns, and the
closed-form sparsity of the synthetic recipes.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

TILE = 128  # neurons per TwELL tile ([TwELL] "TwELL 減掉轉換開銷")


# ----------------------------------------------------------------------------
# rounding to the storage formats
# ----------------------------------------------------------------------------
def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), in fp64.

    bfloat16 has 8 significant bits and fp32's exponent range: normal numbers
    have ulp 2^(e-7) for |a| in [2^e, 2^(e+1)), e >= -126; below 2^-126 the
    spacing is the subnormal step 2^-133.  Rounding is done directly from fp64
    (no detour through fp32, which could double-round).
    """
    a = np.asarray(a, dtype=np.float64)
    out = np.array(a, dtype=np.float64, copy=True)
    fin = np.isfinite(a) & (a != 0.0)
    af = a[fin]
    _, ex = np.frexp(np.abs(af))           # |a| = m·2^ex, m in [0.5, 1)
    e = ex.astype(np.int64) - 1            # |a| in [2^e, 2^(e+1))
    e = np.maximum(e, -126)                # subnormal range shares 2^-133 step
    ulp = np.ldexp(1.0, (e - 7).astype(np.int64))
    q = np.rint(af / ulp) * ulp            # np.rint rounds half to even
    big = np.abs(q) >= 2.0 ** 128          # beyond bf16 max -> infinity
    q[big] = np.copysign(np.inf, q[big])
    out[fin] = q
    return out


def round_fp32(a: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest float32 (ties to even), in fp64."""
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_operand(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round to the operand dtype: "bf16", "fp32", or "fp64" (no rounding: the
    exact-arithmetic variant the finite-difference pins of the backward use)."""
    if dtype == "fp64":
        return np.asarray(a, dtype=np.float64)
    return round_bf16(a) if dtype == "bf16" else round_fp32(a)


# ----------------------------------------------------------------------------
# gate ([LoPA] "How LoPA Gating Restructures FFN Computation")
# ----------------------------------------------------------------------------
def gate_dense(x: np.ndarray, W_gate: np.ndarray, bias: Optional[np.ndarray]) -> np.ndarray:
    """g[t, j] = sum_i x[t, i]·W_gate[j, i] + b[j]  (W_gate neuron-major [d_ff][d])."""
    g = x @ W_gate.T
    if bias is not None:
        g = g + bias[None, :]
    return g


def gate_lowrank(x: np.ndarray, A: np.ndarray, B: np.ndarray, bias: Optional[np.ndarray],
                 dtype: str) -> tuple[np.ndarray, np.ndarray]:
    """Low-rank gate: z = round_dtype(x·A) ([d][r] factor), g = z·B + b ([r][d_ff])."""
    z = round_operand(x @ A, dtype)
    g = z @ B
    if bias is not None:
        g = g + bias[None, :]
    return g, z


# ----------------------------------------------------------------------------
# activation and selection
# ----------------------------------------------------------------------------
def activate(g: np.ndarray, act: str) -> np.ndarray:
    """sigma(g): ReLU max(0, g) ([TwELL] "稀疏不等於提速"), or SiLU g/(1+e^-g)."""
    if act == "relu":
        return np.maximum(g, 0.0)
    if act == "silu":
        return g / (1.0 + np.exp(-g))
    raise ValueError(act)


def keep_threshold(a: np.ndarray, tau: float) -> np.ndarray:
    """Threshold rule on the hidden magnitude: keep iff |a| > tau (strict)."""
    return np.abs(a) > tau


def wina_norms(W_down: np.ndarray) -> np.ndarray:
    """n_j = ||W_down[j, :]||_2 in fp64, rounded to fp32 ([WINA] section 3.1)."""
    return round_fp32(np.sqrt(np.sum(W_down * W_down, axis=1)))


def wina_scores(a: np.ndarray, norms: np.ndarray) -> np.ndarray:
    """s[t, j] = |a[t, j]|·n_j ([WINA] section 3.1)."""
    return np.abs(a) * norms[None, :]


def keep_topk(s: np.ndarray, k: int) -> np.ndarray:
    """Per token, keep the k largest scores; equal scores go to the smaller index."""
    T, F = s.shape
    keep = np.zeros((T, F), dtype=bool)
    j = np.arange(F)
    for t in range(T):
        order = np.lexsort((j, -s[t]))  # primary: score descending; then index
        keep[t, order[:k]] = True
    return keep


# ----------------------------------------------------------------------------
# WINA variants ([WINA] sections 3.1 to 3.3)
# ----------------------------------------------------------------------------
def wina_full_h_scores(a: np.ndarray, u: np.ndarray, norms: np.ndarray) -> np.ndarray:
    """s[t, j] = |a[t, j]·u[t, j]|·n_j: the score of section 3.1 with the
    hidden value taken as the full gated product h = sigma(g)·u (unrounded),
    which needs the up projection of every neuron."""
    return np.abs(a * u) * norms[None, :]


def input_col_norms(W_gate: np.ndarray, W_up: np.ndarray) -> np.ndarray:
    """c_i = ||column i of the stacked [W_gate; W_up]||_2 in fp64, rounded to
    fp32: x feeds the gate and the up projection, so the layer that consumes
    x_i is the stacked [2 d_ff][d] matrix, and its column i is the "weight
    column" of section 3.1 for input coordinate i."""
    return round_fp32(np.sqrt(np.sum(W_gate * W_gate, axis=0) + np.sum(W_up * W_up, axis=0)))


def input_scores(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """s[t, i] = |x[t, i]|·c_i rounded once to fp32 (the precision the
    selection is decided in on both sides: x and c are exact in fp64, so the
    rounded product is unique)."""
    return round_fp32(np.abs(x) * c[None, :])


def select_input(x: np.ndarray, keep_in: np.ndarray) -> np.ndarray:
    """x with the input coordinates that are not kept set to zero."""
    return np.where(keep_in, x, 0.0)


def orthogonal_basis(W_gate: np.ndarray, W_up: np.ndarray) -> np.ndarray:
    """V of the SVD [W_gate; W_up] = U·S·V^T (section 3.3: the weight is
    right-multiplied by V, which makes its columns orthogonal, U·S).  A
    library SVD is the step."""
    _, _, Vt = np.linalg.svd(np.concatenate([W_gate, W_up], axis=0), full_matrices=False)
    return Vt.T.copy()


def rotate(M: np.ndarray, V: np.ndarray, dtype: str) -> np.ndarray:
    """M·V rounded to the operand dtype: a neuron-major weight [n][d] times V
    gives the orthogonalised weight; an activation batch [T][d] times V gives
    the rotated input V^T x_t of each token (so that W V V^T x = W x)."""
    return round_operand(M @ V, dtype)


# ----------------------------------------------------------------------------
# TwELL ([TwELL] "TwELL 減掉轉換開銷")
# ----------------------------------------------------------------------------
def twell_pack(keep: np.ndarray, v: np.ndarray, C: int, tile: int = TILE):
    """Pack kept (t, j) into tile-wise ELL: count[T][P], idx[T][P][C], val[T][P][C].

    count is the true number kept in the tile (it may exceed C); slots hold the
    first min(count, C) kept neurons in ascending order (global index, int16)
    with their values; remaining slots are (-1, +0.0).  overflow[t] is True iff
    some tile of token t holds more than C kept neurons.
    """
    T, F = keep.shape
    P = F // tile
    count = np.zeros((T, P), dtype=np.int16)
    idx = np.full((T, P, C), -1, dtype=np.int16)
    val = np.zeros((T, P, C), dtype=np.float64)
    for t in range(T):
        for p in range(P):
            js = np.nonzero(keep[t, p * tile:(p + 1) * tile])[0] + p * tile
            count[t, p] = len(js)
            n = min(len(js), C)
            idx[t, p, :n] = js[:n]
            val[t, p, :n] = v[t, js[:n]]
    overflow = (count > C).any(axis=1)
    return count, idx, val, overflow


def twell_unpack(count: np.ndarray, idx: np.ndarray, val: np.ndarray, d_ff: int):
    """Expand TwELL back to a dense [T][d_ff] value matrix and kept mask.

    Only tiles with count <= C unpack completely; the others are truncated.
    """
    T, P, C = idx.shape
    dense = np.zeros((T, d_ff), dtype=np.float64)
    mask = np.zeros((T, d_ff), dtype=bool)
    for t in range(T):
        for p in range(P):
            n = min(int(count[t, p]), C)
            js = idx[t, p, :n].astype(np.int64)
            dense[t, js] = val[t, p, :n]
            mask[t, js] = True
    return dense, mask


# ----------------------------------------------------------------------------
# up, product, down ([TwELL] "TwELL 減掉轉換開銷": u and y in one pass)
# ----------------------------------------------------------------------------
def sparse_up_down(x: np.ndarray, W_up: np.ndarray, W_down: np.ndarray,
                   keep: np.ndarray, v: np.ndarray) -> np.ndarray:
    """For each token: u_j = <W_up[j], x_t> on kept j, h_j = v_tj·u_j,
    y_t = sum_j h_j·W_down[j].  Only the kept rows are touched."""
    T, d = x.shape
    y = np.zeros((T, d), dtype=np.float64)
    for t in range(T):
        js = np.nonzero(keep[t])[0]
        if len(js) == 0:
            continue
        u = W_up[js] @ x[t]
        h = v[t, js] * u
        y[t] = h @ W_down[js]
    return y


def dense_masked_ffn(x: np.ndarray, W_up: np.ndarray, W_down: np.ndarray,
                     keep: np.ndarray, v: np.ndarray) -> np.ndarray:
    """The same y as ``sparse_up_down`` with a different loop nest: the full
    dense up projection, the hidden matrix with non-kept entries zeroed, and
    one dense down projection (used as an invariant pin)."""
    U = x @ W_up.T
    H = np.where(keep, v * U, 0.0)
    return H @ W_down


# ----------------------------------------------------------------------------
# bands where fp32 accumulation on the device may legitimately flip a decision
# ----------------------------------------------------------------------------
def gate_band(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """2^-14·sum_i |x_ti·W_ji|: about 16x the statistical fp32 accumulation
    error at K = 4096, used as the width of the decision band."""
    return np.ldexp(np.abs(x) @ np.abs(W).T, -14)


def lowrank_band(z: np.ndarray, B: np.ndarray) -> np.ndarray:
    """Band for the low-rank gate: the accumulation band of z·B plus two
    bf16 rounding flips of the largest z_r·B_rj term."""
    zb = np.abs(z) @ np.abs(B)
    big = np.stack([np.max(np.abs(zt)[:, None] * np.abs(B), axis=0) for zt in z])
    return np.ldexp(zb, -14) + 2.0 * np.ldexp(big, -7)


def exact_grid_ok(x: np.ndarray, W: np.ndarray, grid_exp: int) -> bool:
    """True iff every gate/up partial sum is an integer multiple of 2^-grid_exp
    below 2^24 units in magnitude, so fp32 accumulation is exact in any order."""
    units = np.ldexp(np.abs(x) @ np.abs(W).T, grid_exp)
    return bool(np.all(units < 2.0 ** 24))


# ----------------------------------------------------------------------------
# the whole forward
# ----------------------------------------------------------------------------
@dataclass
class OracleResult:
    y: np.ndarray            # [T][d]   fp64
    g: np.ndarray            # [T][F]   gate pre-activation
    a: np.ndarray            # [T][F]   activation
    v: np.ndarray            # [T][F]   stored (rounded) value
    keep: np.ndarray         # [T][F]   bool
    count: np.ndarray        # [T][P]   int16
    idx: np.ndarray          # [T][P][C] int16
    val: np.ndarray          # [T][P][C] fp64 (already rounded)
    overflow: np.ndarray     # [T]      bool
    band: np.ndarray         # [T][F]   decision band around the selection boundary
    scores: Optional[np.ndarray] = None
    norms: Optional[np.ndarray] = None
    z: Optional[np.ndarray] = None
    x_used: Optional[np.ndarray] = None   # [T][d] the input both projections saw
    x_keep: Optional[np.ndarray] = None   # [T][d] input coordinates kept (input-side WINA)


def forward(x: np.ndarray, W_up: np.ndarray, W_down: np.ndarray, *,
            W_gate: Optional[np.ndarray] = None, A: Optional[np.ndarray] = None,
            B: Optional[np.ndarray] = None, bias: Optional[np.ndarray] = None,
            dtype: str = "bf16", mode: str = "relu_threshold", act: str = "relu",
            threshold: float = 0.0, k: int = 0, C: int = 32,
            input_k: Optional[int] = None, V: Optional[np.ndarray] = None) -> OracleResult:
    """The activation-sparse gated FFN forward, step by step, in fp64.

    All array arguments are float64 decodes of the operands (exact).  Steps:
    [rotation] -> [input selection] -> gate -> activation -> stored value ->
    selection -> TwELL pack/overflow -> up on kept rows -> product -> down on
    kept rows.

    WINA variants ([WINA] sections 3.1 to 3.3): ``mode="wina_full_h"`` scores
    the full gated product |sigma(g)·u| instead of |sigma(g)|; ``input_k``
    keeps, per token, the input_k input coordinates with the largest
    |x_i|·c_i (c = column norms of [W_gate; W_up]) and zeroes the others
    before both projections (dense gate only); ``V`` orthogonalises: the gate
    and up weights become round(W·V) and each token's input round(x·V), which
    leaves W·x unchanged up to those roundings.
    """
    x = np.asarray(x, dtype=np.float64)
    x_in = None
    if V is not None:
        if W_gate is None:
            raise ValueError("the orthogonalisation needs the dense gate")
        W_gate = rotate(W_gate, V, dtype)
        W_up = rotate(W_up, V, dtype)
        x = rotate(x, V, dtype)
    if input_k is not None:
        if W_gate is None:
            raise ValueError("input-side selection needs the dense gate")
        c = input_col_norms(W_gate, W_up)
        x_in = keep_topk(input_scores(x, c), input_k)
        x = select_input(x, x_in)
    z = None
    if W_gate is not None:
        g = gate_dense(x, W_gate, bias)
        band = gate_band(x, W_gate)
    else:
        g, z = gate_lowrank(x, A, B, bias, dtype)
        band = lowrank_band(z, B)
    a = activate(g, act)
    v = round_operand(a, dtype)
    scores = norms = None
    if mode == "relu_threshold":
        keep = keep_threshold(a, threshold)
    elif mode == "wina_topk":
        norms = wina_norms(W_down)
        scores = wina_scores(a, norms)
        keep = keep_topk(scores, k)
        # a score moves by at most |sigma'(g)|·(gate band) times n_j, plus the
        # device's float32 rounding of the activation and of the product
        slope = np.abs(_silu_slope(g)) if act == "silu" else 1.0
        band = (slope * band + np.ldexp(np.abs(a), -21)) * norms[None, :]
    elif mode == "wina_full_h":
        norms = wina_norms(W_down)
        u_all = x @ W_up.T
        scores = wina_full_h_scores(a, u_all, norms)
        keep = keep_topk(scores, k)
        # the score moves with the device's gate error (through sigma'), its
        # up-projection error (the same band on W_up) and fp32 roundings
        slope = np.abs(_silu_slope(g)) if act == "silu" else 1.0
        band = (slope * band * np.abs(u_all) + np.abs(a) * gate_band(x, W_up)
                + np.ldexp(np.abs(a * u_all), -20)) * norms[None, :]
    else:
        raise ValueError(mode)
    count, idx, val, overflow = twell_pack(keep, v, C)
    y = sparse_up_down(x, W_up, W_down, keep, v)
    return OracleResult(y, g, a, v, keep, count, idx, val, overflow, band,
                        scores=scores, norms=norms, z=z, x_used=x, x_keep=x_in)


def _silu_slope(g: np.ndarray) -> np.ndarray:
    s = 1.0 / (1.0 + np.exp(-g))
    return s * (1.0 + g * (1.0 - s))


def forward_inputs(inp, T: Optional[int] = None) -> OracleResult:
    """Run ``forward`` on a ``synth.Inputs`` bundle (duck-typed: no import)."""
    wl = inp.wl

    def f64(t):
        return None if t is None else t.detach().to("cpu").double().numpy()

    x = f64(inp.x)
    if T is not None:
        x = x[:T]
    return forward(x, f64(inp.W_up), f64(inp.W_down), W_gate=f64(inp.W_gate),
                   A=f64(inp.A), B=f64(inp.B), bias=f64(inp.bias), dtype=wl.dtype,
                   mode=wl.mode, act=wl.act, threshold=wl.threshold, k=wl.k,
                   C=wl.tile_capacity, input_k=getattr(wl, "input_k", None),
                   V=f64(getattr(inp, "V", None)))
