"""Plain fp64 CPU definition of the backward pass of the activation-sparse
gated FFN (relu-threshold selection, dense gate).

TEST INFRASTRUCTURE, like the rest of this package: only the tests, the smoke
check and the bench's CPU baseline use it; it shares no code with the CUDA
path.

Source: "Sparser, Faster, Lighter Transformer Language Models" (news
article), section "Hybrid 應對非均勻稀疏": in training, most tokens keep few
activations and go through the compact ELL format, while rare highly active
tokens are routed to a dense tensor-core channel; the page reports the
training step, not its formulas.  The gradients below are the chain rule of
the forward (``oracle.ffn.forward``), y_t = sum_j h_tj W_down[j,:] with
h_tj = keep_tj · v_tj · u_tj, v = round(sigma(g)), u = W_up x, g = W_gate x + b.

Readings where the page is silent:

1. The selection (keep) is a constant of the step: no gradient flows through
   the threshold decision, and a neuron that is not kept gets none.
2. The rounding of the stored value v = round(sigma(g)) passes the gradient
   through unchanged (its derivative is taken as 1).
3. For a loss with upstream gradient dy = dL/dy:
       dh = dy W_down^T (kept entries), du = dh·v, dv = dh·u,
       dg = dv·sigma'(g), db = sum_t dg,
       dW_down = h^T dy, dW_up = du^T x, dW_gate = dg^T x,
       dx = du W_up + dg W_gate,
   all neuron-major like the weights ([d_ff][d]).  sigma'(g) = 1 for ReLU on
   kept neurons (g > threshold >= 0) and s(1 + g(1 - s)) for SiLU.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import ffn


def act_slope(g: np.ndarray, act: str) -> np.ndarray:
    """sigma'(g): ReLU 1 for g > 0 (0 elsewhere), SiLU s(1 + g(1 - s))."""
    if act == "relu":
        return (g > 0).astype(np.float64)
    s = 1.0 / (1.0 + np.exp(-g))
    return s * (1.0 + g * (1.0 - s))


@dataclass
class Grads:
    dx: np.ndarray        # [T][d]
    dW_gate: np.ndarray   # [F][d]
    dW_up: np.ndarray     # [F][d]
    dW_down: np.ndarray   # [F][d]
    db: np.ndarray        # [F]
    keep: np.ndarray      # [T][F]
    h: np.ndarray         # [T][F]
    du: np.ndarray        # [T][F]
    dg: np.ndarray        # [T][F]


def backward(x: np.ndarray, W_gate: np.ndarray, W_up: np.ndarray, W_down: np.ndarray, dy: np.ndarray, *,
             bias: Optional[np.ndarray] = None, dtype: str = "bf16", act: str = "relu",
             threshold: float = 0.0, keep: Optional[np.ndarray] = None) -> Grads:
    """Gradients of the sparse forward for upstream dy, step by step.  keep
    defaults to the forward's own selection; passing it fixes the mask."""
    x = np.asarray(x, dtype=np.float64)
    g = ffn.gate_dense(x, W_gate, bias)
    a = ffn.activate(g, act)
    if keep is None:
        keep = ffn.keep_threshold(a, threshold)
    v = ffn.round_operand(a, dtype)
    u = x @ W_up.T
    h = np.where(keep, v * u, 0.0)
    dh = np.where(keep, dy @ W_down.T, 0.0)
    du = dh * v
    dv = dh * u
    dg = np.where(keep, dv * act_slope(g, act), 0.0)
    return Grads(dx=du @ W_up + dg @ W_gate, dW_gate=dg.T @ x, dW_up=du.T @ x, dW_down=h.T @ dy,
                 db=dg.sum(axis=0), keep=keep, h=h, du=du, dg=dg)


def backward_inputs(inp, dy: np.ndarray, T: Optional[int] = None) -> Grads:
    """Run ``backward`` on a ``synth.Inputs`` bundle (duck-typed: no import)."""
    wl = inp.wl

    def f64(t):
        return None if t is None else t.detach().to("cpu").double().numpy()
    x = f64(inp.x)
    if T is not None:
        x = x[:T]
    return backward(x, f64(inp.W_gate), f64(inp.W_up), f64(inp.W_down), dy, bias=f64(inp.bias),
                    dtype=wl.dtype, act=wl.act, threshold=wl.threshold)
