"""Plain fp64 CPU definition of a mixture-of-experts layer whose experts are
activation-sparse gated FFNs with a low-rank (LoPA) gate.

TEST INFRASTRUCTURE, like the rest of this package: only the tests, the smoke
check and the bench's CPU baseline use it; it shares no code with the CUDA
path.

Source: "Meta FAIR and Inria's LoPA Gating Hits 3.31x Real GPU Speedup for LLM
Inference", section "Model Casting and Quality at 90% Sparsity": LoPA gating
is compatible with mixture-of-experts layers whose experts share the gated FFN
structure (Mixtral, DeepSeek-V3).  The page gives no routing rule; the
reading taken is Mixtral's, the plainest:

1. router logits l[t][e] = <W_r[e], x_t> (W_r [E][d], no bias);
2. each token keeps the top_k experts of largest logit (equal logits go to
   the smaller expert index);
3. their weights are the softmax over the kept logits only;
4. y_t = sum over kept e of w[t][e] · FFN_e(x_t), each FFN_e the sparse
   gated FFN of ``oracle.ffn.forward`` with its own weights (low-rank gate
   z = round(x·A_e), g = z·B_e + b, ReLU, threshold, TwELL, sparse up/down).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import ffn


def router_logits(x: np.ndarray, W_r: np.ndarray) -> np.ndarray:
    """l[t][e] = sum_i x[t][i]·W_r[e][i]."""
    return x @ W_r.T


def select_experts(logits: np.ndarray, top_k: int) -> np.ndarray:
    """[T][top_k] expert indices: largest logit first, ties to the smaller index."""
    T, E = logits.shape
    e = np.arange(E)
    return np.stack([np.lexsort((e, -logits[t]))[:top_k] for t in range(T)])


def expert_weights(logits: np.ndarray, sel: np.ndarray) -> np.ndarray:
    """Softmax over each token's kept logits ([T][top_k])."""
    z = np.take_along_axis(logits, sel, axis=1)
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    return p / p.sum(axis=1, keepdims=True)


@dataclass
class MoeResult:
    y: np.ndarray              # [T][d]
    logits: np.ndarray         # [T][E]
    sel: np.ndarray            # [T][top_k]
    w: np.ndarray              # [T][top_k]
    expert_out: dict           # e -> (tokens, OracleResult of FFN_e on them)
    logit_band: np.ndarray     # [T][E] where fp32 device logits may order otherwise


def forward(x: np.ndarray, W_r: np.ndarray, experts: list, top_k: int, *, dtype: str = "bf16",
            threshold: float = 0.0, C: int = 32) -> MoeResult:
    """experts[e] = dict(A=[d][r], B=[r][F], W_up=[F][d], W_down=[F][d], bias=[F] or None)."""
    x = np.asarray(x, dtype=np.float64)
    T, d = x.shape
    logits = router_logits(x, W_r)
    sel = select_experts(logits, top_k)
    w = expert_weights(logits, sel)
    y = np.zeros((T, d))
    out = {}
    for e, ex in enumerate(experts):
        tok = np.nonzero((sel == e).any(axis=1))[0]
        if len(tok) == 0:
            continue
        res = ffn.forward(x[tok], ex["W_up"], ex["W_down"], A=ex["A"], B=ex["B"], bias=ex.get("bias"),
                          dtype=dtype, threshold=threshold, C=C)
        out[e] = (tok, res)
        for i, t in enumerate(tok):
            y[t] += w[t][list(sel[t]).index(e)] * res.y[i]
    band = np.ldexp(np.abs(x) @ np.abs(W_r).T, -14)
    return MoeResult(y, logits, sel, w, out, band)


def forward_inputs(inp, T: Optional[int] = None) -> MoeResult:
    """Run ``forward`` on a synthetic MoE input bundle (duck-typed)."""
    def f64(t):
        return None if t is None else t.detach().to("cpu").double().numpy()
    x = f64(inp.x)
    if T is not None:
        x = x[:T]
    ex = [{k: f64(v) for k, v in e.items()} for e in inp.experts]
    wl = inp.wl
    return forward(x, f64(inp.W_r), ex, wl.top_k, dtype="bf16", threshold=wl.threshold, C=wl.tile_capacity)
