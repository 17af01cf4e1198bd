"""Plain fp64 CPU definition of the gated subspace linear layer (GSI).

TEST INFRASTRUCTURE, like the rest of this package: only the tests, the smoke
check and the bench's CPU baseline use it; it shares no code with the CUDA
path.

Source: "Gated Subspace Inference for Transformer Acceleration" (technical
summary page), section 2.1 "核心分解" and section 2.2 "门控残差直通".  For a
linear layer y = W x with W [d_out][d] (the PyTorch Linear layout) and an
orthonormal basis V_k [d][k] of the activation subspace:

    g = V_k^T x,   r = x - V_k g,   M = W V_k  (cached),   W x = M g + W r.

Per token the residual ratio rho = ||r|| / ||x|| decides the path: below the
threshold eps the fast path y = M g reads only the k columns' image M; at or
above it the slow path computes y = W x in full.  Section 2.2 bounds the fast
path's error by ||W||_2 · eps · ||x|| (its Theorem 4).

Readings where the page is silent:

1. Precision: M is stored in the operand dtype, M = round(W V_k) (it is a
   weight, cached like the others); g is rounded to the operand dtype before
   M g (the plainest point at which two GEMMs must round, as for LoPA's z);
   r and rho use the unrounded g; y is fp32 on the device, fp64 here.
2. The comparison is strict: fast iff rho < eps (the page: "低于阈值").
   rho is compared squared, ||r||^2 < eps^2 ||x||^2, so no root or division
   decides a token; x = 0 takes the slow path (y = 0 either way).
3. The slow path computes W x, not M g + W r (the page: "执行完整计算").
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .ffn import round_operand


def project(x: np.ndarray, Vk: np.ndarray) -> np.ndarray:
    """g[t] = V_k^T x_t  ([T][k])."""
    return x @ Vk


def residual(x: np.ndarray, Vk: np.ndarray, g: np.ndarray) -> np.ndarray:
    """r[t] = x_t - V_k g_t  ([T][d])."""
    return x - g @ Vk.T


def image(W: np.ndarray, Vk: np.ndarray, dtype: str) -> np.ndarray:
    """M = W V_k rounded to the operand dtype ([d_out][k]), the cached image."""
    return round_operand(W @ Vk, dtype)


def route_fast(x: np.ndarray, r: np.ndarray, eps: float) -> np.ndarray:
    """fast[t] iff ||r_t||^2 < eps^2 ||x_t||^2 (rho < eps, strict)."""
    return np.sum(r * r, axis=1) < (eps * eps) * np.sum(x * x, axis=1)


@dataclass
class GsiResult:
    y: np.ndarray          # [T][d_out]
    g: np.ndarray          # [T][k] unrounded projection
    g_hat: np.ndarray      # [T][k] rounded projection (the fast path's operand)
    r: np.ndarray          # [T][d]
    rho: np.ndarray        # [T]
    fast: np.ndarray       # [T] bool
    M: np.ndarray          # [d_out][k]
    rho_band: np.ndarray   # [T] width around eps in which the device may decide otherwise


def forward(x: np.ndarray, W: np.ndarray, Vk: np.ndarray, eps: float, dtype: str = "bf16") -> GsiResult:
    """GSI forward, step by step: projection, residual, routing, then the
    fast path M·round(g) or the slow path W·x per token."""
    x = np.asarray(x, dtype=np.float64)
    g = project(x, Vk)
    r = residual(x, Vk, g)
    xn = np.sqrt(np.sum(x * x, axis=1))
    rn = np.sqrt(np.sum(r * r, axis=1))
    rho = np.where(xn > 0, rn / np.where(xn > 0, xn, 1.0), 0.0)
    fast = route_fast(x, r, eps)
    M = image(W, Vk, dtype)
    g_hat = round_operand(g, dtype)
    y = np.where(fast[:, None], g_hat @ M.T, x @ W.T)
    # the device's fp32 sums: g_j within 2^-14 sum_i |V_ij x_i| and r_i within
    # 2^-14 sum_j |V_ij g_j| (the band convention of the gate); ||r|| moves by
    # at most the norms of those errors (V_k has orthonormal columns)
    dg = np.ldexp(np.abs(x) @ np.abs(Vk), -14)
    dr = np.ldexp(np.abs(g) @ np.abs(Vk).T, -14)
    band = (np.sqrt(np.sum(dg * dg, axis=1)) + np.sqrt(np.sum(dr * dr, axis=1))
            + np.ldexp(rn, -20)) / np.where(xn > 0, xn, 1.0)
    return GsiResult(y, g, g_hat, r, rho, fast, M, band)


def dense(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """The plain linear layer y = W x, what the slow path computes."""
    return np.asarray(x, dtype=np.float64) @ W.T


def forward_inputs(inp, T: Optional[int] = None) -> GsiResult:
    """Run ``forward`` on a synthetic GSI input bundle (duck-typed)."""
    def f64(t):
        return t.detach().to("cpu").double().numpy()
    x = f64(inp.x)
    if T is not None:
        x = x[:T]
    return forward(x, f64(inp.W), f64(inp.Vk), inp.wl.eps, inp.wl.dtype)
