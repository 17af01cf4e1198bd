"""Seeded synthetic inputs for the activation-sparse gated FFN.

This module only draws and quantises input tensors.  It holds none of the
method's arithmetic (no gate, no activation, no selection, no projection), so
that both the fp64 oracle and the CUDA path can be fed from it without sharing
any code with each other.

Every tensor is drawn from ``numpy.random.default_rng([seed, tensor_id])``
(PCG64 seeded through SeedSequence) in float32, scaled, and then rounded to the
operand dtype (bf16 by round-to-nearest-even through torch, or kept in fp32).

Tensor ids: x = 0, W_gate = 1, W_up = 2, W_down = 3, A = 4, B = 5, bias = 6,
nnz draw = 7, exact-grid sparsity pattern of A = 8, rotation V = 9.

Weight scales follow N(0, 1/fan_in): fan_in = d for W_gate, W_up and A, r for
B, and d_ff for W_down (the down projection sums over the d_ff neurons).  All
weights are stored neuron-major, i.e. W_gate, W_up and W_down are [d_ff][d]
row-major; row j belongs to neuron j.  A is [d][r] and B is [r][d_ff], so the
low-rank gate is x·A·B.

Workload recipes (the activation statistics that the pages' trained models
produce, stood in for by Gaussian draws):

* ``tiny_fp32``: d=256, d_ff=1024, T=64, fp32, ReLU, bias -1.2816 per neuron
  (P(N(0,1) > 1.2816) = 0.1000, about 90 % zeros), threshold 0, C = 128.
* ``decode_bf16``: d=4096, d_ff=14336, T in {1, 4, 8}, bf16, same gate
  statistics (about 90 % zeros), C = 32.
* ``lopa_bf16``: low-rank gate with r = d/8 = 512 (rank ratio 1/8 of the
  LoPA page), A ~ N(0, 1/d), B ~ N(0, 1/r) so x·A·B has unit variance; bias
  -1.2816 (about 90 % zeros); T = 32; C = 32.
* ``prefill_bf16``: d=2048, d_ff=8192, T=4096.  Per-token activity
  nnz_t = min(d_ff, round(exp(ln 60 + xi_t))), xi_t ~ N(0, 1) (lognormal,
  median 60, mean 60·e^0.5 = 98.9, i.e. about 98.8 % sparsity).  Realised by
  x_t = s_t·z_t with z_t ~ N(0, I), bias -beta (beta = 3) and
  s_t = beta / Phi^-1(1 - min(nnz_t/d_ff, 0.45)), so that
  P(g_tj > 0) = min(nnz_t/d_ff, 0.45).  C = 8, so heavy tokens overflow.
* ``wina_bf16``: d=4096, d_ff=14336, T=32, SiLU, no bias, keep the top
  k = round(0.35·14336) = 5018 neurons per token, C = 128.
* ``wina_fullh_bf16``: the same shapes and k, scored on the full gated
  product |sigma(g)·u|.
* ``wina_input_bf16``: the same shapes and k, after an orthogonal rotation V
  (a randomly signed and permuted Hadamard matrix over 64) and input-side
  selection of 2048 of the 4096 rotated input coordinates per token.

The optional ``exact_grid`` flag quantises every operand to a coarse dyadic
grid (x to multiples of 2^-4, weights to k·2^-e with |k| <= 255, the bias to
the 2^-14 accumulator grid) so that every fp32 partial sum of the gate and up
projections is exact in any order; parity runs use it to demand bit-exact
TwELL values as well as indices.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from statistics import NormalDist
from typing import Optional

import numpy as np
import torch

TID_X, TID_WGATE, TID_WUP, TID_WDOWN, TID_A, TID_B, TID_BIAS, TID_NNZ, TID_APAT, TID_V = range(10)


@dataclass(frozen=True)
class Workload:
    name: str
    d_model: int
    d_ff: int
    tokens: int
    dtype: str = "bf16"          # "bf16" or "fp32"
    mode: str = "relu_threshold"  # or "wina_topk"
    act: str = "relu"            # "relu" or "silu"
    rank: int = 0                # 0 = dense gate
    bias: Optional[float] = -1.2816
    threshold: float = 0.0
    k: int = 0
    tile_capacity: int = 32
    x_kind: str = "gauss"        # "gauss" or "lognormal_nnz"
    beta: float = 3.0            # prefill bias magnitude
    nnz_mu: float = math.log(60.0)
    nnz_sigma: float = 1.0
    nnz_cap_frac: float = 0.45
    exact_grid: bool = False
    seed: int = 0
    input_k: Optional[int] = None  # input-side WINA: input coordinates kept per token
    rotation: str = "none"         # "none", "signed_perm", "hadamard" or "orthogonal": a V [d][d]

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 256, 1024, 64, dtype="fp32", tile_capacity=128),
    "decode_bf16": Workload("decode_bf16", 4096, 14336, 8, tile_capacity=32),
    "lopa_bf16": Workload("lopa_bf16", 4096, 14336, 32, rank=512, tile_capacity=32),
    "prefill_bf16": Workload("prefill_bf16", 2048, 8192, 4096, tile_capacity=8,
                             x_kind="lognormal_nnz", bias=None),
    "wina_bf16": Workload("wina_bf16", 4096, 14336, 32, mode="wina_topk", act="silu",
                          bias=None, k=5018, tile_capacity=128),
    # WINA variants: the full-h score, and input-side selection (half of the
    # input coordinates) after an orthogonal rotation, on the WINA shapes
    "wina_fullh_bf16": Workload("wina_fullh_bf16", 4096, 14336, 32, mode="wina_full_h", act="silu",
                                bias=None, k=5018, tile_capacity=128),
    "wina_input_bf16": Workload("wina_input_bf16", 4096, 14336, 32, mode="wina_topk", act="silu",
                                bias=None, k=5018, tile_capacity=128, input_k=2048, rotation="hadamard"),
}


def _rng(seed: int, tid: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tid)])


def _normal(seed: int, tid: int, shape, scale: float) -> np.ndarray:
    a = _rng(seed, tid).standard_normal(int(np.prod(shape)), dtype=np.float32)
    a *= np.float32(scale)
    return a.reshape(shape)


def _to_dtype(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "fp32":
        return t.clone()
    raise ValueError(dtype)


def _grid(a: np.ndarray, e: int, kmax: int = 255) -> np.ndarray:
    """Quantise to integer multiples of 2^-e with |k| <= kmax (exact in bf16)."""
    k = np.clip(np.rint(a.astype(np.float64) * (2.0 ** e)), -kmax, kmax)
    return (k / (2.0 ** e)).astype(np.float32)


def _grid_exp(std: float) -> int:
    """Grid exponent e such that a N(0, std^2) draw spans about +-16 grid units
    per standard deviation (and fits |k| <= 255 with a 16-sigma margin)."""
    return int(round(math.log2(16.0 / std)))


@dataclass
class Inputs:
    """Host tensors for one workload.  Weights are neuron-major [d_ff][d]."""
    wl: Workload
    x: torch.Tensor
    W_gate: Optional[torch.Tensor]
    A: Optional[torch.Tensor]
    B: Optional[torch.Tensor]
    W_up: torch.Tensor
    W_down: torch.Tensor
    bias: Optional[torch.Tensor]          # fp32 [d_ff] or None
    nnz_target: Optional[np.ndarray] = None
    extra: dict = field(default_factory=dict)
    V: Optional[torch.Tensor] = None      # [d][d] orthogonalising rotation, or None


def rotation_matrix(kind: str, d: int, seed: int, dtype: str) -> torch.Tensor:
    """A seeded d x d rotation to orthogonalise with (an input of the method,
    like the weights): "signed_perm" is a permutation with random signs
    (exact in any dtype); "orthogonal" is the Q factor of a Gaussian matrix,
    rounded to the operand dtype (orthogonal up to that rounding)."""
    rng = _rng(seed, TID_V)
    if kind == "signed_perm":
        V = np.zeros((d, d), dtype=np.float32)
        V[np.arange(d), rng.permutation(d)] = rng.choice(np.array([-1.0, 1.0], dtype=np.float32), d)
    elif kind == "orthogonal":
        q, r = np.linalg.qr(rng.standard_normal((d, d)))
        V = (q * np.sign(np.diag(r))[None, :]).astype(np.float32)
    elif kind == "hadamard":
        # Sylvester's Hadamard matrix over sqrt(d), with its columns permuted
        # and signed at random: orthogonal, entries +-2^-m for d = 4^m, so x·V
        # and W·V of grid operands are exact fp32 sums
        m = int(round(math.log(d, 4)))
        if 4 ** m != d:
            raise ValueError("the Hadamard rotation needs d = 4^m")
        H = np.ones((1, 1), dtype=np.float32)
        while H.shape[0] < d:
            H = np.block([[H, H], [H, -H]])
        V = (H / np.float32(2 ** m))[:, rng.permutation(d)] * rng.choice(
            np.array([-1.0, 1.0], dtype=np.float32), d)[None, :]
    else:
        raise ValueError(kind)
    return _to_dtype(V, dtype)


def token_scales(wl: Workload, T: Optional[int] = None) -> tuple[np.ndarray, np.ndarray]:
    """Per-token activity targets and x scales of the lognormal-nnz recipe."""
    T = wl.tokens if T is None else T
    xi = _normal(wl.seed, TID_NNZ, (T,), 1.0).astype(np.float64)
    nnz = np.minimum(wl.d_ff, np.rint(np.exp(wl.nnz_mu + wl.nnz_sigma * xi)))
    nnz = np.maximum(nnz, 1.0)
    p = np.minimum(nnz / wl.d_ff, wl.nnz_cap_frac)
    inv = NormalDist()
    s = np.array([wl.beta / inv.inv_cdf(1.0 - pi) for pi in p])
    return nnz.astype(np.int64), s


def make_inputs(wl: Workload, T: Optional[int] = None, weights_only: bool = False,
                x_only: bool = False) -> Inputs:
    """Draw the seeded tensors of ``wl`` (optionally with a different token count)."""
    T = wl.tokens if T is None else T
    d, F, r, seed = wl.d_model, wl.d_ff, wl.rank, wl.seed
    eg = wl.exact_grid

    # activations
    nnz = None
    x = None
    if not weights_only:
        if wl.x_kind == "gauss":
            xa = _normal(seed, TID_X, (T, d), 1.0)
            if eg:
                xa = _grid(xa, 4)
        elif wl.x_kind == "lognormal_nnz":
            nnz, s = token_scales(wl, T)
            xa = _normal(seed, TID_X, (T, d), 1.0) * s[:, None].astype(np.float32)
            if eg:
                # x_t = s_t·z_t on the 2^-3 grid (s_t reaches about 24)
                xa = _grid(xa, 3, kmax=4095)
        else:
            raise ValueError(wl.x_kind)
        x = _to_dtype(xa, wl.dtype)
    if x_only:
        return Inputs(wl, x, None, None, None, None, None, None, nnz)

    def wmat(tid, shape, fan_in):
        std = 1.0 / math.sqrt(fan_in)
        a = _normal(seed, tid, shape, std)
        if eg:
            a = _grid(a, _grid_exp(std))
        return _to_dtype(a, wl.dtype)

    W_gate = A = B = None
    if r == 0:
        W_gate = wmat(TID_WGATE, (F, d), d)
    else:
        if eg:
            # exact-grid low-rank gate: every column of A holds 8 entries of
            # +-1/2 and zeros elsewhere, so each z = x·A is a sum of 8 grid
            # values, exact in fp32 and on the 2^-5 grid after bf16 rounding.
            rng = _rng(seed, TID_APAT)
            Aa = np.zeros((d, r), dtype=np.float32)
            for c in range(r):
                rows = rng.choice(d, size=8, replace=False)
                Aa[rows, c] = rng.choice(np.array([-0.5, 0.5], dtype=np.float32), size=8)
            A = _to_dtype(Aa, wl.dtype)
        else:
            A = wmat(TID_A, (d, r), d)
        B = wmat(TID_B, (r, F), r)
    W_up = wmat(TID_WUP, (F, d), d)
    W_down = wmat(TID_WDOWN, (F, d), F)

    bias = None
    if wl.x_kind == "lognormal_nnz":
        bias = torch.full((F,), -wl.beta, dtype=torch.float32)
    elif wl.bias is not None:
        b = wl.bias
        if eg:
            b = round(b * 2.0 ** 14) / 2.0 ** 14
        bias = torch.full((F,), b, dtype=torch.float32)
    V = rotation_matrix(wl.rotation, d, seed, wl.dtype) if wl.rotation != "none" else None
    return Inputs(wl, x, W_gate, A, B, W_up, W_down, bias, nnz, V=V)


def to_f64(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    """Exact decode of a bf16/fp32 tensor to a float64 numpy array."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


# ---------------------------------------------------------------------------
# gated subspace linear layer (GSI)
# ---------------------------------------------------------------------------
TID_GSI_W, TID_GSI_Q, TID_GSI_C, TID_GSI_E, TID_GSI_RHO = range(20, 25)


@dataclass(frozen=True)
class GsiWorkload:
    """A linear layer y = W x with W [d_out][d_in] and a k-column basis V_k
    of the activation subspace; tokens x_t = V_k c_t + Q_perp e_t with
    c_t ~ N(0, I_k), e_t a random direction of the orthogonal complement whose
    length gives the residual ratio rho_t = ||e_t|| / ||x_t|| a lognormal
    target (median rho_med, log-spread rho_sigma, capped at 0.95).  The basis
    and its complement are the columns of one orthogonal matrix Q: a Hadamard
    matrix over sqrt(d_in) with its columns permuted and signed at random
    (d_in = 4^m), so V_k is exact in bf16."""
    name: str
    d_in: int
    d_out: int
    k: int
    tokens: int
    eps: float = 0.10
    rho_med: float = 0.025
    rho_sigma: float = 0.5
    dtype: str = "bf16"
    exact_grid: bool = False
    seed: int = 0

    def with_(self, **kw) -> "GsiWorkload":
        return replace(self, **kw)


# GPT-J's MLP input projection (d = 4096, d_ff = 16384) at the page's working
# point k = 256, eps = 0.10 (99.8 % of its tokens took the fast path there;
# here P(rho > eps) = 1 - Phi(ln(0.1/0.025)/0.5) = 0.28 %), decode batches
GSI_WORKLOADS = {
    "gsi_bf16": GsiWorkload("gsi_bf16", 4096, 16384, 256, 8),
}


@dataclass
class GsiInputs:
    wl: GsiWorkload
    x: torch.Tensor        # [T][d_in]
    W: torch.Tensor        # [d_out][d_in]
    Vk: torch.Tensor       # [d_in][k]
    rho_target: np.ndarray


def make_gsi_inputs(wl: GsiWorkload, T: Optional[int] = None) -> GsiInputs:
    T = wl.tokens if T is None else T
    d, k, seed = wl.d_in, wl.k, wl.seed
    Q = rotation_matrix("hadamard", d, seed + 1000, "fp32").numpy().astype(np.float64)
    Vk = Q[:, :k]
    c = _normal(seed, TID_GSI_C, (T, k), 1.0).astype(np.float64)
    e = _normal(seed, TID_GSI_E, (T, d - k), 1.0).astype(np.float64)
    e /= np.linalg.norm(e, axis=1, keepdims=True)
    xi = _normal(seed, TID_GSI_RHO, (T,), 1.0).astype(np.float64)
    rho = np.minimum(wl.rho_med * np.exp(wl.rho_sigma * xi), 0.95)
    cn = np.linalg.norm(c, axis=1)
    e *= (rho * cn / np.sqrt(1.0 - rho * rho))[:, None]
    xa = (c @ Vk.T + e @ Q[:, k:].T).astype(np.float32)
    std = 1.0 / math.sqrt(d)
    Wa = _normal(seed, TID_GSI_W, (wl.d_out, d), std)
    if wl.exact_grid:
        xa = _grid(xa, 4, kmax=4095)
        Wa = _grid(Wa, _grid_exp(std))
    return GsiInputs(wl, _to_dtype(xa, wl.dtype), _to_dtype(Wa, wl.dtype),
                     _to_dtype(Vk.astype(np.float32), wl.dtype), rho)


# ---------------------------------------------------------------------------
# mixture of LoPA-gated sparse experts
# ---------------------------------------------------------------------------
TID_MOE_WR = 30


@dataclass(frozen=True)
class MoeWorkload:
    """E experts, each the low-rank-gated sparse FFN of ``lopa_bf16``'s
    recipe (its own seeded weights), a router W_r ~ N(0, 1/d) [E][d] and
    x ~ N(0, 1): the router logits are about N(0, 1), so tokens spread over
    the experts at random."""
    name: str
    d_model: int
    d_ff: int
    rank: int
    experts: int
    top_k: int
    tokens: int
    bias: Optional[float] = -1.2816
    threshold: float = 0.0
    tile_capacity: int = 32
    exact_grid: bool = False
    seed: int = 0

    def with_(self, **kw) -> "MoeWorkload":
        return replace(self, **kw)

    def expert_workload(self, e: int) -> Workload:
        return Workload(f"{self.name}.e{e}", self.d_model, self.d_ff, self.tokens, rank=self.rank,
                        bias=self.bias, threshold=self.threshold, tile_capacity=self.tile_capacity,
                        exact_grid=self.exact_grid, seed=self.seed * 1009 + 17 + e)


# Mixtral's layout (8 experts, 2 per token) on the decode shapes, LoPA gate
# rank d/8, about 90 % zeros per expert
MOE_WORKLOADS = {
    "moe_lopa_bf16": MoeWorkload("moe_lopa_bf16", 4096, 14336, 512, 8, 2, 8),
}


@dataclass
class MoeInputs:
    wl: MoeWorkload
    x: torch.Tensor                 # [T][d]
    W_r: torch.Tensor               # [E][d]
    experts: list                   # per expert: dict(A, B, W_up, W_down, bias)


def make_moe_inputs(wl: MoeWorkload, T: Optional[int] = None) -> MoeInputs:
    T = wl.tokens if T is None else T
    xa = _normal(wl.seed, TID_X, (T, wl.d_model), 1.0)
    std = 1.0 / math.sqrt(wl.d_model)
    Wr = _normal(wl.seed, TID_MOE_WR, (wl.experts, wl.d_model), std)
    if wl.exact_grid:
        xa = _grid(xa, 4)
        Wr = _grid(Wr, _grid_exp(std))
    ex = []
    for e in range(wl.experts):
        inp = make_inputs(wl.expert_workload(e), weights_only=True)
        ex.append({"A": inp.A, "B": inp.B, "W_up": inp.W_up, "W_down": inp.W_down, "bias": inp.bias})
    return MoeInputs(wl, _to_dtype(xa, "bf16"), _to_dtype(Wr, "bf16"), ex)


# ---------------------------------------------------------------------------
# upstream gradient for the backward pass
# ---------------------------------------------------------------------------
TID_DY = 40


def upstream_grad(wl: Workload, T: Optional[int] = None) -> torch.Tensor:
    """dy = dL/dy [T][d_model] fp32 ~ N(0, 1), seeded by the workload."""
    T = wl.tokens if T is None else T
    return torch.from_numpy(_normal(wl.seed, TID_DY, (T, wl.d_model), 1.0))
