"""GPU parity of the sparse backward (TwELL news article, section "Hybrid
應對非均勻稀疏": training over the sparse format) through the C ABI against
the fp64 oracle's backward.

Rules: on exact-grid operands the forward's selection equals the oracle's,
so every gradient is compared whole; on Gaussian operands the pairs whose
gate lies in the forward's decision band may be selected either way, so the
dW rows of neurons and the dx rows of tokens that own such a pair are left
out, and the rest must match.  Gradients within max|err| / max|ref| <= 2e-3
(the bf16 parity tolerance; the arithmetic is fp32 on bf16 operands).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import oracle.backward as OB
import synth
from activation_sparse_gated_relu_b200 import SffnError

from parity_util import ambiguous, make_ffn, rel_err, to_dev

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
NAMES = ("dx", "dW_gate", "dW_up", "dW_down", "d_bias")


def _run(inp, T, path="rows", C=None):
    ffn = make_ffn(inp, max_tokens=T, path=path, C=C, backward=True)
    try:
        x = to_dev(inp.x[:T])
        ffn.forward(x)
        dy = to_dev(synth.upstream_grad(inp.wl, T))
        g = ffn.backward(x, dy)
        torch.cuda.synchronize()
        assert ffn.read_status() == 0
        return {k: v.double().cpu().numpy() for k, v in g.items()}
    finally:
        ffn.close()


def _check(inp, T, exact, path="rows", C=None):
    wl = inp.wl
    dy = synth.upstream_grad(wl, T).double().numpy()
    ref = OB.backward_inputs(inp, dy, T=T)
    got = _run(inp, T, path, C)
    want = {"dx": ref.dx, "dW_gate": ref.dW_gate, "dW_up": ref.dW_up, "dW_down": ref.dW_down, "d_bias": ref.db}
    if exact:
        rows_ok = np.ones(wl.d_ff, dtype=bool)
        tok_ok = np.ones(T, dtype=bool)
    else:
        res = oracle.forward_inputs(inp, T=T)
        amb = ambiguous(res, wl.mode, wl.threshold, wl.k, False)
        rows_ok = ~amb.any(axis=0)
        tok_ok = ~amb.any(axis=1)
        assert rows_ok.mean() > 0.25 and tok_ok.mean() > 0.25
    for k in NAMES:
        sel = tok_ok if k == "dx" else rows_ok
        e = rel_err(got[k][sel], want[k][sel])
        assert e <= 2e-3, (k, e)
    return got, want


@pytest.mark.parametrize("T", [8, 32])
def test_backward_exact_grid_small(T):
    inp = synth.make_inputs(synth.Workload("small", 256, 512, T, tile_capacity=32, exact_grid=True))
    _check(inp, T, exact=True)


@pytest.mark.parametrize("C", [8, 16])
def test_backward_heavy_tokens_exact_grid(C):
    # a small tile capacity makes most tokens overflow: their gradients take
    # the dense tensor-core channel, the others the sparse passes
    inp = synth.make_inputs(synth.Workload("small", 256, 512, 32, tile_capacity=C, exact_grid=True))
    res = oracle.forward_inputs(inp, T=32)
    assert res.overflow.any() and (C == 8 or not res.overflow.all())
    _check(inp, 32, exact=True, C=C)


def test_backward_silu_threshold_gaussian():
    inp = synth.make_inputs(synth.Workload("small", 512, 1024, 40, tile_capacity=16, act="silu",
                                           threshold=0.3, bias=None))
    _check(inp, 40, exact=False)


def test_backward_after_single_launch_decode():
    inp = synth.make_inputs(W["decode_bf16"].with_(d_model=1024, d_ff=4096, tile_capacity=8))
    _check(inp, 8, exact=False)


def test_backward_prefill_config():
    # the training shape (d 2048, d_ff 8192, 4096 tokens, heavy-tailed
    # activity, C = 8 so heavy tokens overflow): heavy tokens' pairs are
    # split over several chunks of the token pass
    inp = synth.make_inputs(W["prefill_bf16"])
    _check(inp, 4096, exact=False)


def test_backward_requires_the_flag_and_the_forward():
    inp = synth.make_inputs(synth.Workload("small", 256, 512, 8, tile_capacity=32))
    x = to_dev(inp.x)
    dy = to_dev(synth.upstream_grad(inp.wl, 8))
    plain = make_ffn(inp, max_tokens=8)
    try:
        plain.forward(x)
        with pytest.raises(SffnError):
            plain.backward(x, dy)
    finally:
        plain.close()
    ffn = make_ffn(inp, max_tokens=8, backward=True)
    try:
        ffn.forward(x)
        with pytest.raises(SffnError):          # T differs from the last forward's
            ffn.backward(x[:4], dy[:4])
        a = ffn.backward(x, dy)
        b = ffn.backward(x, dy)
        torch.cuda.synchronize()
        for k in ("dW_gate", "dW_up", "dW_down", "d_bias"):   # the neuron pass is deterministic
            assert torch.equal(a[k], b[k]), k
    finally:
        ffn.close()
