"""GPU parity of the gated subspace linear layer (GSI technical summary,
sections 2.1 and 2.2) through the C ABI against the fp64 oracle.

Rules: the per-token route (fast iff ||r||^2 < eps^2 ||x||^2) must match the
oracle's for every token whose residual ratio lies outside the oracle's
decision band; a token inside the band may take either path, and its y must
then match the oracle's y for the path it took.  y within max|y - y_ref| /
max|y_ref| <= 2e-3 per path.  On exact-grid operands (Hadamard basis,
entries +-2^-6) the projection g and the cached image M must be bit-exact.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.gsi as G
import synth
from activation_sparse_gated_relu_b200 import GsiLinear

from parity_util import rel_err, to_dev

pytestmark = pytest.mark.gpu

GW = synth.GSI_WORKLOADS


def _run(inp, T, max_tokens=None):
    lay = GsiLinear(to_dev(inp.W), to_dev(inp.Vk), inp.wl.eps, max_tokens=max_tokens or T)
    try:
        x = to_dev(inp.x[:T])
        y = torch.full((T, inp.wl.d_out), float("nan"), dtype=torch.float32, device="cuda")
        lay.forward(x, y)
        torch.cuda.synchronize()
        dbg = lay.debug(T)
        out = {"y": y.double().cpu().numpy(), "n_slow": lay.n_slow(),
               "g": dbg["g"].double().cpu().numpy(), "rn2": dbg["rn2"].double().cpu().numpy(),
               "xn2": dbg["xn2"].double().cpu().numpy(), "M": dbg["M"].double().cpu().numpy()}
    finally:
        lay.close()
    return out


def _check(inp, T, max_tokens=None):
    res = G.forward_inputs(inp, T=T)
    got = _run(inp, T, max_tokens)
    assert np.all(np.isfinite(got["y"])), "y not fully written"
    eps2 = np.float32(inp.wl.eps) * np.float32(inp.wl.eps)
    fast_dev = got["rn2"] < eps2 * got["xn2"]
    amb = np.abs(res.rho - inp.wl.eps) <= res.rho_band
    assert np.all((fast_dev == res.fast) | amb), "routes differ outside the band"
    assert got["n_slow"] == int((~fast_dev).sum())
    x = synth.to_f64(inp.x[:T])
    y_fast = res.g_hat @ res.M.T
    y_slow = x @ synth.to_f64(inp.W).T
    ref = np.where(fast_dev[:, None], y_fast, y_slow)
    scale = np.abs(np.concatenate([y_fast, y_slow])).max()
    assert np.abs(got["y"] - ref).max() <= 2e-3 * scale
    return res, got, fast_dev


def test_gsi_config():
    inp = synth.make_gsi_inputs(GW["gsi_bf16"])
    res, got, fast = _check(inp, GW["gsi_bf16"].tokens)


def test_gsi_full_size_batch_with_slow_tokens():
    inp = synth.make_gsi_inputs(GW["gsi_bf16"], T=64)
    res, got, fast = _check(inp, 64)
    assert (~fast).any() and fast.any()


@pytest.mark.parametrize("T", [1, 5, 8, 13, 64])
def test_gsi_mixed_routes(T):
    # a wide spread of residual ratios: about half the tokens on each path
    wl = GW["gsi_bf16"].with_(d_in=1024, d_out=3072, k=128, rho_med=0.1, rho_sigma=1.0)
    inp = synth.make_gsi_inputs(wl, T=T)
    res, got, fast = _check(inp, T, max_tokens=64)
    if T >= 13:
        assert (~fast).any() and fast.any()


def test_gsi_exact_grid_projection_and_image():
    wl = GW["gsi_bf16"].with_(d_in=1024, d_out=2048, k=128, exact_grid=True, rho_med=0.08)
    inp = synth.make_gsi_inputs(wl, T=16)
    res, got, fast = _check(inp, 16)
    np.testing.assert_array_equal(got["g"], res.g)        # exact fp32 sums of grid products
    np.testing.assert_array_equal(got["M"], res.M)


def test_gsi_eps_limits_and_zero_token():
    wl = GW["gsi_bf16"].with_(d_in=1024, d_out=2048, k=64)
    inp = synth.make_gsi_inputs(wl, T=8)
    inp.x[3] = 0.0
    slow = synth.GsiInputs(wl.with_(eps=0.0), inp.x, inp.W, inp.Vk, inp.rho_target)
    res, got, fast = _check(slow, 8)
    assert not fast.any() and got["n_slow"] == 8
    np.testing.assert_array_equal(got["y"][3], 0.0)
    allfast = synth.GsiInputs(wl.with_(eps=1e30), inp.x, inp.W, inp.Vk, inp.rho_target)
    res, got, fast = _check(allfast, 8)
    assert fast.sum() == 7 and not fast[3]                 # x = 0 stays on the slow path
