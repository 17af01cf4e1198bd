"""Pins of the oracle's gated subspace linear layer (CPU only).

Source: "Gated Subspace Inference for Transformer Acceleration" (technical
summary), sections 2.1 and 2.2.  The oracle is tied to a case worked by hand
(tests/golden/gsi_hand_worked.json), to the decomposition W x = M g + W r, to
the limits eps = 0 (every token slow: the plain layer) and eps = infinity
(every token fast), to the page's Theorem 4 bound on the fast path's error
(with numpy's spectral norm), to the strictness of the router, and to the
closed-form fast fraction of the synthetic recipe.  Planted mistakes at the
end must each fail one of these.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest

import oracle.gsi
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _G():
    import oracle.gsi as G  # looked up at call time, as the forward does
    return G


def test_hand_worked():
    d = json.load(open(os.path.join(GOLDEN, "gsi_hand_worked.json")))
    res = _G().forward(np.array(d["x"]), np.array(d["W"]), np.array(d["Vk"]), d["eps"], "bf16")
    assert res.fast.tolist() == d["fast"]
    np.testing.assert_array_equal(res.g_hat, np.array(d["g_hat"]))
    np.testing.assert_allclose(res.y, np.array(d["y"]), rtol=1e-13, atol=1e-13)


def _random_case(seed, T=12, d=64, k=8, d_out=48):
    rng = np.random.default_rng(seed)
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    Vk = Q[:, :k]
    W = rng.standard_normal((d_out, d)) / math.sqrt(d)
    c = rng.standard_normal((T, k))
    e = rng.standard_normal((T, d - k)) * rng.uniform(0.0, 0.3, size=(T, 1))
    x = c @ Vk.T + e @ Q[:, k:].T
    return x, W, Vk, Q


def test_decomposition_is_exact():
    # section 2.1: W x = (W V_k)(V_k^T x) + W r, with the unrounded image
    x, W, Vk, _ = _random_case(0)
    G = _G()
    g = G.project(x, Vk)
    r = G.residual(x, Vk, g)
    np.testing.assert_allclose(g @ (W @ Vk).T + r @ W.T, x @ W.T, rtol=0, atol=1e-12)
    # r is orthogonal to the subspace
    assert np.abs(r @ Vk).max() < 1e-12


def test_eps_limits():
    x, W, Vk, _ = _random_case(1)
    G = _G()
    slow = G.forward(x, W, Vk, 0.0, "bf16")
    assert not slow.fast.any()
    np.testing.assert_array_equal(slow.y, x @ W.T)
    fast = G.forward(x, W, Vk, math.inf, "bf16")
    assert fast.fast.all()
    np.testing.assert_array_equal(fast.y, fast.g_hat @ fast.M.T)


def test_theorem_4_bound_on_fast_tokens():
    # ||M g - W x|| = ||W r|| <= ||W||_2 ||r|| < ||W||_2 eps ||x|| for a fast token
    # (the unrounded image and projection, as the theorem states them)
    G = _G()
    for seed in range(5):
        x, W, Vk, _ = _random_case(10 + seed)
        eps = 0.15
        res = G.forward(x, W, Vk, eps, "fp32")
        assert res.fast.any() and (~res.fast).any()
        w2 = np.linalg.norm(W, 2)
        exact_fast = res.g @ (W @ Vk).T
        err = np.linalg.norm(exact_fast - x @ W.T, axis=1)
        bound = w2 * eps * np.linalg.norm(x, axis=1)
        assert np.all(err[res.fast] < bound[res.fast])
        # the ratio routes: rho < eps exactly on the fast tokens
        assert np.array_equal(res.fast, res.rho < eps)


def test_router_is_strict():
    # x in the complement: rho = 1; eps = 1 keeps it on the slow path
    G = _G()
    Vk = np.array([[1.0], [0.0]])
    W = np.array([[1.0, 2.0], [3.0, 4.0]])
    res = G.forward(np.array([[0.0, 1.0], [2.0, 0.0]]), W, Vk, 1.0, "bf16")
    assert res.fast.tolist() == [False, True]
    np.testing.assert_array_equal(res.y, [[2.0, 4.0], [2.0, 6.0]])


def test_recipe_fast_fraction_closed_form():
    # rho_t is lognormal(ln 0.025, 0.5) by construction (up to the bf16
    # rounding of x), so P(slow) = 1 - Phi(ln(eps / 0.025) / 0.5) = 0.28 %
    wl = synth.GSI_WORKLOADS["gsi_bf16"].with_(d_out=128)
    inp = synth.make_gsi_inputs(wl, T=512)
    res = _G().forward(synth.to_f64(inp.x), synth.to_f64(inp.W), synth.to_f64(inp.Vk), wl.eps)
    assert np.all(np.abs(res.rho - inp.rho_target) <= 0.002 + 0.01 * inp.rho_target)
    p_slow = 0.5 * math.erfc(math.log(wl.eps / wl.rho_med) / wl.rho_sigma / math.sqrt(2))
    assert abs(p_slow - 0.0028) < 2e-4
    n_slow = int((~res.fast).sum())
    assert n_slow <= 512 * p_slow + 5 * math.sqrt(512 * p_slow) + 1


@pytest.mark.parametrize("mutation", ["nonstrict", "g_unrounded", "image_unrounded", "slow_via_image",
                                      "residual_sign"])
def test_gsi_pins_catch_planted_mistakes(monkeypatch, mutation):
    import oracle.gsi as G
    if mutation == "nonstrict":
        monkeypatch.setattr(G, "route_fast", lambda x, r, eps: np.sum(r * r, axis=1)
                            <= (eps * eps) * np.sum(x * x, axis=1))
    elif mutation == "g_unrounded":
        monkeypatch.setattr(G, "round_operand", lambda a, dt: a)
    elif mutation == "image_unrounded":
        monkeypatch.setattr(G, "image", lambda W, Vk, dt: W @ Vk)
    elif mutation == "slow_via_image":
        orig = G.forward

        def bad(x, W, Vk, eps, dtype="bf16"):
            res = orig(x, W, Vk, eps, dtype)
            res.y = res.g_hat @ res.M.T + res.r @ W.T
            return res
        monkeypatch.setattr(G, "forward", bad)
    elif mutation == "residual_sign":
        monkeypatch.setattr(G, "residual", lambda x, Vk, g: x + g @ Vk.T)
    failures = 0
    for test in (test_hand_worked, test_decomposition_is_exact, test_eps_limits,
                 test_theorem_4_bound_on_fast_tokens, test_router_is_strict):
        try:
            test()
        except AssertionError:
            failures += 1
    assert failures > 0, mutation
