"""Pins of the oracle's backward pass (CPU only).

Source: "Sparser, Faster, Lighter Transformer Language Models" (news
article), section "Hybrid 應對非均勻稀疏" (the training step over the sparse
format, heavy tokens through a dense channel); the gradients are the chain
rule of the forward with the selection held fixed and the rounding of the
stored value passed straight through.  Tied to central finite differences of
the forward itself (the exact-arithmetic variant, with every activation far
from the threshold so the selection cannot move), to a case worked by hand
(tests/golden/hand_worked.json, "backward"), and to exact zeros for neurons
that are not kept.  Planted mistakes at the end must each fail a pin.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _B():
    import oracle.backward as B  # looked up at call time
    return B


def _case(seed, act, T=3, d=5, F=128, tau=0.1):
    rng = np.random.default_rng(seed)
    while True:
        x = rng.standard_normal((T, d))
        Wg = rng.standard_normal((F, d)) / np.sqrt(d)
        Wu = rng.standard_normal((F, d)) / np.sqrt(d)
        Wd = rng.standard_normal((F, d)) / np.sqrt(F)
        b = rng.standard_normal(F) * 0.3 - 0.3
        a = oracle.activate(x @ Wg.T + b, act)
        if np.abs(np.abs(a) - tau).min() > 1e-3:   # no activation near the threshold
            return x, Wg, Wu, Wd, b, tau


def _loss(x, Wg, Wu, Wd, b, tau, act, dy):
    return float(np.sum(dy * oracle.forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="fp64", act=act,
                                            threshold=tau, C=128).y))


@pytest.mark.parametrize("act", ["relu", "silu"])
def test_finite_differences(act):
    x, Wg, Wu, Wd, b, tau = _case(1 if act == "relu" else 2, act)
    dy = np.random.default_rng(7).standard_normal((x.shape[0], x.shape[1]))
    gr = _B().backward(x, Wg, Wu, Wd, dy, bias=b, dtype="fp64", act=act, threshold=tau)
    assert 0 < gr.keep.sum() < gr.keep.size
    eps = 1e-6
    rng = np.random.default_rng(3)

    def fd(arr, idx):
        old = arr[idx]
        arr[idx] = old + eps
        lp = _loss(x, Wg, Wu, Wd, b, tau, act, dy)
        arr[idx] = old - eps
        lm = _loss(x, Wg, Wu, Wd, b, tau, act, dy)
        arr[idx] = old
        return (lp - lm) / (2 * eps)

    for name, arr, grad in (("x", x, gr.dx), ("W_gate", Wg, gr.dW_gate), ("W_up", Wu, gr.dW_up),
                            ("W_down", Wd, gr.dW_down), ("b", b, gr.db)):
        kept_rows = np.nonzero(gr.keep.any(axis=0))[0]
        picks = [tuple(rng.integers(0, s) for s in arr.shape) for _ in range(12)]
        if name != "x":   # also rows of kept neurons, where the gradient is not zero
            picks += [(j,) + tuple(rng.integers(0, s) for s in arr.shape[1:]) for j in kept_rows[:12]]
        for idx in picks:
            want = fd(arr, idx)
            assert abs(grad[idx] - want) <= 1e-6 * max(1.0, abs(want)), (name, idx, grad[idx], want)


def test_hand_worked():
    d = json.load(open(os.path.join(GOLDEN, "hand_worked.json")))
    F, dm = 128, 2
    x = np.array(d["x"])
    Wg = np.zeros((F, dm)); Wu = np.zeros((F, dm)); Wd = np.zeros((F, dm))
    b = np.full(F, -1.0)
    for j, r in d["rows"].items():
        j = int(j)
        Wg[j] = r["gate"]; Wu[j] = r["up"]; Wd[j] = r["down"]; b[j] = r["bias"]
    ref = d["backward"]
    gr = _B().backward(x, Wg, Wu, Wd, np.array(ref["dy"]), bias=b, dtype="bf16", act="relu", threshold=0.0)
    np.testing.assert_array_equal(gr.dx, np.array(ref["dx"]))
    for name in ("dW_down", "dW_up", "dW_gate"):
        want = np.zeros((F, dm))
        for j, row in ref[name].items():
            want[int(j)] = row
        np.testing.assert_array_equal(getattr(gr, name), want, err_msg=name)
    want_b = np.zeros(F)
    for j, v in ref["db"].items():
        want_b[int(j)] = v
    np.testing.assert_array_equal(gr.db, want_b)


def test_neurons_not_kept_get_no_gradient():
    x, Wg, Wu, Wd, b, tau = _case(5, "silu")
    dy = np.ones((x.shape[0], x.shape[1]))
    gr = _B().backward(x, Wg, Wu, Wd, dy, bias=b, dtype="bf16", act="silu", threshold=tau)
    off = ~gr.keep.any(axis=0)
    assert off.any()
    for arr in (gr.dW_gate, gr.dW_up, gr.dW_down):
        assert np.all(arr[off] == 0)
    assert np.all(gr.db[off] == 0)


@pytest.mark.parametrize("mutation", ["no_slope", "du_with_u", "down_with_dh", "dx_no_gate", "dh_unmasked"])
def test_backward_pins_catch_planted_mistakes(monkeypatch, mutation):
    import oracle.backward as B
    orig = B.backward

    def patched(x, Wg, Wu, Wd, dy, *, bias=None, dtype="bf16", act="relu", threshold=0.0, keep=None):
        g = oracle.gate_dense(np.asarray(x, float), Wg, bias)
        a = oracle.activate(g, act)
        kp = oracle.keep_threshold(a, threshold) if keep is None else keep
        v = oracle.round_operand(a, dtype)
        u = x @ Wu.T
        h = np.where(kp, v * u, 0.0)
        dh = dy @ Wd.T if mutation == "dh_unmasked" else np.where(kp, dy @ Wd.T, 0.0)
        du = dh * (u if mutation == "du_with_u" else v)
        dv = dh * u
        sl = 1.0 if mutation == "no_slope" else B.act_slope(g, act)
        dg = np.where(kp, dv * sl, 0.0)
        dx = du @ Wu + (0 if mutation == "dx_no_gate" else dg @ Wg)
        dWd = (dh.T if mutation == "down_with_dh" else h.T) @ dy
        return B.Grads(dx=dx, dW_gate=dg.T @ x, dW_up=du.T @ x, dW_down=dWd, db=dg.sum(0), keep=kp, h=h,
                       du=du, dg=dg)
    monkeypatch.setattr(B, "backward", patched)
    failures = 0
    for test in (lambda: test_finite_differences("relu"), lambda: test_finite_differences("silu"),
                 test_hand_worked, test_neurons_not_kept_get_no_gradient):
        try:
            test()
        except AssertionError:
            failures += 1
    assert failures > 0, mutation
    assert orig is not None
