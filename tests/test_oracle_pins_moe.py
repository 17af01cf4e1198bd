"""Pins of the oracle's mixture of LoPA-gated sparse experts (CPU only).

Source: "Meta FAIR and Inria's LoPA Gating Hits 3.31x Real GPU Speedup for
LLM Inference", sections "Model Casting and Quality at 90% Sparsity" (MoE
compatibility) and "How LoPA Gating Restructures FFN Computation" (the
low-rank gate); routing read as Mixtral's (top_k by logit, softmax over the
kept logits).  Tied to a hand-worked case (tests/golden/moe_hand_worked.json),
to the single-expert reduction, to top_k = E giving the full softmax, to
invariance under renumbering the experts, and to the router's tie rule;
planted mistakes at the end must each fail one of them.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _M():
    import oracle.moe as M  # looked up at call time, as the forward does
    return M


def _hand():
    d = json.load(open(os.path.join(GOLDEN, "moe_hand_worked.json")))
    F, dm = 128, 2
    ex = []
    for j, gcol, up, down in ((5, [1.0, 0.0], [1.0, 1.0], [1.0, 0.0]), (9, [0.0, 1.0], [0.0, 2.0], [0.0, 1.0])):
        B = np.zeros((dm, F)); B[:, j] = gcol
        Wu = np.zeros((F, dm)); Wu[j] = up
        Wd = np.zeros((F, dm)); Wd[j] = down
        b = np.full(F, -1.0); b[j] = 0.0
        ex.append({"A": np.eye(dm), "B": B, "W_up": Wu, "W_down": Wd, "bias": b})
    return d, np.array(d["x"]), np.eye(2), ex


@pytest.mark.parametrize("k", [1, 2])
def test_hand_worked(k):
    d, x, Wr, ex = _hand()
    ref = d["top%d" % k]
    res = _M().forward(x, Wr, ex, k, C=8)
    assert res.sel.tolist() == ref["sel"]
    np.testing.assert_allclose(res.y, np.array(ref["y"]), rtol=1e-15, atol=1e-15)


def _small(E=4, k=2, T=6, seed=3):
    wl = synth.MOE_WORKLOADS["moe_lopa_bf16"].with_(d_model=64, d_ff=256, rank=16, experts=E, top_k=k,
                                                    tokens=T, seed=seed)
    inp = synth.make_moe_inputs(wl)
    f = synth.to_f64
    ex = [{kk: f(v) for kk, v in e.items()} for e in inp.experts]
    return f(inp.x), f(inp.W_r), ex


def test_single_expert_is_the_plain_ffn():
    x, Wr, ex = _small(E=1, k=1)
    res = _M().forward(x, Wr, ex, 1)
    plain = oracle.forward(x, ex[0]["W_up"], ex[0]["W_down"], A=ex[0]["A"], B=ex[0]["B"], bias=ex[0]["bias"])
    np.testing.assert_array_equal(res.y, plain.y)
    assert np.all(res.w == 1.0)


def test_all_experts_take_the_full_softmax():
    x, Wr, ex = _small(E=4, k=4)
    res = _M().forward(x, Wr, ex, 4)
    l = x @ Wr.T
    p = np.exp(l - l.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    y = sum(p[:, e:e + 1] * oracle.forward(x, ex[e]["W_up"], ex[e]["W_down"], A=ex[e]["A"], B=ex[e]["B"],
                                           bias=ex[e]["bias"]).y for e in range(4))
    np.testing.assert_allclose(res.y, y, rtol=1e-13, atol=1e-13 * np.abs(y).max())


def test_renumbering_experts_changes_nothing():
    x, Wr, ex = _small(E=5, k=2)
    perm = [3, 0, 4, 1, 2]
    a = _M().forward(x, Wr, ex, 2)
    b = _M().forward(x, Wr[perm], [ex[p] for p in perm], 2)
    np.testing.assert_allclose(a.y, b.y, rtol=1e-13, atol=1e-13 * np.abs(a.y).max())
    assert np.array_equal(np.array(perm)[b.sel], a.sel)


def test_router_selects_by_sorting():
    rng = np.random.default_rng(0)
    l = rng.integers(-3, 4, size=(40, 6)).astype(float)     # many ties
    sel = _M().select_experts(l, 3)
    for t in range(40):
        want = sorted(range(6), key=lambda e: (-l[t, e], e))[:3]
        assert list(sel[t]) == want


@pytest.mark.parametrize("mutation", ["ties_high", "softmax_all", "unnormalised", "smallest"])
def test_moe_pins_catch_planted_mistakes(monkeypatch, mutation):
    import oracle.moe as M
    if mutation == "ties_high":
        monkeypatch.setattr(M, "select_experts", lambda l, k: np.stack(
            [np.lexsort((-np.arange(l.shape[1]), -l[t]))[:k] for t in range(l.shape[0])]))
    elif mutation == "softmax_all":
        def sm_all(l, sel):
            p = np.exp(l - l.max(1, keepdims=True))
            p /= p.sum(1, keepdims=True)
            return np.take_along_axis(p, sel, axis=1)
        monkeypatch.setattr(M, "expert_weights", sm_all)
    elif mutation == "unnormalised":
        monkeypatch.setattr(M, "expert_weights", lambda l, sel: np.exp(np.take_along_axis(l, sel, axis=1)))
    elif mutation == "smallest":
        monkeypatch.setattr(M, "select_experts", lambda l, k: np.stack(
            [np.lexsort((np.arange(l.shape[1]), l[t]))[:k] for t in range(l.shape[0])]))
    failures = 0
    for test in (lambda: test_hand_worked(1), lambda: test_hand_worked(2), test_single_expert_is_the_plain_ffn,
                 test_all_experts_take_the_full_softmax, test_router_selects_by_sorting):
        try:
            test()
        except AssertionError:
            failures += 1
    assert failures > 0, mutation
