"""Pins of the oracle's WINA variants (CPU only): the full-h score, input-side
selection and the orthogonalising rotation (WINA framework explainer,
sections 3.1 to 3.3).

Each check ties the oracle to something outside its own code: the optimality
statement of Lemma 3.1 checked by brute force over every k-subset (exact
dyadic arithmetic, orthogonal weight columns built from a Hadamard matrix),
values worked by hand (tests/golden/hand_worked.json), reductions to the
plain forward, and invariants of the SVD and of signed permutations.  Planted
mistakes at the end must each fail one of them.
"""
from __future__ import annotations

import itertools
import json
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hadamard(n: int) -> np.ndarray:
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def _hand():
    d = json.load(open(os.path.join(GOLDEN, "hand_worked.json")))
    F, dm = 128, 2
    x = np.array(d["x"], dtype=np.float64)
    Wg = np.zeros((F, dm)); Wu = np.zeros((F, dm)); Wd = np.zeros((F, dm))
    b = np.full(F, -1.0)
    for j, r in d["rows"].items():
        j = int(j)
        Wg[j] = r["gate"]; Wu[j] = r["up"]; Wd[j] = r["down"]; b[j] = r["bias"]
    return d, x, Wg, Wu, Wd, b


def _F():
    import oracle.ffn as F  # looked up at call time, as the oracle's forward does
    return F


# ----------------------------------------------------------------------------
# hand-worked
# ----------------------------------------------------------------------------
def test_hand_worked_full_h():
    d, x, Wg, Wu, Wd, b = _hand()
    ref = d["wina_full_h_relu"]["k2"]
    res = _F().forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", mode="wina_full_h", act="relu",
                       k=2, C=128)
    for t in range(2):
        assert list(np.nonzero(res.keep[t])[0]) == ref["kept"][t]
    np.testing.assert_array_equal(res.y, np.array(ref["y"]))


def test_hand_worked_input_side():
    d, x, Wg, Wu, Wd, b = _hand()
    ref = d["input_side"]
    F = _F()
    np.testing.assert_array_equal(F.input_col_norms(Wg, Wu), ref["col_norms"])
    res = F.forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", C=128, input_k=ref["k_in"])
    np.testing.assert_array_equal(res.x_used, np.array(ref["x_sel"]))
    for t in range(2):
        assert list(np.nonzero(res.keep[t])[0]) == ref["kept"][t]
    np.testing.assert_array_equal(res.y, np.array(ref["y"]))


def test_full_h_scores_the_unrounded_activation():
    # neuron 5: a = 1 + 2^-8 (bf16 value 1), u = 1, n = 1 -> s = 1.00390625;
    # neuron 6: a = 1, u = 1, n = 1 + 2^-9 -> s = 1.001953125.  The unrounded
    # activation ranks 5 first; its bf16 value would rank 6 first
    F, dm = 128, 2
    x = np.array([[1.0, 2.0 ** -8]])
    Wg = np.zeros((F, dm)); Wu = np.zeros((F, dm)); Wd = np.zeros((F, dm))
    b = np.full(F, -1.0)
    Wg[5] = [1.0, 1.0]; b[5] = 0.0; Wu[5] = [1.0, 0.0]; Wd[5] = [1.0, 0.0]
    Wg[6] = [1.0, 0.0]; b[6] = 0.0; Wu[6] = [1.0, 0.0]; Wd[6] = [0.0, 1.0 + 2.0 ** -9]
    res = _F().forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", mode="wina_full_h", act="relu",
                       k=1, C=128)
    assert list(np.nonzero(res.keep[0])[0]) == [5]
    np.testing.assert_array_equal(res.y, [[1.0, 0.0]])   # v = bf16(1 + 2^-8) = 1


# ----------------------------------------------------------------------------
# Lemma 3.1 by brute force: with orthogonal weight columns, keeping the k
# largest |h_j|·||w_j|| minimises ||W h - W h_S|| over every k-subset S
# ----------------------------------------------------------------------------
def _orthogonal_rows(rng, F, d):
    """F mutually orthogonal rows in R^d (F <= d): Hadamard rows, each scaled
    by its own power of two (exact in fp64)."""
    H = _hadamard(d)[:F]
    return H * (2.0 ** rng.integers(-3, 3, size=F))[:, None]


@pytest.mark.parametrize("seed,k", [(0, 3), (1, 4), (2, 5)])
def test_lemma_3_1_full_h_bruteforce(seed, k):
    rng = np.random.default_rng(seed)
    T, d, F = 3, 16, 10
    x = rng.integers(-8, 9, size=(T, d)) / 8.0
    Wg = rng.integers(-8, 9, size=(F, d)) / 16.0
    Wu = rng.integers(-8, 9, size=(F, d)) / 16.0
    Wd = _orthogonal_rows(rng, F, d)          # neuron-major: rows are the weight columns
    b = np.full(F, 0.25)
    res = _F().forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", mode="wina_full_h", act="relu",
                       k=k, C=128)
    g = x @ Wg.T + b
    h = np.maximum(g, 0) * (x @ Wu.T)           # the full gated product, unrounded
    for t in range(T):
        y_all = h[t] @ Wd
        best = min(itertools.combinations(range(F), k),
                   key=lambda S: (float(np.sum((y_all - h[t, list(S)] @ Wd[list(S)]) ** 2)), S))
        errs = sorted(float(np.sum((y_all - h[t, list(S)] @ Wd[list(S)]) ** 2))
                      for S in itertools.combinations(range(F), k))
        assert errs[0] < errs[1] or k >= np.count_nonzero(h[t]), "no unique optimum: bad test draw"
        assert set(np.nonzero(res.keep[t])[0]) == set(best)


@pytest.mark.parametrize("seed,k", [(3, 2), (4, 5)])
def test_lemma_3_1_input_side_bruteforce(seed, k):
    rng = np.random.default_rng(seed)
    T, d, F = 3, 8, 8
    x = rng.integers(-8, 9, size=(T, d)) / 8.0
    # the stacked [W_gate; W_up] has orthogonal columns: Hadamard columns,
    # each scaled by its own power of two
    Hs = _hadamard(16)[:, :d] * (2.0 ** rng.integers(-3, 3, size=d))[None, :]
    Wg, Wu = Hs[:F], Hs[F:]
    Wd = rng.integers(-8, 9, size=(F, d)) / 16.0
    res = _F().forward(x, Wu, Wd, W_gate=Wg, dtype="bf16", C=128, input_k=k)
    for t in range(T):
        full = Hs @ x[t]
        best = min(itertools.combinations(range(d), k),
                   key=lambda S: (float(np.sum((full - Hs[:, list(S)] @ x[t, list(S)]) ** 2)), S))
        assert set(np.nonzero(res.x_keep[t])[0]) == set(best)


# ----------------------------------------------------------------------------
# reductions
# ----------------------------------------------------------------------------
def _small(seed=9, act="silu"):
    wl = synth.Workload("t", 64, 256, 4, mode="wina_topk", act=act, bias=None, k=0,
                        tile_capacity=128, seed=seed)
    inp = synth.make_inputs(wl)
    return (synth.to_f64(inp.x), synth.to_f64(inp.W_gate), synth.to_f64(inp.W_up),
            synth.to_f64(inp.W_down))


def test_full_h_reductions():
    x, Wg, Wu, Wd = _small()
    F = _F()
    full = F.forward(x, Wu, Wd, W_gate=Wg, mode="wina_full_h", act="silu", k=256, C=128)
    dense = F.forward(x, Wu, Wd, W_gate=Wg, mode="wina_topk", act="silu", k=256, C=128)
    assert full.keep.all()
    np.testing.assert_array_equal(full.y, dense.y)
    none = F.forward(x, Wu, Wd, W_gate=Wg, mode="wina_full_h", act="silu", k=0, C=128)
    assert not none.keep.any() and np.all(none.y == 0)
    # u = 1 for every neuron (x_0 = 1 feeds W_up's first column of ones, all
    # else zero): the full-h score is the gate-only score
    x1 = x.copy(); x1[:, 0] = 1.0
    Wu1 = np.zeros_like(Wu); Wu1[:, 0] = 1.0
    a = F.forward(x1, Wu1, Wd, W_gate=Wg, mode="wina_full_h", act="silu", k=40, C=128)
    b = F.forward(x1, Wu1, Wd, W_gate=Wg, mode="wina_topk", act="silu", k=40, C=128)
    assert np.array_equal(a.keep, b.keep)


def test_input_side_reductions():
    x, Wg, Wu, Wd = _small(act="relu")
    F = _F()
    plain = F.forward(x, Wu, Wd, W_gate=Wg, dtype="bf16", C=128)
    alld = F.forward(x, Wu, Wd, W_gate=Wg, dtype="bf16", C=128, input_k=x.shape[1])
    np.testing.assert_array_equal(alld.y, plain.y)
    assert alld.x_keep.all()
    b = np.full(Wg.shape[0], 0.5)
    none = F.forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", C=128, input_k=0)
    assert np.all(none.x_used == 0) and np.all(none.y == 0)
    assert none.keep.all()          # g = b = 0.5 > 0 everywhere, but u = 0
    # exactly input_k coordinates per token, or fewer non-zero ones kept as zeros
    some = F.forward(x, Wu, Wd, W_gate=Wg, dtype="bf16", C=128, input_k=20)
    assert np.all(some.x_keep.sum(axis=1) == 20)


def test_rotation_identity_and_signed_permutation():
    wl = synth.Workload("t", 64, 256, 6, exact_grid=True, tile_capacity=128, seed=4)
    inp = synth.make_inputs(wl)
    x, Wg, Wu, Wd = (synth.to_f64(t) for t in (inp.x, inp.W_gate, inp.W_up, inp.W_down))
    b = synth.to_f64(inp.bias)
    F = _F()
    plain = F.forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", C=128)
    same = F.forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", C=128, V=np.eye(64))
    np.testing.assert_array_equal(same.y, plain.y)
    # a signed permutation is orthogonal and exact in bf16: W V V^T x = W x
    # with every product and sum exact on the grid
    rng = np.random.default_rng(1)
    P = np.zeros((64, 64)); P[np.arange(64), rng.permutation(64)] = rng.choice([-1.0, 1.0], 64)
    rot = F.forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", C=128, V=P)
    assert np.array_equal(rot.keep, plain.keep)
    np.testing.assert_array_equal(rot.y, plain.y)
    np.testing.assert_array_equal(rot.x_used, x @ P)


def test_orthogonal_basis_gives_orthogonal_columns():
    x, Wg, Wu, Wd = _small()
    F = _F()
    V = F.orthogonal_basis(Wg, Wu)
    np.testing.assert_allclose(V.T @ V, np.eye(V.shape[0]), atol=1e-12)
    S = np.linalg.svd(np.concatenate([Wg, Wu]), compute_uv=False)
    Wr = np.concatenate([Wg, Wu]) @ V
    G = Wr.T @ Wr
    off = G - np.diag(np.diag(G))
    assert np.abs(off).max() < 1e-10 * np.abs(G).max()
    np.testing.assert_allclose(np.sqrt(np.diag(G)), S, rtol=1e-12)
    # after the rotation (fp32 operands keep the roundings small) the
    # forward's output is the unrotated one
    a = F.forward(x, Wu, Wd, W_gate=Wg, dtype="fp32", mode="wina_topk", act="silu", k=256, C=128)
    r = F.forward(x, Wu, Wd, W_gate=Wg, dtype="fp32", mode="wina_topk", act="silu", k=256, C=128, V=V)
    assert np.abs(r.y - a.y).max() < 1e-5 * np.abs(a.y).max()
    # the input column norms of the rotated stack are the singular values
    np.testing.assert_allclose(F.input_col_norms(Wr[:256], Wr[256:]), S, rtol=1e-6)


# ----------------------------------------------------------------------------
# planted mistakes
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mutation", ["full_h_gate_only", "input_norms_gate_only", "rotate_transposed",
                                      "input_keep_smallest", "full_h_rounded_v"])
def test_wina_pins_catch_planted_mistakes(monkeypatch, mutation):
    import oracle.ffn as F
    if mutation == "full_h_gate_only":
        monkeypatch.setattr(F, "wina_full_h_scores", lambda a, u, n: np.abs(a) * n[None, :])
    elif mutation == "input_norms_gate_only":
        monkeypatch.setattr(F, "input_col_norms",
                            lambda Wg, Wu: F.round_fp32(np.sqrt(np.sum(Wg * Wg, axis=0))))
    elif mutation == "rotate_transposed":
        monkeypatch.setattr(F, "rotate", lambda M, V, dt: F.round_operand(M @ V.T, dt))
    elif mutation == "input_keep_smallest":
        orig = F.input_scores
        monkeypatch.setattr(F, "input_scores", lambda x, c: -orig(x, c))
    elif mutation == "full_h_rounded_v":
        monkeypatch.setattr(F, "wina_full_h_scores",
                            lambda a, u, n: np.abs(F.round_bf16(a) * u) * n[None, :])
    failures = 0
    for test in (test_hand_worked_full_h, test_hand_worked_input_side,
                 test_full_h_scores_the_unrounded_activation,
                 lambda: test_lemma_3_1_full_h_bruteforce(0, 3),
                 lambda: test_lemma_3_1_input_side_bruteforce(3, 2),
                 test_full_h_reductions, test_input_side_reductions,
                 test_rotation_identity_and_signed_permutation):
        try:
            test()
        except AssertionError:
            failures += 1
    assert failures > 0, mutation
