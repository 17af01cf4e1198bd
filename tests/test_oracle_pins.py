"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test fixes the oracle to an independent source: hand-worked fixtures,
exact-rational brute force, closed forms, library routines it does not call,
or an equivalent computation with a different loop nest.  A mutation test at
the end plants mistakes in the oracle and checks that these pins notice.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# bf16 rounding
# ----------------------------------------------------------------------------
def test_round_bf16_hand_cases():
    cases = json.load(open(os.path.join(GOLDEN, "bf16_rounding.json")))["cases"]
    inp = np.array([c["input"] for c in cases])
    got = oracle.round_bf16(inp)
    for c, gv in zip(cases, got):
        want = math.inf if c["bf16"] == "inf" else c["bf16"]
        assert gv == want, c
        # the bit pattern, via torch's exact bf16 encoding of a bf16-exact value
        bits = torch.tensor([gv], dtype=torch.float32).to(torch.bfloat16).view(torch.int16)
        assert int(bits.item()) & 0xFFFF == int(c["bits"], 16), c


def test_round_bf16_matches_torch_rne_on_fp32_inputs():
    rng = np.random.default_rng(123)
    a = np.concatenate([
        rng.standard_normal(200000).astype(np.float32),
        (rng.standard_normal(20000) * 1e-39).astype(np.float32),     # subnormals
        (rng.standard_normal(20000) * 1e37).astype(np.float32),
        # exact ties: bf16 value + half spacing
        (np.arange(1, 20001, dtype=np.float32) * np.float32(2.0 ** -7) + 1).astype(np.float32)
        + np.float32(2.0 ** -8),
    ])
    want = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(a.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_round_fp32_matches_numpy_cast():
    rng = np.random.default_rng(5)
    a = rng.standard_normal(10000) * 3
    assert np.all(oracle.round_fp32(a) == a.astype(np.float32).astype(np.float64))


# ----------------------------------------------------------------------------
# hand-worked fixture
# ----------------------------------------------------------------------------
def _hand_case():
    d = json.load(open(os.path.join(GOLDEN, "hand_worked.json")))
    F, dm = 128, 2
    x = np.array(d["x"], dtype=np.float64)
    Wg = np.zeros((F, dm)); Wu = np.zeros((F, dm)); Wd = np.zeros((F, dm))
    b = np.full(F, -1.0)
    for j, r in d["rows"].items():
        j = int(j)
        Wg[j] = r["gate"]; Wu[j] = r["up"]; Wd[j] = r["down"]; b[j] = r["bias"]
    return d, x, Wg, Wu, Wd, b


def test_hand_worked_threshold():
    d, x, Wg, Wu, Wd, b = _hand_case()
    th = d["threshold"]
    for C in (3, 2):
        res = oracle.forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", C=C)
        np.testing.assert_array_equal(res.y, np.array(th["y"]))
        for t in range(2):
            assert list(np.nonzero(res.keep[t])[0]) == th["kept"][t]
            assert list(res.v[t, th["kept"][t]]) == th["values"][t]
        ref = th["C%d" % C]
        assert res.count.tolist() == ref["count"]
        assert res.idx.tolist() == ref["idx"]
        assert res.overflow.tolist() == ref["overflow"]
        if "val" in ref:
            assert res.val.tolist() == ref["val"]


def test_hand_worked_wina_relu():
    d, x, Wg, Wu, Wd, b = _hand_case()
    for kk, ref in d["wina_relu"].items():
        k = int(kk[1:])
        res = oracle.forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", mode="wina_topk",
                             act="relu", k=k, C=128)
        for t in range(2):
            assert list(np.nonzero(res.keep[t])[0]) == ref["kept"][t]
        np.testing.assert_array_equal(res.y, np.array(ref["y"]))


# ----------------------------------------------------------------------------
# exact-rational brute force
# ----------------------------------------------------------------------------
def _frac_bf16(q: Fraction) -> Fraction:
    """Round a rational to bf16 (8 significant bits, ties to even), exactly."""
    if q == 0:
        return Fraction(0)
    s = -1 if q < 0 else 1
    m = abs(q)
    e = m.numerator.bit_length() - m.denominator.bit_length()
    while Fraction(2) ** e > m:
        e -= 1
    while Fraction(2) ** (e + 1) <= m:
        e += 1
    e = max(e, -126)
    step = Fraction(2) ** (e - 7)
    n = m / step
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return s * fl * step


def _brute(x, Wg, b, Wu, Wd, tau):
    T, d = len(x), len(x[0])
    F = len(Wg)
    y = [[Fraction(0)] * d for _ in range(T)]
    keep = [[False] * F for _ in range(T)]
    for t in range(T):
        for j in range(F):
            g = sum((x[t][i] * Wg[j][i] for i in range(d)), Fraction(0)) + b[j]
            a = g if g > 0 else Fraction(0)
            if abs(a) > tau:
                keep[t][j] = True
                v = _frac_bf16(a)
                u = sum((x[t][i] * Wu[j][i] for i in range(d)), Fraction(0))
                for i in range(d):
                    y[t][i] += v * u * Wd[j][i]
    return y, keep


@pytest.mark.parametrize("seed,F,d,T,tau", [(0, 128, 4, 3, 0.0), (1, 256, 8, 2, 0.5),
                                            (2, 128, 6, 3, 0.25)])
def test_bruteforce_rational(seed, F, d, T, tau):
    rng = np.random.default_rng(seed)
    # dyadic values, so that fp64 holds every intermediate exactly
    x = rng.integers(-16, 17, size=(T, d)) / 8.0
    Wg = rng.integers(-8, 9, size=(F, d)) / 16.0
    Wu = rng.integers(-8, 9, size=(F, d)) / 16.0
    Wd = rng.integers(-8, 9, size=(F, d)) / 16.0
    b = rng.integers(-64, 17, size=F) / 64.0
    yb, kb = _brute([[Fraction(v) for v in r] for r in x],
                    [[Fraction(v) for v in r] for r in Wg], [Fraction(v) for v in b],
                    [[Fraction(v) for v in r] for r in Wu],
                    [[Fraction(v) for v in r] for r in Wd], Fraction(tau))
    res = oracle.forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", threshold=tau, C=128)
    assert res.keep.tolist() == kb
    assert 0 < res.keep.sum() < T * F
    np.testing.assert_array_equal(res.y, np.array([[float(v) for v in r] for r in yb]))


# ----------------------------------------------------------------------------
# invariants and reductions
# ----------------------------------------------------------------------------
def _eg_small(T=16, d=256, F=512, seed=3, **kw):
    wl = synth.Workload("t", d, F, T, exact_grid=True, seed=seed, tile_capacity=16, **kw)
    return wl, synth.make_inputs(wl)


def test_sparse_equals_masked_dense_exact_grid():
    wl, inp = _eg_small()
    res = oracle.forward_inputs(inp)
    x = synth.to_f64(inp.x)
    assert oracle.exact_grid_ok(x, synth.to_f64(inp.W_gate), 14)
    dense = oracle.dense_masked_ffn(x, synth.to_f64(inp.W_up), synth.to_f64(inp.W_down),
                                    res.keep, res.v)
    # both are exact: grid products and sums stay far below 2^53 units
    np.testing.assert_array_equal(res.y, dense)


def test_tau0_relu_equals_textbook_dense_ffn():
    """With tau = 0 every positive activation is kept, so y is the plain dense
    ReLU gated FFN.  Activations are made bf16-exact (small integers), so the
    stored-value rounding is the identity and the equality is exact."""
    rng = np.random.default_rng(7)
    T, d, F = 5, 16, 256
    x = rng.integers(-3, 4, size=(T, d)).astype(np.float64)
    Wg = rng.integers(-2, 3, size=(F, d)).astype(np.float64)
    Wu = rng.integers(-2, 3, size=(F, d)).astype(np.float64)
    Wd = rng.integers(-2, 3, size=(F, d)).astype(np.float64)
    res = oracle.forward(x, Wu, Wd, W_gate=Wg, bias=None, threshold=0.0, C=128)
    textbook = (np.maximum(x @ Wg.T, 0) * (x @ Wu.T)) @ Wd
    np.testing.assert_array_equal(res.y, textbook)


def test_twell_roundtrip_and_overflow():
    rng = np.random.default_rng(11)
    T, F = 7, 512
    keep = rng.random((T, F)) < 0.08
    keep[3, 130:190] = True                     # a heavy tile
    v = oracle.round_bf16(rng.standard_normal((T, F)))
    for C in (8, 16, 128):
        count, idx, val, ovf = oracle.twell_pack(keep, v, C)
        assert np.all(count == keep.reshape(T, F // 128, 128).sum(axis=2))
        assert np.array_equal(ovf, (count > C).any(axis=1))
        for t in range(T):
            for p in range(F // 128):
                n = min(int(count[t, p]), C)
                s = idx[t, p, :n]
                assert np.all(np.diff(s) > 0) and np.all(s // 128 == p)
                assert np.all(idx[t, p, n:] == -1) and np.all(val[t, p, n:] == 0)
        dense, mask = oracle.twell_unpack(count, idx, val, F)
        ok = ~ovf
        assert np.array_equal(mask[ok], keep[ok])
        assert np.array_equal(dense[ok], np.where(keep, v, 0.0)[ok])
    assert oracle.twell_pack(keep, v, 8)[3][3] and not oracle.twell_pack(keep, v, 128)[3][3]


def test_lowrank_identity_reduces_to_dense_gate():
    wl = synth.Workload("t", 64, 256, 6, seed=4)
    inp = synth.make_inputs(wl)
    x, Wg, b = synth.to_f64(inp.x), synth.to_f64(inp.W_gate), synth.to_f64(inp.bias)
    A = np.eye(64)
    g_lr, z = oracle.gate_lowrank(x, A, Wg.T.copy(), b, "bf16")
    assert np.array_equal(z, x)                   # x is bf16 already: z = x exactly
    np.testing.assert_array_equal(g_lr, oracle.gate_dense(x, Wg, b))
    r1 = oracle.forward(x, synth.to_f64(inp.W_up), synth.to_f64(inp.W_down), A=A,
                        B=Wg.T.copy(), bias=b, C=32)
    r2 = oracle.forward(x, synth.to_f64(inp.W_up), synth.to_f64(inp.W_down), W_gate=Wg,
                        bias=b, C=32)
    assert np.array_equal(r1.keep, r2.keep)
    np.testing.assert_array_equal(r1.y, r2.y)


def test_wina_reductions():
    wl = synth.Workload("t", 64, 256, 4, mode="wina_topk", act="silu", bias=None, k=0,
                        tile_capacity=128, seed=9)
    inp = synth.make_inputs(wl)
    x, Wg = synth.to_f64(inp.x), synth.to_f64(inp.W_gate)
    Wu, Wd = synth.to_f64(inp.W_up), synth.to_f64(inp.W_down)
    # k = d_ff keeps everything: the dense SiLU gated FFN with stored values
    full = oracle.forward(x, Wu, Wd, W_gate=Wg, mode="wina_topk", act="silu", k=256, C=128)
    a = x @ Wg.T
    a = a / (1 + np.exp(-a))
    dense = (oracle.round_bf16(a) * (x @ Wu.T)) @ Wd
    np.testing.assert_allclose(full.y, dense, rtol=0, atol=1e-12 * np.abs(dense).max())
    assert full.keep.all()
    # k = 0 keeps nothing
    none = oracle.forward(x, Wu, Wd, W_gate=Wg, mode="wina_topk", act="silu", k=0, C=128)
    assert not none.keep.any() and np.all(none.y == 0)
    # equal norms: the selection is the plain top-k on |a|
    Wd_eq = np.zeros_like(Wd); Wd_eq[:, 0] = 0.5
    eq = oracle.forward(x, Wu, Wd_eq, W_gate=Wg, mode="wina_topk", act="silu", k=40, C=128)
    for t in range(4):
        order = sorted(range(256), key=lambda j: (-abs(a[t, j]), j))[:40]
        assert set(np.nonzero(eq.keep[t])[0]) == set(order)
    assert np.all(eq.keep.sum(axis=1) == 40)


def _ulp_close(got: float, want: Fraction, n_ulp: int) -> bool:
    """|got - want| <= n_ulp fp64 ulps of want, compared in exact rationals."""
    if want == 0:
        return got == 0.0
    ulp = Fraction(math.ulp(float(want)))
    return abs(Fraction(got) - want) <= n_ulp * ulp


def test_silu_hand_worked_values():
    # SiLU(g) = g/(1 + e^-g) at points worked by hand from e's decimal
    # expansion (tests/golden/silu.json), to 2 ulp of fp64
    cases = json.load(open(os.path.join(GOLDEN, "silu.json")))["cases"]
    g = np.array([c["g"] for c in cases])
    import oracle.ffn as F  # looked up at call time, as the oracle's forward does
    got = F.activate(g, "silu")
    for c, gv in zip(cases, got):
        assert _ulp_close(float(gv), Fraction(c["silu"]), 2), (c, gv)


def test_silu_odd_part_identity():
    # SiLU(g) - SiLU(-g) = g·(sigma(g) + sigma(-g)) - 0 = g for every g,
    # since sigma(g) + sigma(-g) = 1
    import oracle.ffn as F  # looked up at call time, as the oracle's forward does
    g = np.linspace(-20.0, 20.0, 4001)
    d = F.activate(g, "silu") - F.activate(-g, "silu")
    assert np.all(np.abs(d - g) <= 4 * np.finfo(np.float64).eps * np.maximum(np.abs(g), 1))


def test_threshold_tests_the_unrounded_activation():
    # reading 2: keep iff |sigma(g)| > tau on the unrounded activation, strict.
    # a = 1 + 2^-10 with tau = 1: kept, although its stored bf16 value is
    # 1.0 = tau (2^-10 is below half a bf16 ulp at 1); a = 1 exactly is not
    F, dm = 128, 2
    x = np.array([[1.0, 2.0 ** -10], [1.0, 0.0]])
    Wg = np.zeros((F, dm)); Wu = np.zeros((F, dm)); Wd = np.zeros((F, dm))
    b = np.full(F, -1.0)
    Wg[5] = [1.0, 1.0]; b[5] = 0.0; Wu[5] = [2.0, 0.0]; Wd[5] = [1.0, 3.0]
    res = oracle.forward(x, Wu, Wd, W_gate=Wg, bias=b, dtype="bf16", threshold=1.0, C=8)
    assert res.keep[0, 5] and not res.keep[1, 5]
    assert res.keep.sum() == 1 and res.v[0, 5] == 1.0
    # h = v·u = 1·2, y = h·W_down[5] = [2, 6]; token 1 keeps nothing
    np.testing.assert_array_equal(res.y, [[2.0, 6.0], [0.0, 0.0]])
    assert res.count.tolist() == [[1], [0]]


def test_lowrank_z_is_rounded_to_the_operand_dtype():
    # reading 4: z = round(x·A) before z·B.  Here x·A = 1 + 2^-8, halfway
    # between the bf16 neighbours 1 and 1 + 2^-7; round-to-nearest-even gives 1
    # in bf16, while fp32 holds 1 + 2^-8 exactly
    x = np.array([[1.0, 2.0 ** -8]])
    A = np.array([[1.0], [1.0]])
    B = np.array([[1.0, -3.0]])
    import oracle.ffn as F  # looked up at call time, as the oracle's forward does
    g, z = F.gate_lowrank(x, A, B, None, "bf16")
    assert z[0, 0] == 1.0
    assert np.array_equal(g, [[1.0, -3.0]])
    g32, z32 = F.gate_lowrank(x, A, B, None, "fp32")
    assert z32[0, 0] == 1.0 + 2.0 ** -8
    assert np.array_equal(g32, [[1.0 + 2.0 ** -8, -3.0 - 3.0 * 2.0 ** -8]])


def test_wina_norms_closed_form():
    Wd = np.zeros((128, 4)); Wd[:, 0] = 3.0; Wd[:, 1] = 4.0
    assert np.all(oracle.wina_norms(Wd) == 5.0)


def test_wina_norms_are_fp32_rounded():
    # reading 5: n_j is the fp64 norm rounded to fp32; ||(1, 1)|| = sqrt(2)
    # is not an fp32 number, and its fp32 rounding is 1.41421353816986083984375
    import oracle.ffn as F  # looked up at call time, as the oracle's forward does
    Wd = np.zeros((128, 2)); Wd[:, :] = 1.0
    n = F.wina_norms(Wd)
    assert np.all(n == 1.41421353816986083984375)
    assert n[0] != math.sqrt(2.0)


# ----------------------------------------------------------------------------
# closed-form sparsity of the synthetic recipes
# ----------------------------------------------------------------------------
def test_bias_gives_ninety_percent_zeros():
    wl = synth.Workload("t", 1024, 4096, 16, seed=0)
    inp = synth.make_inputs(wl)
    g = oracle.gate_dense(synth.to_f64(inp.x), synth.to_f64(inp.W_gate), synth.to_f64(inp.bias))
    zeros = float(np.mean(oracle.activate(g, "relu") == 0))
    p = 0.5 * (1 + math.erf(1.2816 / math.sqrt(2)))      # Phi(1.2816) = 0.9000
    assert abs(p - 0.9) < 1e-4
    sigma = math.sqrt(p * (1 - p) / g.size)
    assert abs(zeros - p) < 5 * sigma + 0.01   # +0.01: token norms fluctuate about 1


def test_lognormal_nnz_recipe():
    wl = synth.WORKLOADS["prefill_bf16"].with_(d_model=512, d_ff=2048)
    T = 96
    inp = synth.make_inputs(wl, T=T)
    g = oracle.gate_dense(synth.to_f64(inp.x), synth.to_f64(inp.W_gate), synth.to_f64(inp.bias))
    nnz = (oracle.activate(g, "relu") > 0).sum(axis=1)
    target, _ = synth.token_scales(wl, T)
    p = np.minimum(target / wl.d_ff, 0.45)
    exp = p * wl.d_ff
    sd = np.sqrt(exp * (1 - p))
    # per-token counts follow Binomial(d_ff, p_t) up to the spread of ||z_t||
    assert np.all(np.abs(nnz - exp) < 6 * sd + 0.15 * exp + 3)
    # lognormal mean exp(mu + sigma^2/2) = 60·e^0.5 = 98.9 (before the cap)
    big = synth.token_scales(synth.WORKLOADS["prefill_bf16"], 20000)[0]
    assert abs(big.mean() - 60 * math.exp(0.5)) < 4.0


# ----------------------------------------------------------------------------
# mutations: plant mistakes in the oracle and check that the pins catch them
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mutation", ["no_bias", "no_value_round", "transposed_down",
                                      "nonstrict", "silu_sign", "topk_tie_high", "no_z_round",
                                      "keep_on_rounded", "norms_unrounded", "silu_is_sigmoid"])
def test_pins_catch_planted_mistakes(monkeypatch, mutation):
    import oracle.ffn as F
    if mutation == "no_bias":
        monkeypatch.setattr(F, "gate_dense", lambda x, W, b: x @ W.T)
    elif mutation == "no_value_round":
        monkeypatch.setattr(F, "round_operand", lambda a, dt: a)
    elif mutation == "transposed_down":
        orig = F.sparse_up_down

        def bad(x, Wu, Wd, keep, v):
            return orig(x, Wu, Wd[:, ::-1].copy(), keep, v)
        monkeypatch.setattr(F, "sparse_up_down", bad)
    elif mutation == "nonstrict":
        monkeypatch.setattr(F, "keep_threshold", lambda a, tau: np.abs(a) >= tau)
    elif mutation == "silu_sign":
        orig_act = F.activate
        monkeypatch.setattr(F, "activate",
                            lambda g, act: g / (1 + np.exp(g)) if act == "silu" else orig_act(g, act))
    elif mutation == "topk_tie_high":
        def bad_topk(s, k):
            T, Fn = s.shape
            keep = np.zeros((T, Fn), dtype=bool)
            for t in range(T):
                order = np.lexsort((-np.arange(Fn), -s[t]))
                keep[t, order[:k]] = True
            return keep
        monkeypatch.setattr(F, "keep_topk", bad_topk)
    elif mutation == "norms_unrounded":
        monkeypatch.setattr(F, "wina_norms", lambda W: np.sqrt(np.sum(W * W, axis=1)))
    elif mutation == "keep_on_rounded":
        monkeypatch.setattr(F, "keep_threshold", lambda a, tau: np.abs(F.round_bf16(a)) > tau)
    elif mutation == "silu_is_sigmoid":
        orig_act = F.activate
        monkeypatch.setattr(F, "activate",
                            lambda g, act: 1 / (1 + np.exp(-g)) if act == "silu" else orig_act(g, act))
    elif mutation == "no_z_round":
        def no_round(x, A, B, bias, dtype):
            z = x @ A
            g = z @ B
            return (g + bias[None, :] if bias is not None else g), z
        monkeypatch.setattr(F, "gate_lowrank", no_round)
    failures = 0
    for test in (test_hand_worked_threshold, test_hand_worked_wina_relu,
                 lambda: test_bruteforce_rational(0, 128, 4, 3, 0.0),
                 test_wina_reductions, test_lowrank_z_is_rounded_to_the_operand_dtype,
                 test_threshold_tests_the_unrounded_activation, test_wina_norms_are_fp32_rounded,
                 test_silu_hand_worked_values, test_silu_odd_part_identity):
        try:
            test()
        except AssertionError:
            failures += 1
    assert failures > 0, mutation


def test_silu_goldens_alone_catch_sigmoid_for_silu(monkeypatch):
    # the hand-worked values and the odd-part identity each reject a SiLU
    # replaced by the plain logistic sigmoid, without any other pin's help
    import oracle.ffn as F
    orig_act = F.activate
    monkeypatch.setattr(F, "activate",
                        lambda g, act: 1 / (1 + np.exp(-g)) if act == "silu" else orig_act(g, act))
    for test in (test_silu_hand_worked_values, test_silu_odd_part_identity):
        with pytest.raises(AssertionError):
            test()
