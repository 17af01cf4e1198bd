"""GPU parity of the TILES path's single launch (up to 32 tokens, threshold
selection, dense or low-rank gate) against the fp64 oracle, through the C ABI:
full-size layers (the gate split across CTAs, every z and up range a partial
sum), small and ragged shapes, forced overflow (the overflow tokens' h from the
same tiles), the separate-kernel tile path beside it, repeated and concurrent
forwards (the seq-tagged flags) and the bounded waits."""
from __future__ import annotations

import pytest
import torch

import oracle
import synth
from activation_sparse_gated_relu_b200 import SFFN_OK, SFFN_PATH_TILES

from parity_util import check, make_ffn, rel_err, to_dev

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def small(**kw):
    base = dict(name="small", d_model=256, d_ff=512, tokens=32, tile_capacity=32)
    base.update(kw)
    return synth.Workload(**base)


def fused(st):
    return st["path"] == SFFN_PATH_TILES and st["launches"] == 1


@pytest.fixture(scope="module")
def dense32():
    return synth.make_inputs(W["decode_bf16"].with_(tokens=32))


@pytest.fixture(scope="module")
def lopa32():
    return synth.make_inputs(W["lopa_bf16"])


@pytest.mark.parametrize("T", [32, 17, 9])
def test_full_size_dense_gate(dense32, T):
    # d 4096, d_ff 14336: each 64-block gate is split between two CTAs
    st = check(dense32, T=T, path="tiles")
    assert fused(st)


@pytest.mark.parametrize("T", [32, 20, 1])
def test_full_size_low_rank_gate(lopa32, T):
    st = check(lopa32, T=T, path="tiles")
    assert fused(st)


def test_full_size_exact_grid_bit_exact():
    # sums of exact-grid products are exact in fp32 in any order, so the split
    # gate and z, added in K order, give the oracle's TwELL bit for bit
    for wl in (W["decode_bf16"].with_(tokens=32, exact_grid=True), W["lopa_bf16"].with_(exact_grid=True)):
        st = check(synth.make_inputs(wl), path="tiles")
        assert fused(st) and st["mismatch"] == 0


@pytest.mark.parametrize("T", [1, 5, 13, 32])
@pytest.mark.parametrize("rank", [0, 64, 192])
def test_small_shapes(T, rank):
    inp = synth.make_inputs(small(tokens=T, rank=rank))
    st = check(inp, path="tiles")
    assert fused(st)


def test_ragged_model_width():
    # d not a multiple of 64 or 128: the last K block and output tile are partial
    for d in (208, 264, 136):
        inp = synth.make_inputs(small(tokens=11, d_model=d, d_ff=384, threshold=0.25))
        assert fused(check(inp, path="tiles"))
    inp = synth.make_inputs(small(tokens=11, d_model=264, d_ff=384, rank=128))
    assert fused(check(inp, path="tiles"))


@pytest.mark.parametrize("C", [8, 16])
def test_forced_overflow_same_y(dense32, C):
    # a token whose record overflows gets the dense channel's h from the same
    # tiles: y matches the oracle and the records and flags are exact
    st = check(dense32, T=32, C=C, path="tiles")
    assert fused(st) and st["overflow"] > 0


def test_silu_threshold_no_bias():
    inp = synth.make_inputs(small(tokens=24, d_model=512, d_ff=1024, act="silu", bias=None, threshold=0.05))
    assert fused(check(inp, path="tiles"))


def test_matches_the_separate_kernels(lopa32, dense32):
    res = oracle.forward_inputs(lopa32, T=32)
    one = check(lopa32, T=32, res=res)
    sep = check(lopa32, T=32, res=res, separate=True)
    assert fused(one) and sep["launches"] > 1
    res = oracle.forward_inputs(dense32, T=20)
    assert check(dense32, T=20, res=res, separate=True)["launches"] > 1
    assert fused(check(dense32, T=20, res=res))


def test_repeated_mixed_T_one_handle(dense32):
    # each launch's flags carry its own sequence number: back-to-back launches
    # of different sizes see only their own partial sums and tiles
    ffn = make_ffn(dense32, max_tokens=32, path="tiles")
    res = {}
    try:
        for T in (32, 9, 32, 1, 17, 32, 32):
            if T not in res:
                res[T] = oracle.forward_inputs(dense32, T=T)
            st = check(dense32, T=T, ffn=ffn, res=res[T])
            assert fused(st)
    finally:
        ffn.close()


def test_zero_input_and_canaries(lopa32):
    ffn = make_ffn(lopa32, max_tokens=32)
    try:
        x = torch.zeros((32, ffn.d_model), dtype=torch.bfloat16, device="cuda")
        buf = torch.full((34, ffn.d_model), 7.0, dtype=torch.float32, device="cuda")
        out = buf[1:33]
        ffn.forward(x, out)
        torch.cuda.synchronize()
        assert ffn.read_status() == SFFN_OK
        assert torch.all(buf[0] == 7.0) and torch.all(buf[33] == 7.0)
        # zero x: z = 0, g = bias < 0, nothing kept, y = 0
        assert torch.all(out == 0.0), float(out.abs().max())
    finally:
        ffn.close()


@pytest.mark.parametrize("cooperative", [False, True])
def test_two_handles_concurrently_on_two_streams(lopa32, cooperative):
    a = make_ffn(lopa32, max_tokens=32, cooperative=cooperative)
    b = make_ffn(lopa32, max_tokens=32, cooperative=cooperative)
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    xa, xb = to_dev(lopa32.x[:32]), to_dev(lopa32.x[10:30])
    oa = torch.full((32, a.d_model), float("nan"), dtype=torch.float32, device="cuda")
    ob = torch.full((20, b.d_model), float("nan"), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    try:
        for _ in range(20):
            a.forward(xa, oa, stream=sa.cuda_stream)
            b.forward(xb, ob, stream=sb.cuda_stream)
        torch.cuda.synchronize()
        assert a.read_status(sa.cuda_stream) == SFFN_OK
        assert b.read_status(sb.cuda_stream) == SFFN_OK
        assert a.stats(sa.cuda_stream).launch_attrs & 1 == (1 if cooperative else 0)
        ra = oracle.forward_inputs(lopa32, T=32)
        assert rel_err(oa.double().cpu().numpy(), ra.y) <= 2e-3
        rb = oracle.forward_inputs(lopa32, T=30)
        assert rel_err(ob.double().cpu().numpy(), rb.y[10:30]) <= 2e-3
    finally:
        a.close()
        b.close()


def test_bounded_waits(lopa32):
    # a CTA counted in the job lists that never runs: the tiles and partial
    # sums it owns are never published, so the waits on them give up after
    # the limit, the launch reports a timeout, and the handle works afterwards
    from activation_sparse_gated_relu_b200 import SFFN_ERR_TIMEOUT
    ffn = make_ffn(lopa32, max_tokens=32)
    try:
        x = to_dev(lopa32.x[:32])
        out = torch.full((32, ffn.d_model), 7.0, dtype=torch.float32, device="cuda")
        ffn.debug_decode_waits(1, 20000)
        ffn.forward(x, out)
        torch.cuda.synchronize()
        assert ffn.read_status() == SFFN_ERR_TIMEOUT
        ffn.debug_decode_waits(0, 0)
        st = check(lopa32, T=32, ffn=ffn)
        assert fused(st)
    finally:
        ffn.close()
