"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Rules: TwELL counts/indices/overflow flags bit-exact outside a decision band
of 2^-14·sum|x_i w_i| around the selection boundary (no band on exact-grid
inputs, where values must also match bit for bit); y within
max|y - y_ref| / max|y_ref| <= 2e-3 (bf16 operands) or 1e-5 (fp32).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from activation_sparse_gated_relu_b200 import SFFN_OK, SFFN_PATH_ROWS, SFFN_PATH_TILES

from parity_util import check, make_ffn, rel_err, run_gpu, to_dev

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def small(**kw):
    base = dict(name="small", d_model=256, d_ff=512, tokens=32, tile_capacity=32)
    base.update(kw)
    return synth.Workload(**base)


# ------------------------------------------------------------ small shapes
@pytest.mark.parametrize("T", [1, 5, 8, 13, 32])
@pytest.mark.parametrize("path", ["rows", "tiles"])
def test_small_bf16_paths(T, path):
    inp = synth.make_inputs(small(tokens=T))
    st = check(inp, path=path)
    assert st["path"] == (SFFN_PATH_ROWS if path == "rows" else SFFN_PATH_TILES)


@pytest.mark.parametrize("T", [8, 32])
def test_small_bf16_exact_grid_bit_exact(T):
    inp = synth.make_inputs(small(tokens=T, exact_grid=True))
    st = check(inp)
    assert st["mismatch"] == 0


def test_gate_tensor_core_sum_is_exact_on_grid():
    """Dense fp32 gate from tcgen05 vs the oracle: identical on exact-grid inputs."""
    inp = synth.make_inputs(small(tokens=16, exact_grid=True))
    ffn = make_ffn(inp, max_tokens=16, debug_gate=True)
    run_gpu(ffn, inp.x)
    g = ffn.gate_debug(16).double().cpu().numpy()
    ref = oracle.gate_dense(synth.to_f64(inp.x), synth.to_f64(inp.W_gate), synth.to_f64(inp.bias))
    ffn.close()
    assert np.array_equal(g, ref)


def test_gate_tensor_core_within_band_gaussian():
    inp = synth.make_inputs(small(tokens=16, d_model=1024, d_ff=1024))
    ffn = make_ffn(inp, max_tokens=16, debug_gate=True)
    run_gpu(ffn, inp.x)
    g = ffn.gate_debug(16).double().cpu().numpy()
    x, Wg = synth.to_f64(inp.x), synth.to_f64(inp.W_gate)
    ref = oracle.gate_dense(x, Wg, synth.to_f64(inp.bias))
    ffn.close()
    assert np.all(np.abs(g - ref) <= oracle.gate_band(x, Wg))


@pytest.mark.parametrize("C", [8, 16, 128])
def test_small_overflow_capacity_does_not_change_y(C):
    inp = synth.make_inputs(small(tokens=24, d_model=512, d_ff=1024))
    st = check(inp, C=C, path="rows")
    if C == 8:
        assert st["overflow"] > 0
    if C == 128:
        assert st["overflow"] == 0


def test_small_overflow_tiles_path():
    inp = synth.make_inputs(small(tokens=40, d_model=512, d_ff=1024))
    st = check(inp, C=8, path="tiles")
    assert st["overflow"] > 0


def test_single_heavy_token_overflows():
    wl = small(tokens=8, d_model=512, d_ff=1024)
    inp = synth.make_inputs(wl)
    x = inp.x.clone()
    x[3] = (x[3].float() * 4).to(x.dtype)
    inp.x = x
    st = check(inp, path="rows")
    assert st["overflow"] == 1


def test_ragged_dims_and_threshold():
    # d not a multiple of 64 (ragged K block of the gate), a positive threshold, one tile
    inp = synth.make_inputs(small(tokens=11, d_model=208, d_ff=128, threshold=0.25))
    check(inp, path="tiles")
    inp = synth.make_inputs(small(tokens=11, d_model=768, d_ff=128, threshold=0.25))
    check(inp, path="rows")


def test_row_path_shape_rule():
    # the fused row kernel needs d % 256 == 0; AUTO then takes the tile path
    inp = synth.make_inputs(small(tokens=6, d_model=200, d_ff=256))
    st = check(inp)
    assert st["path"] == SFFN_PATH_TILES
    from activation_sparse_gated_relu_b200 import SffnError
    with pytest.raises(SffnError):
        check(inp, path="rows")


def test_silu_threshold_and_no_bias():
    inp = synth.make_inputs(small(tokens=9, act="silu", threshold=0.3, bias=None))
    check(inp, path="rows")


def test_zero_input_gives_zero():
    inp = synth.make_inputs(small(tokens=8))
    inp.x = torch.zeros_like(inp.x)
    st = check(inp)
    assert st["err"] == 0.0


def test_T0_is_a_noop_and_bad_T_rejected():
    inp = synth.make_inputs(small(tokens=8))
    ffn = make_ffn(inp, max_tokens=8)
    x = to_dev(inp.x)
    out = torch.full((8, 256), 7.0, device="cuda")
    ffn.forward(x[:0], out[:0])
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
    from activation_sparse_gated_relu_b200 import SffnError
    with pytest.raises(SffnError):
        from activation_sparse_gated_relu_b200 import binding
        binding.sffn_forward(ffn.h, x.data_ptr(), 9, out.data_ptr(), 0)
    ffn.close()


def test_repeated_forwards_and_host_entry_point():
    inp = synth.make_inputs(small(tokens=16))
    ffn = make_ffn(inp, max_tokens=16)
    x = to_dev(inp.x)
    y1 = ffn(x).clone()
    y2 = ffn(x[:8]).clone()
    y3 = ffn(x).clone()
    torch.cuda.synchronize()
    # the output split over CTAs is summed with fp32 atomics, so the order of
    # the partial sums (and the last bits) may change between launches
    assert rel_err(y2.double().cpu().numpy(), y1[:8].double().cpu().numpy()) < 1e-5
    assert rel_err(y3.double().cpu().numpy(), y1.double().cpu().numpy()) < 1e-5
    yh = ffn.forward_host(inp.x.contiguous().pin_memory())
    assert rel_err(yh.double().numpy(), y1.double().cpu().numpy()) < 1e-5
    assert ffn.read_status() == SFFN_OK
    ffn.close()


def test_output_canaries_intact():
    inp = synth.make_inputs(small(tokens=12))
    ffn = make_ffn(inp, max_tokens=12)
    pad = 16384
    buf = torch.full((pad + 12 * 256 + pad,), 12345.0, device="cuda")
    out = buf[pad:pad + 12 * 256].view(12, 256)
    ffn.forward(to_dev(inp.x), out)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == 12345.0) and torch.all(buf[pad + 12 * 256:] == 12345.0)
    ffn.close()


# ------------------------------------------------------------------ fp32
def test_tiny_fp32_config():
    inp = synth.make_inputs(W["tiny_fp32"])
    st = check(inp)
    assert st["err"] <= 1e-5


def test_tiny_fp32_exact_grid_and_overflow():
    inp = synth.make_inputs(W["tiny_fp32"].with_(exact_grid=True))
    st = check(inp)
    assert st["mismatch"] == 0
    st = check(inp, C=8)
    assert st["overflow"] > 0


def test_fp32_wina():
    inp = synth.make_inputs(small(dtype="fp32", mode="wina_topk", act="silu", bias=None, k=180,
                                  tile_capacity=128, tokens=10))
    check(inp)


# ------------------------------------------------------- full-size configs
@pytest.fixture(scope="module")
def decode_inputs():
    return synth.make_inputs(W["decode_bf16"])


@pytest.mark.parametrize("T", [1, 4, 8])
def test_decode_config(decode_inputs, T):
    st = check(decode_inputs, T=T)
    assert st["path"] == SFFN_PATH_ROWS


def test_decode_exact_grid_bit_exact():
    inp = synth.make_inputs(W["decode_bf16"].with_(exact_grid=True))
    x = synth.to_f64(inp.x)
    assert oracle.exact_grid_ok(x, synth.to_f64(inp.W_gate), 14)
    st = check(inp)
    assert st["mismatch"] == 0


def test_decode_forced_overflow_same_y(decode_inputs):
    a = check(decode_inputs, T=8, C=8)
    assert a["overflow"] == 8
    b = check(decode_inputs, T=8, C=128)
    assert b["overflow"] == 0


def test_decode_single_launch_and_separate_kernels(decode_inputs):
    # T <= 8 runs as one persistent launch; the flag keeps the separate
    # gate, up x down and dense-channel launches, which must agree
    one = check(decode_inputs, T=8)
    assert one["launches"] == 1 and one["path"] == SFFN_PATH_ROWS
    sep = check(decode_inputs, T=8, separate=True)
    assert sep["launches"] == 4 and sep["path"] == SFFN_PATH_ROWS
    check(decode_inputs, T=3, C=8, separate=True)


@pytest.mark.parametrize("C", [8, 16])
def test_decode_single_launch_dense_channel(decode_inputs, C):
    # small capacities make tokens overflow: in the single launch their kept
    # rows stream with everyone else's (the dense channel's sum without its
    # zero terms); their TwELL records cap at C and their flags are set
    st = check(decode_inputs, T=8, C=C)
    assert st["overflow"] > 0 and st["launches"] == 1


@pytest.mark.parametrize("d_ff,T", [(128, 8), (512, 3), (1024, 1)])
def test_decode_single_launch_few_gate_groups(d_ff, T):
    # fewer 8-neuron gate groups than SMs: most CTAs gate nothing, build no
    # list and only steal; one tile at d_ff = 128
    inp = synth.make_inputs(small(tokens=T, d_model=512, d_ff=d_ff))
    st = check(inp, path="rows")
    assert st["launches"] == 1


def test_decode_single_launch_silu_no_bias():
    inp = synth.make_inputs(small(tokens=7, d_model=1024, d_ff=2048, act="silu", threshold=0.3, bias=None))
    st = check(inp, path="rows")
    assert st["launches"] == 1


def test_decode_single_launch_bounded_waits(decode_inputs):
    # every wait on another CTA is bounded: with a CTA in the grid that never
    # runs (a list never published, a slice of out never zeroed) the launch
    # gives up after the limit and reports a timeout, and the handle works
    # again afterwards
    from activation_sparse_gated_relu_b200 import SFFN_ERR_TIMEOUT
    ffn = make_ffn(decode_inputs, max_tokens=8)
    try:
        x = to_dev(decode_inputs.x[:8])
        out = torch.full((8, ffn.d_model), 7.0, dtype=torch.float32, device="cuda")
        ffn.debug_decode_waits(1, 20000)
        ffn.forward(x, out)
        torch.cuda.synchronize()
        assert ffn.read_status() == SFFN_ERR_TIMEOUT
        ffn.debug_decode_waits(0, 0)
        st = check(decode_inputs, T=8, ffn=ffn)
        assert st["launches"] == 1
    finally:
        ffn.close()


def test_decode_handle_holds_no_dense_channel_copies(decode_inputs):
    # a handle for at most 8 tokens takes the single launch on every forward:
    # it holds neither the transposed W_down (117 MB at these sizes) nor the
    # h buffers, and its device memory is its one workspace allocation
    from activation_sparse_gated_relu_b200 import SparseFFN
    inp = decode_inputs
    dev = {k: to_dev(getattr(inp, k)) for k in ("W_gate", "W_up", "W_down", "bias")}

    def make(max_tokens):
        return SparseFFN(dev["W_up"], dev["W_down"], W_gate=dev["W_gate"], bias=dev["bias"],
                         tile_capacity=32, max_tokens=max_tokens)

    make(8).close()          # loads the kernels once, outside the measurement
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    ffn = make(8)
    try:
        torch.cuda.synchronize()
        grew = free0 - torch.cuda.mem_get_info()[0]
        ws = ffn.workspace_bytes()
        assert ws < (4 << 20), ws
        assert grew <= ws + (5 << 20), (grew, ws)
        check(inp, T=8, ffn=ffn)
    finally:
        ffn.close()
    # room for 9 tokens: other paths can run, so the handle keeps W_down^T
    big = make(9)
    try:
        assert big.workspace_bytes() > inp.wl.d_model * inp.wl.d_ff * 2
        check(inp, T=8, ffn=big)
    finally:
        big.close()


@pytest.mark.parametrize("cooperative", [False, True])
def test_decode_two_handles_concurrently_on_two_streams(decode_inputs, cooperative):
    # two handles' single launches issued on two streams at once, with and
    # without the cooperative attribute: both grids run whole (one after the
    # other: each fills every SM) and both match the oracle
    ffn_a = make_ffn(decode_inputs, max_tokens=8, cooperative=cooperative)
    ffn_b = make_ffn(decode_inputs, max_tokens=8, cooperative=cooperative)
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    xa, xb = to_dev(decode_inputs.x[:8]), to_dev(decode_inputs.x[5:8])
    oa = torch.full((8, ffn_a.d_model), float("nan"), dtype=torch.float32, device="cuda")
    ob = torch.full((3, ffn_b.d_model), float("nan"), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    try:
        for _ in range(25):
            ffn_a.forward(xa, oa, stream=sa.cuda_stream)
            ffn_b.forward(xb, ob, stream=sb.cuda_stream)
        torch.cuda.synchronize()
        assert ffn_a.read_status(sa.cuda_stream) == SFFN_OK
        assert ffn_b.read_status(sb.cuda_stream) == SFFN_OK
        assert ffn_a.stats(sa.cuda_stream).launch_attrs & 1 == (1 if cooperative else 0)
        ra = oracle.forward_inputs(decode_inputs, T=8)
        assert rel_err(oa.double().cpu().numpy(), ra.y) <= 2e-3
        assert rel_err(ob.double().cpu().numpy(), ra.y[5:8]) <= 2e-3
    finally:
        ffn_a.close()
        ffn_b.close()


def test_decode_single_launch_repeated_mixed_T(decode_inputs):
    # the scheduler words carry each forward's epoch: back-to-back forwards of
    # different sizes through one handle see only their own lists and zeros
    ffn = make_ffn(decode_inputs, max_tokens=8)
    res = {}
    try:
        for T in (8, 3, 8, 1, 5, 8, 8):
            if T not in res:
                res[T] = oracle.forward_inputs(decode_inputs, T=T)
            st = check(decode_inputs, T=T, ffn=ffn, res=res[T])
            assert st["launches"] == 1
    finally:
        ffn.close()


def test_decode_single_launch_across_epoch_windows(decode_inputs):
    # the scheduler words carry the low 16 bits of the epoch; forwards that
    # cross a window of 65536 epochs, and the 32-bit wrap (which skips 0),
    # still see only their own lists
    ffn = make_ffn(decode_inputs, max_tokens=8)
    res = {T: oracle.forward_inputs(decode_inputs, T=T) for T in (8, 3)}
    try:
        for start, epochs in ((0xFFFD, (0xFFFE, 0xFFFF, 0x10000, 0x10001)),
                              (0x2FFFE, (0x2FFFF, 0x30000, 0x30001, 0x30002)),
                              (0xFFFFFFFD, (0xFFFFFFFE, 0xFFFFFFFF, 1, 2))):
            ffn.debug_set_epoch(start)
            for T, ep in zip((8, 3, 8, 8), epochs):
                st = check(decode_inputs, T=T, ffn=ffn, res=res[T])
                assert st["launches"] == 1
                assert ffn.stats().epoch == ep
    finally:
        ffn.close()


def test_lopa_config():
    inp = synth.make_inputs(W["lopa_bf16"])
    st = check(inp)
    assert st["path"] == SFFN_PATH_TILES
    check(inp, T=8, path="rows")


def test_lopa_exact_grid():
    inp = synth.make_inputs(W["lopa_bf16"].with_(exact_grid=True, tokens=16))
    st = check(inp)
    assert st["mismatch"] == 0


def test_wina_config():
    inp = synth.make_inputs(W["wina_bf16"])
    ffn = make_ffn(inp, max_tokens=32)
    st = check(inp, ffn=ffn)
    n = ffn.norms().double().cpu().numpy()
    assert np.array_equal(n, oracle.wina_norms(synth.to_f64(inp.W_down)))
    tw = ffn.twell(32)
    assert np.all(tw["count"].sum(1).cpu().numpy() == W["wina_bf16"].k)
    ffn.close()


def test_prefill_sampled_full_size():
    """Full 4096-token prefill launch; the oracle recomputes sampled tokens."""
    wl = W["prefill_bf16"]
    inp = synth.make_inputs(wl)
    ffn = make_ffn(inp, max_tokens=wl.tokens)
    g = run_gpu(ffn, inp.x)
    ffn.close()
    assert g.path == SFFN_PATH_ROWS
    rng = np.random.default_rng(0)
    ovf_tok = np.nonzero(g.overflow)[0]
    sample = np.unique(np.concatenate([rng.choice(wl.tokens, 48, replace=False), ovf_tok[:16]]))
    x = synth.to_f64(inp.x)[sample]
    res = oracle.forward(x, synth.to_f64(inp.W_up), synth.to_f64(inp.W_down), W_gate=synth.to_f64(inp.W_gate),
                         bias=synth.to_f64(inp.bias), dtype="bf16", C=wl.tile_capacity)
    err = rel_err(g.y[sample], res.y)
    assert err <= 2e-3, err
    assert 0.04 < g.overflow.mean() < 0.3
    # TwELL of the sampled tokens
    from parity_util import GpuRun, ambiguous, compare_twell
    sub = GpuRun(g.y[sample], g.count[sample], g.idx[sample], g.val[sample], g.overflow[sample],
                 int(g.overflow[sample].sum()), g.path, g.launches)
    compare_twell(sub, res, wl.tile_capacity, ambiguous(res, "relu_threshold", 0.0, 0, False), False, "bf16")


@pytest.mark.parametrize("exact", [False, True])
def test_persistent_gate_many_tiles(exact):
    # more 128-neuron x token tiles than SMs: the persistent gate (two TMEM
    # accumulators, each tile's emission beside the next tile's MMAs); 1200
    # tokens leave a ragged last token tile.  The separate flag keeps the
    # one-CTA-per-tile gate, which must agree.
    inp = synth.make_inputs(small(tokens=1200, d_model=256, d_ff=4096, exact_grid=exact))
    res = oracle.forward_inputs(inp)
    a = check(inp, res=res)
    b = check(inp, res=res, separate=True)
    if exact:
        assert a["mismatch"] == 0 and b["mismatch"] == 0


def test_prefill_reduced_full_check():
    inp = synth.make_inputs(W["prefill_bf16"], T=384)
    st = check(inp)
    assert st["overflow"] > 0


@pytest.mark.parametrize("T", [1, 5, 8])
def test_lopa_row_gate_exact_grid(T):
    # up to 8 tokens with a rank that is a multiple of 128 the low-rank
    # gate's z streams the rank rows of A^T; on grid inputs every value is exact
    inp = synth.make_inputs(W["lopa_bf16"].with_(exact_grid=True, tokens=T, d_model=1024, d_ff=2048, rank=256))
    st = check(inp, path="rows")
    assert st["mismatch"] == 0 and st["path"] == SFFN_PATH_ROWS


@pytest.mark.parametrize("T", [1, 8])
def test_lopa_row_gate_full_size(T):
    inp = synth.make_inputs(W["lopa_bf16"].with_(tokens=T))
    st = check(inp, path="rows")
    assert st["path"] == SFFN_PATH_ROWS
