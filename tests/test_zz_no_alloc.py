"""The allocation-free low-rank gate entry point (sffn_lowrank_twell_noalloc).

It serves callers that cannot allocate device memory where they run (code in
a runtime that owns all device memory, or on a latency-critical path where
cudaMalloc may synchronise or fail): its scratch lives in fixed arrays inside
the library.  These tests call it through the C ABI twice in a row and check
its TwELL records against the fp64 oracle's: bit for bit on exact-grid inputs
(up to the documented maximum sizes, and with a rank that leaves the last
128-row tile of z partial), and under the usual decision band on Gaussian
inputs.  They also check that a bounded wait that runs out (a test hook makes
the kernels wait on a barrier that nothing signals) is reported by
sffn_lowrank_twell_noalloc_status, and that the next call is correct again.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from activation_sparse_gated_relu_b200 import SFFN_ERR_TIMEOUT, SFFN_ERR_UNSUPPORTED, SFFN_OK, binding

from parity_util import GpuRun, ambiguous, compare_twell

pytestmark = pytest.mark.gpu


def _lib():
    lib = binding.load_library()
    f = lib.sffn_lowrank_twell_noalloc
    vp = ctypes.c_void_p
    f.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, vp, ctypes.c_int, vp, ctypes.c_int,
                  ctypes.c_float, ctypes.c_int, vp, vp, vp, vp, vp]
    f.restype = ctypes.c_int
    lib.sffn_lowrank_twell_noalloc_status.argtypes = [vp]
    lib.sffn_lowrank_twell_noalloc_status.restype = ctypes.c_int
    lib.sffn_debug_noalloc_waits.argtypes = [ctypes.c_uint]
    lib.sffn_debug_noalloc_waits.restype = ctypes.c_int
    return lib


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _call(lib, dev_in, T, C, check_status=True):
    x, At, Bt, bias, wl = dev_in
    d, r, F = wl.d_model, wl.rank, wl.d_ff
    P = F // 128
    # canaries: every output element must be overwritten
    count = torch.full((T, P), -7, dtype=torch.int16, device="cuda")
    idx = torch.full((T, P, C), -7, dtype=torch.int16, device="cuda")
    val = torch.full((T, P, C), 7.0, dtype=torch.bfloat16, device="cuda")
    ovf = torch.full((T,), 0xDEAD, dtype=torch.int32, device="cuda")
    st = lib.sffn_lowrank_twell_noalloc(
        x.data_ptr(), T, d, At.data_ptr(), r, Bt.data_ptr(), F,
        bias.data_ptr() if bias is not None else None, 0 if wl.act == "relu" else 1,
        float(wl.threshold), C, count.data_ptr(), idx.data_ptr(), val.data_ptr(), ovf.data_ptr(), _stream())
    assert st == SFFN_OK, binding.status_string(st)
    if check_status:
        assert lib.sffn_lowrank_twell_noalloc_status(_stream()) == SFFN_OK
    torch.cuda.synchronize()
    ov = ovf.cpu().numpy()
    assert np.all((ov == 0) | (ov == 1)), "overflow flags not written as 0/1"
    return GpuRun(None, count.cpu().numpy(), idx.cpu().numpy(), val.float().cpu().numpy().astype(np.float64),
                  ov == 1, int((ov == 1).sum()), 0, 2)


def _device_inputs(inp, T):
    dev = lambda t: t.to("cuda").contiguous()  # noqa: E731
    bias = dev(inp.bias) if inp.bias is not None else None
    return dev(inp.x[:T]), dev(inp.A.t()), dev(inp.B.t()), bias, inp.wl


def _oracle_gate(inp, T, C):
    """The oracle's low-rank gate, activation, selection and TwELL pack (no up
    or down: this entry point stops at the TwELL records)."""
    wl = inp.wl
    x = synth.to_f64(inp.x[:T])
    B = synth.to_f64(inp.B)
    g, z = oracle.gate_lowrank(x, synth.to_f64(inp.A), B, synth.to_f64(inp.bias), wl.dtype)
    a = oracle.activate(g, wl.act)
    v = oracle.round_operand(a, wl.dtype)
    keep = oracle.keep_threshold(a, wl.threshold)
    count, idx, val, overflow = oracle.twell_pack(keep, v, C)
    band = oracle.lowrank_band(z, B)
    return oracle.OracleResult(np.zeros((T, wl.d_model)), g, a, v, keep, count, idx, val, overflow, band, z=z)


def _exact_case(wl, C):
    T = wl.tokens
    inp = synth.make_inputs(wl)
    res = _oracle_gate(inp, T, C)
    # exact grid: z is a sum of 8 grid values and every partial sum of z·B is
    # an integer number of grid units below 2^24, so fp32 is exact in any order
    assert oracle.exact_grid_ok(res.z, synth.to_f64(inp.B).T, 14)
    lib = _lib()
    dev_in = _device_inputs(inp, T)
    for _ in range(2):  # two calls in a row share the scratch
        g = _call(lib, dev_in, T, C)
        assert np.array_equal(g.count, res.count)
        assert np.array_equal(g.idx, res.idx)
        assert np.array_equal(g.val, res.val)
        assert np.array_equal(g.overflow, res.overflow)
    return res


@pytest.mark.parametrize("T,C", [(16, 32), (64, 8)])
def test_noalloc_matches_oracle_exact_grid_twice(T, C):
    wl = synth.Workload("noalloc", 1024, 2048, T, rank=128, exact_grid=True, tile_capacity=C)
    res = _exact_case(wl, C)
    if C == 8:
        assert res.overflow.any()


def test_noalloc_partial_last_rank_tile():
    # rank 192: z has one full 128-row tile and one of 64 rows
    wl = synth.Workload("noalloc", 1024, 2048, 24, rank=192, exact_grid=True, tile_capacity=32)
    _exact_case(wl, 32)


def test_noalloc_at_its_maximum_sizes():
    # T = 64, d_model = 4096, rank = 1024, d_ff = 16384: every split partial,
    # z row and ticket of the fixed scratch is in use
    wl = synth.Workload("noalloc", 4096, 16384, 64, rank=1024, exact_grid=True, tile_capacity=32)
    _exact_case(wl, 32)


def test_noalloc_matches_oracle_gaussian_within_band():
    T, C = 32, 32
    wl = synth.WORKLOADS["lopa_bf16"].with_(tokens=T, d_model=2048, d_ff=4096, rank=256)
    inp = synth.make_inputs(wl)
    res = _oracle_gate(inp, T, C)
    amb = ambiguous(res, wl.mode, wl.threshold, wl.k, exact=False)
    lib = _lib()
    dev_in = _device_inputs(inp, T)
    for _ in range(2):
        g = _call(lib, dev_in, T, C)
        # counts, indices, ascending slots, pads and overflow flags exactly
        # outside the decision band; values within one bf16 rounding plus the
        # gate's accumulation band
        compare_twell(g, res, C, amb, exact_vals=False, dtype="bf16")


def test_noalloc_reports_an_expired_wait_and_recovers():
    T, C = 16, 32
    wl = synth.Workload("noalloc", 1024, 2048, T, rank=128, exact_grid=True, tile_capacity=C)
    inp = synth.make_inputs(wl)
    res = _oracle_gate(inp, T, C)
    lib = _lib()
    dev_in = _device_inputs(inp, T)
    assert lib.sffn_lowrank_twell_noalloc_status(_stream()) == SFFN_OK
    lib.sffn_debug_noalloc_waits(20000)   # 20 ms on a barrier that nothing signals
    try:
        _call(lib, dev_in, T, C, check_status=False)
    except AssertionError:
        pass  # the outputs of a timed-out call are undefined
    finally:
        lib.sffn_debug_noalloc_waits(0)
    assert lib.sffn_lowrank_twell_noalloc_status(_stream()) == SFFN_ERR_TIMEOUT
    # read and cleared: the next read is clean, the next call correct
    assert lib.sffn_lowrank_twell_noalloc_status(_stream()) == SFFN_OK
    g = _call(lib, dev_in, T, C)
    assert np.array_equal(g.idx, res.idx) and np.array_equal(g.val, res.val)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = _lib()
    f = lib.sffn_lowrank_twell_noalloc
    fake = 0x7F0000000000
    args = lambda T, d, r, F: (fake, T, d, fake, r, fake, F, None, 0, 0.0, 32,  # noqa: E731
                               fake, fake, fake, fake, None)
    assert f(*args(65, 1024, 128, 2048)) == SFFN_ERR_UNSUPPORTED
    assert f(*args(16, 8192, 128, 2048)) == SFFN_ERR_UNSUPPORTED
    assert f(*args(16, 1024, 2048, 2048)) == SFFN_ERR_UNSUPPORTED
    assert f(*args(16, 1024, 128, 32768)) == SFFN_ERR_UNSUPPORTED
    assert f(*args(0, 1024, 128, 2048)) == SFFN_OK
