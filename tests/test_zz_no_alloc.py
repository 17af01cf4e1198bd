"""The allocation-free low-rank gate entry point (sffn_lowrank_twell_noalloc).

It serves callers that cannot allocate device memory where they run (code in
a runtime that owns all device memory, or on a latency-critical path where
cudaMalloc may synchronise or fail): its scratch lives in fixed arrays inside
the library.  These tests call it through the C ABI twice in a row and check
that its TwELL records match those sffn_forward produces on the same inputs,
bit for bit on exact-grid inputs and under the usual decision band on Gaussian
ones.  This file is collected last so that a run stopping at the first failure
has already run every other test.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from activation_sparse_gated_relu_b200 import SFFN_ERR_UNSUPPORTED, SFFN_OK, binding

from parity_util import make_ffn, run_gpu

pytestmark = pytest.mark.gpu


def _lib():
    lib = binding.load_library()
    f = lib.sffn_lowrank_twell_noalloc
    vp = ctypes.c_void_p
    f.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, vp, ctypes.c_int, vp, ctypes.c_int,
                  ctypes.c_float, ctypes.c_int, vp, vp, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


def _call(f, inp, T, C):
    wl = inp.wl
    d, r, F = wl.d_model, wl.rank, wl.d_ff
    dev = lambda t: t.to("cuda").contiguous()  # noqa: E731
    x, At, Bt = dev(inp.x[:T]), dev(inp.A.t()), dev(inp.B.t())
    bias = dev(inp.bias) if inp.bias is not None else None
    P = F // 128
    count = torch.full((T, P), -7, dtype=torch.int16, device="cuda")
    idx = torch.full((T, P, C), -7, dtype=torch.int16, device="cuda")
    val = torch.full((T, P, C), 7.0, dtype=torch.bfloat16, device="cuda")
    ovf = torch.full((T,), 0xDEAD, dtype=torch.int32, device="cuda")
    st = f(x.data_ptr(), T, d, At.data_ptr(), r, Bt.data_ptr(), F,
           bias.data_ptr() if bias is not None else None, 0 if wl.act == "relu" else 1,
           float(wl.threshold), C, count.data_ptr(), idx.data_ptr(), val.data_ptr(), ovf.data_ptr(),
           torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == SFFN_OK, binding.status_string(st)
    return (count.cpu().numpy(), idx.cpu().numpy(), val.float().cpu().numpy().astype(np.float64),
            ovf.cpu().numpy() != 0)


def _reference(inp, T, C):
    ffn = make_ffn(inp, max_tokens=T, C=C, path="tiles")
    g = run_gpu(ffn, inp.x[:T])
    ffn.close()
    return g


@pytest.mark.parametrize("T,C", [(16, 32), (64, 8)])
def test_noalloc_matches_forward_exact_grid_twice(T, C):
    wl = synth.Workload("noalloc", 1024, 2048, T, rank=128, exact_grid=True, tile_capacity=C)
    inp = synth.make_inputs(wl)
    ref = _reference(inp, T, C)
    f = _lib()
    for _ in range(2):  # two calls in a row share the scratch
        count, idx, val, ovf = _call(f, inp, T, C)
        assert np.array_equal(count, ref.count)
        assert np.array_equal(idx, ref.idx)
        assert np.array_equal(val, ref.val)
        assert np.array_equal(ovf, ref.overflow)
    if C == 8:
        assert ovf.any()


def test_noalloc_matches_forward_gaussian_within_band():
    T, C = 32, 32
    wl = synth.WORKLOADS["lopa_bf16"].with_(tokens=T, d_model=2048, d_ff=4096, rank=256)
    inp = synth.make_inputs(wl)
    ref = _reference(inp, T, C)
    res = oracle.forward_inputs(inp)
    amb = np.abs(res.g - wl.threshold) <= res.band     # the usual decision band
    amb_tile = amb.reshape(T, -1, 128).any(-1)
    f = _lib()
    for _ in range(2):
        count, idx, val, ovf = _call(f, inp, T, C)
        same = (count == ref.count) & (idx == ref.idx).all(-1)
        assert np.all(same | amb_tile)
        # same tolerance as the parity tests: one rounding of the stored bf16
        # value plus twice the gate's decision band at that neuron (z is summed
        # with split-K atomics, so a z coordinate at a bf16 rounding midpoint
        # may round either way between two runs)
        band = res.band[np.arange(T)[:, None, None], np.maximum(ref.idx, 0)]
        close = np.abs(val - ref.val) <= 2.0 ** -7 * np.abs(ref.val) + 2 * band
        assert np.all(close.all(-1) | amb_tile)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    f = _lib()
    fake = 0x7F0000000000
    args = lambda T, d, r, F: (fake, T, d, fake, r, fake, F, None, 0, 0.0, 32,  # noqa: E731
                               fake, fake, fake, fake, None)
    assert f(*args(65, 1024, 128, 2048)) == SFFN_ERR_UNSUPPORTED
    assert f(*args(16, 8192, 128, 2048)) == SFFN_ERR_UNSUPPORTED
    assert f(*args(16, 1024, 2048, 2048)) == SFFN_ERR_UNSUPPORTED
    assert f(*args(16, 1024, 128, 32768)) == SFFN_ERR_UNSUPPORTED
    assert f(*args(0, 1024, 128, 2048)) == SFFN_OK
