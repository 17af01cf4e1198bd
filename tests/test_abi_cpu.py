"""Host-side checks of the C ABI (no GPU needed): the library builds and loads,
exports every entry point include/sffn.h declares, and rejects bad arguments
before touching CUDA."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

from activation_sparse_gated_relu_b200 import binding as B
from activation_sparse_gated_relu_b200.build import HEADER, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return B.load_library()


def _declared_symbols() -> set[str]:
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"\b(sffn_[a-z_]+)\s*\(", text))


def test_header_declares_the_north_star_calls():
    syms = _declared_symbols()
    assert {"sffn_create", "sffn_forward", "sffn_destroy"} <= syms


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (sffn_\w+)", out))
    missing = _declared_symbols() - exported
    assert not missing, missing
    for s in _declared_symbols():
        assert hasattr(lib, s)


def test_status_strings(lib):
    for s in range(8):
        assert B.status_string(s) and B.status_string(s) != "unknown status"
    assert B.status_string(99) == "unknown status"
    assert "sm_100a" in B.sffn_version()


def _desc(**kw):
    d = B.sffn_desc()
    d.d_model, d.d_ff, d.max_tokens, d.rank = 4096, 14336, 8, 0
    d.dtype, d.mode, d.act = B.SFFN_BF16, B.SFFN_MODE_RELU_THRESHOLD, B.SFFN_ACT_RELU
    d.threshold, d.k, d.tile_capacity, d.path, d.flags = 0.0, 0, 32, 0, 0
    fake = 0x7F0000000000  # 16-byte aligned, never dereferenced by validation
    d.W_gate, d.W_up, d.W_down, d.gate_bias = fake, fake + 0x100, fake + 0x200, fake + 0x300
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def _create(lib, d):
    h = ctypes.c_void_p()
    s = lib.sffn_create(ctypes.byref(d) if d is not None else None, None, ctypes.byref(h))
    return s, h


@pytest.mark.parametrize("kw,want", [
    (dict(d_ff=14335), B.SFFN_ERR_UNSUPPORTED),           # not a multiple of 128
    (dict(d_ff=32768), B.SFFN_ERR_UNSUPPORTED),           # int16 indices
    (dict(d_model=4100), B.SFFN_ERR_UNSUPPORTED),         # d % 8
    (dict(d_model=8192), B.SFFN_ERR_UNSUPPORTED),
    (dict(d_model=0), B.SFFN_ERR_INVALID_ARG),
    (dict(max_tokens=0), B.SFFN_ERR_INVALID_ARG),
    (dict(max_tokens=1 << 20), B.SFFN_ERR_UNSUPPORTED),
    (dict(tile_capacity=24), B.SFFN_ERR_INVALID_ARG),
    (dict(dtype=7), B.SFFN_ERR_INVALID_ARG),
    (dict(mode=3), B.SFFN_ERR_INVALID_ARG),
    (dict(act=5), B.SFFN_ERR_INVALID_ARG),
    (dict(path=9), B.SFFN_ERR_INVALID_ARG),
    (dict(threshold=-1.0), B.SFFN_ERR_INVALID_ARG),
    (dict(threshold=float("nan")), B.SFFN_ERR_INVALID_ARG),
    (dict(W_up=None), B.SFFN_ERR_INVALID_ARG),
    (dict(W_gate=None), B.SFFN_ERR_INVALID_ARG),         # dense gate needs W_gate
    (dict(W_gate=0x7F0000000008), B.SFFN_ERR_INVALID_ARG),  # misaligned
    (dict(rank=512), B.SFFN_ERR_INVALID_ARG),             # W_gate given with rank > 0
    (dict(mode=1, k=20000), B.SFFN_ERR_INVALID_ARG),      # k > d_ff
    (dict(mode=1, k=100, tile_capacity=32), B.SFFN_ERR_UNSUPPORTED),  # WINA needs C = 128
    (dict(mode=1, k=-1, tile_capacity=128), B.SFFN_ERR_INVALID_ARG),  # k < 0
    (dict(flags=1 << 7), B.SFFN_ERR_INVALID_ARG),         # an undefined flag bit
    (dict(dtype=B.SFFN_FP32, d_ff=16384), B.SFFN_ERR_UNSUPPORTED),  # fp32 rows kernel: d_ff <= 8192
])
def test_create_rejects_bad_descriptors(lib, kw, want):
    s, h = _create(lib, _desc(**kw))
    assert s == want, (kw, B.status_string(s))
    assert h.value is None


def test_create_lowrank_rules(lib):
    fake = 0x7F0000001000
    ok = dict(rank=512, W_gate=None, A=fake, B=fake + 0x100)
    assert _create(lib, _desc(**ok))[0] in (B.SFFN_ERR_NO_DEVICE, B.SFFN_OK)
    assert _create(lib, _desc(**{**ok, "rank": 100}))[0] == B.SFFN_ERR_UNSUPPORTED
    assert _create(lib, _desc(**{**ok, "dtype": B.SFFN_FP32}))[0] == B.SFFN_ERR_UNSUPPORTED
    assert _create(lib, _desc(**{**ok, "B": None}))[0] == B.SFFN_ERR_INVALID_ARG
    assert _create(lib, _desc(**{**ok, "rank": 4160}))[0] == B.SFFN_ERR_UNSUPPORTED
    # the dense debug gate exists for the dense gate only
    assert _create(lib, _desc(**{**ok, "flags": B.SFFN_FLAG_DEBUG_GATE}))[0] == B.SFFN_ERR_UNSUPPORTED


def test_null_arguments(lib):
    h = ctypes.c_void_p()
    assert lib.sffn_create(None, None, ctypes.byref(h)) == B.SFFN_ERR_INVALID_ARG
    d = _desc()
    assert lib.sffn_create(ctypes.byref(d), None, None) == B.SFFN_ERR_INVALID_ARG
    assert lib.sffn_destroy(None) == B.SFFN_OK
    assert lib.sffn_forward(None, None, 1, None, None) == B.SFFN_ERR_INVALID_ARG
    assert lib.sffn_forward_host(None, None, 1, None, None) == B.SFFN_ERR_INVALID_ARG
    assert lib.sffn_read_status(None, None) == B.SFFN_ERR_INVALID_ARG
    assert lib.sffn_get_stats(None, None, None) == B.SFFN_ERR_INVALID_ARG
    assert lib.sffn_debug_set_epoch(None, 5) == B.SFFN_ERR_INVALID_ARG
    assert lib.sffn_debug_decode_waits(None, 0, 0) == B.SFFN_ERR_INVALID_ARG


@pytest.mark.skipif(os.path.exists("/dev/nvidia0"), reason="a GPU is present")
def test_valid_descriptor_without_gpu_reports_no_device(lib):
    s, h = _create(lib, _desc())
    assert s == B.SFFN_ERR_NO_DEVICE and h.value is None


def test_binding_raises_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(ImportError):
        B.load_library(str(tmp_path / "missing.so"))


def _handle_stub(dtype: str = "bf16", d_model: int = 64, max_tokens: int = 8):
    """A SparseFFN whose argument checks run without a device: the checks use
    only the descriptor-level attributes, and every bad call below must raise
    before the library is reached (a null handle would be rejected there)."""
    import torch
    f = B.SparseFFN.__new__(B.SparseFFN)
    f.h = None
    f.dtype = dtype
    f._torch_dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
    f.d_model, f.d_ff, f.max_tokens = d_model, 256, max_tokens
    return f


def test_binding_rejects_mismatched_activations():
    import torch
    f = _handle_stub()
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="x must be torch.bfloat16"):
        f.forward(x.float())                           # fp32 x on a bf16 handle
    with pytest.raises(ValueError, match="shape"):
        f.forward(torch.zeros((4, 32), dtype=torch.bfloat16))   # wrong d_model
    with pytest.raises(ValueError, match="contiguous"):
        f.forward(torch.zeros((64, 4), dtype=torch.bfloat16).t())  # a transposed view
    with pytest.raises(ValueError, match="CUDA"):
        f.forward(x)                                   # host tensor on the device entry point
    with pytest.raises(ValueError, match="max_tokens"):
        f.forward(torch.zeros((9, 64), dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="out must be torch.float32"):
        f.forward_host(x, torch.zeros((4, 64), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out must have shape"):
        f.forward_host(x, torch.zeros((3, 64), dtype=torch.float32))


def test_binding_rejects_host_or_misshaped_weights():
    import torch
    W = torch.zeros((256, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        B.SparseFFN(W, W, W_gate=W)                   # host weights
    with pytest.raises(ValueError, match="give either W_gate"):
        B.SparseFFN(W, W)                             # no gate at all


def test_gsi_create_rejects_bad_descriptors(lib):
    fake = 0x7F0000000000
    def desc(**kw):
        d = B.sffn_gsi_desc()
        d.d_in, d.d_out, d.k, d.max_tokens, d.eps, d.W, d.Vk = 4096, 16384, 256, 8, 0.1, fake, fake
        for k, v in kw.items():
            setattr(d, k, v)
        return d
    h = ctypes.c_void_p()
    for kw, want in [({"d_in": 4100}, B.SFFN_ERR_UNSUPPORTED), ({"k": 513}, B.SFFN_ERR_UNSUPPORTED),
                     ({"max_tokens": 65}, B.SFFN_ERR_UNSUPPORTED), ({"k": 0}, B.SFFN_ERR_INVALID_ARG),
                     ({"eps": -1.0}, B.SFFN_ERR_INVALID_ARG), ({"W": None}, B.SFFN_ERR_INVALID_ARG),
                     ({"W": fake + 8}, B.SFFN_ERR_INVALID_ARG), ({"d_in": 64, "k": 128}, B.SFFN_ERR_INVALID_ARG)]:
        d = desc(**kw)
        assert lib.sffn_gsi_create(ctypes.byref(d), None, ctypes.byref(h)) == want, kw
        assert not h.value
    assert lib.sffn_gsi_create(ctypes.byref(desc()), None, ctypes.byref(h)) == B.SFFN_ERR_NO_DEVICE
    assert lib.sffn_gsi_destroy(None) == B.SFFN_OK
