"""ctypes binding of libsffn.so: the same entry points as include/sffn.h.

Argument marshalling only.  Every step of the forward runs in the library's
CUDA kernels; if the library is missing this module raises instead of falling
back to anything else.  PyTorch supplies device memory and the stream.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsffn.so")

# status codes (include/sffn.h)
SFFN_OK, SFFN_ERR_INVALID_ARG, SFFN_ERR_UNSUPPORTED, SFFN_ERR_ALLOC, SFFN_ERR_CUDA, \
    SFFN_ERR_TIMEOUT, SFFN_ERR_DEVICE, SFFN_ERR_NO_DEVICE = range(8)
SFFN_BF16, SFFN_FP32 = 0, 1
SFFN_MODE_RELU_THRESHOLD, SFFN_MODE_WINA_TOPK, SFFN_MODE_WINA_FULL_H = 0, 1, 2
SFFN_ACT_RELU, SFFN_ACT_SILU = 0, 1
SFFN_PATH_AUTO, SFFN_PATH_ROWS, SFFN_PATH_TILES = 0, 1, 2
SFFN_FLAG_DEBUG_GATE = 1
SFFN_FLAG_SEPARATE = 2
SFFN_FLAG_COOPERATIVE = 4
SFFN_FLAG_BACKWARD = 8


class sffn_desc(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int), ("d_ff", ctypes.c_int), ("max_tokens", ctypes.c_int),
        ("rank", ctypes.c_int), ("dtype", ctypes.c_int), ("mode", ctypes.c_int),
        ("act", ctypes.c_int), ("threshold", ctypes.c_float), ("k", ctypes.c_int),
        ("tile_capacity", ctypes.c_int), ("path", ctypes.c_int), ("flags", ctypes.c_uint),
        ("W_gate", ctypes.c_void_p), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p),
        ("W_up", ctypes.c_void_p), ("W_down", ctypes.c_void_p), ("gate_bias", ctypes.c_void_p),
        ("input_k", ctypes.c_int), ("V", ctypes.c_void_p),
    ]


class sffn_gsi_desc(ctypes.Structure):
    _fields_ = [("d_in", ctypes.c_int), ("d_out", ctypes.c_int), ("k", ctypes.c_int),
                ("max_tokens", ctypes.c_int), ("eps", ctypes.c_float), ("W", ctypes.c_void_p),
                ("Vk", ctypes.c_void_p)]


class sffn_moe_desc(ctypes.Structure):
    _fields_ = [("n_experts", ctypes.c_int), ("top_k", ctypes.c_int), ("d_model", ctypes.c_int),
                ("d_ff", ctypes.c_int), ("rank", ctypes.c_int), ("max_tokens", ctypes.c_int),
                ("tile_capacity", ctypes.c_int), ("threshold", ctypes.c_float), ("W_router", ctypes.c_void_p),
                ("A", ctypes.POINTER(ctypes.c_void_p)), ("B", ctypes.POINTER(ctypes.c_void_p)),
                ("W_up", ctypes.POINTER(ctypes.c_void_p)), ("W_down", ctypes.POINTER(ctypes.c_void_p)),
                ("gate_bias", ctypes.POINTER(ctypes.c_void_p))]


class sffn_stats(ctypes.Structure):
    _fields_ = [("n_overflow", ctypes.c_int), ("n_launches", ctypes.c_int), ("path", ctypes.c_int),
                ("epoch", ctypes.c_uint), ("launch_attrs", ctypes.c_uint)]


class SffnError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})" if what else status_string(status))


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsffn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m activation_sparse_gated_relu_b200.build`")
    lib = ctypes.CDLL(path)
    vp, ip, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
    lib.sffn_create.argtypes = [ctypes.POINTER(sffn_desc), vp, ctypes.POINTER(vp)]
    lib.sffn_create.restype = st
    lib.sffn_forward.argtypes = [vp, vp, ip, vp, vp]
    lib.sffn_forward.restype = st
    lib.sffn_forward_host.argtypes = [vp, vp, ip, vp, vp]
    lib.sffn_forward_host.restype = st
    lib.sffn_destroy.argtypes = [vp]
    lib.sffn_destroy.restype = st
    lib.sffn_status_string.argtypes = [st]
    lib.sffn_status_string.restype = ctypes.c_char_p
    lib.sffn_read_status.argtypes = [vp, vp]
    lib.sffn_read_status.restype = st
    lib.sffn_debug_twell.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                                     ctypes.POINTER(vp), ctypes.POINTER(ip), ctypes.POINTER(ip)]
    lib.sffn_debug_twell.restype = st
    lib.sffn_debug_decode_waits.argtypes = [vp, ctypes.c_int, ctypes.c_uint]
    lib.sffn_debug_decode_waits.restype = st
    lib.sffn_debug_set_epoch.argtypes = [vp, ctypes.c_uint]
    lib.sffn_debug_set_epoch.restype = st
    lib.sffn_debug_keep.argtypes = [vp, ctypes.POINTER(vp)]
    lib.sffn_debug_keep.restype = st
    lib.sffn_debug_tile_schedule.argtypes = [ip, ip, ip, ip, vp, ip, vp, ctypes.POINTER(ip)]
    lib.sffn_debug_tile_schedule.restype = st
    lib.sffn_debug_gate.argtypes = [vp, ctypes.POINTER(vp)]
    lib.sffn_debug_gate.restype = st
    lib.sffn_backward.argtypes = [vp, vp, vp, ip, vp, vp, vp, vp, vp, vp]
    lib.sffn_backward.restype = st
    lib.sffn_workspace_bytes.argtypes = [vp, ctypes.POINTER(ctypes.c_size_t)]
    lib.sffn_workspace_bytes.restype = st
    lib.sffn_debug_norms.argtypes = [vp, ctypes.POINTER(vp)]
    lib.sffn_debug_norms.restype = st
    lib.sffn_get_stats.argtypes = [vp, vp, ctypes.POINTER(sffn_stats)]
    lib.sffn_get_stats.restype = st
    lib.sffn_timing_begin.argtypes = [vp, ip, ip]
    lib.sffn_timing_begin.restype = st
    lib.sffn_timing_end.argtypes = [vp, ip, vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ip),
                                    ctypes.POINTER(ip)]
    lib.sffn_timing_end.restype = st
    lib.sffn_gsi_create.argtypes = [ctypes.POINTER(sffn_gsi_desc), vp, ctypes.POINTER(vp)]
    lib.sffn_gsi_create.restype = st
    lib.sffn_gsi_forward.argtypes = [vp, vp, ip, vp, vp]
    lib.sffn_gsi_forward.restype = st
    lib.sffn_gsi_destroy.argtypes = [vp]
    lib.sffn_gsi_destroy.restype = st
    lib.sffn_gsi_stats.argtypes = [vp, vp, ctypes.POINTER(ip)]
    lib.sffn_gsi_stats.restype = st
    lib.sffn_gsi_debug.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(ip),
                                   ctypes.POINTER(vp)]
    lib.sffn_gsi_debug.restype = st
    lib.sffn_gsi_timing_begin.argtypes = [vp, ip, ip]
    lib.sffn_gsi_timing_begin.restype = st
    lib.sffn_gsi_timing_end.argtypes = [vp, ip, vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ip),
                                        ctypes.POINTER(ip)]
    lib.sffn_gsi_timing_end.restype = st
    lib.sffn_moe_create.argtypes = [ctypes.POINTER(sffn_moe_desc), vp, ctypes.POINTER(vp)]
    lib.sffn_moe_create.restype = st
    lib.sffn_moe_forward.argtypes = [vp, vp, ip, vp, vp]
    lib.sffn_moe_forward.restype = st
    lib.sffn_moe_destroy.argtypes = [vp]
    lib.sffn_moe_destroy.restype = st
    lib.sffn_moe_expert.argtypes = [vp, ip, ctypes.POINTER(vp)]
    lib.sffn_moe_expert.restype = st
    lib.sffn_moe_debug.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp)]
    lib.sffn_moe_debug.restype = st
    lib.sffn_moe_read_status.argtypes = [vp, vp]
    lib.sffn_moe_read_status.restype = st
    lib.sffn_moe_timing_begin.argtypes = [vp, ip, ip]
    lib.sffn_moe_timing_begin.restype = st
    lib.sffn_moe_timing_end.argtypes = [vp, ip, vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ip),
                                        ctypes.POINTER(ip)]
    lib.sffn_moe_timing_end.restype = st
    lib.sffn_version.argtypes = []
    lib.sffn_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(s: int) -> str:
    return load_library().sffn_status_string(int(s)).decode()


def _check(status: int, what: str) -> None:
    if status != SFFN_OK:
        raise SffnError(status, what)


# ----------------------------------------------------------------- raw entry points
def sffn_create(desc: sffn_desc, stream: int = 0) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(load_library().sffn_create(ctypes.byref(desc), ctypes.c_void_p(stream), ctypes.byref(h)),
           "sffn_create")
    return h


def sffn_forward(h, x_ptr: int, T: int, out_ptr: int, stream: int = 0) -> None:
    _check(load_library().sffn_forward(h, ctypes.c_void_p(x_ptr), int(T), ctypes.c_void_p(out_ptr),
                                       ctypes.c_void_p(stream)), "sffn_forward")


def sffn_forward_host(h, x_ptr: int, T: int, out_ptr: int, stream: int = 0) -> None:
    _check(load_library().sffn_forward_host(h, ctypes.c_void_p(x_ptr), int(T),
                                            ctypes.c_void_p(out_ptr), ctypes.c_void_p(stream)),
           "sffn_forward_host")


def sffn_destroy(h) -> None:
    _check(load_library().sffn_destroy(h), "sffn_destroy")


def sffn_read_status(h, stream: int = 0) -> int:
    return load_library().sffn_read_status(h, ctypes.c_void_p(stream))


def sffn_get_stats(h, stream: int = 0) -> sffn_stats:
    st = sffn_stats()
    _check(load_library().sffn_get_stats(h, ctypes.c_void_p(stream), ctypes.byref(st)), "sffn_get_stats")
    return st


def sffn_timing_begin(h, max_forwards: int, stride: int = 1) -> None:
    _check(load_library().sffn_timing_begin(h, int(max_forwards), int(stride)), "sffn_timing_begin")


def sffn_timing_end(h, fn: str = "sffn_timing_end") -> dict:
    """{label: (total_ms, launches)} over the forwards timed since sffn_timing_begin."""
    n_max = 24
    names = (ctypes.c_char * 32 * n_max)()
    ms = (ctypes.c_float * n_max)()
    cnt = (ctypes.c_int * n_max)()
    n = ctypes.c_int()
    _check(getattr(load_library(), fn)(h, n_max, ctypes.cast(names, ctypes.c_void_p), ms, cnt,
                                       ctypes.byref(n)), fn)
    return {names[i].value.decode(): (float(ms[i]), int(cnt[i])) for i in range(min(n.value, n_max))}


def sffn_version() -> str:
    return load_library().sffn_version().decode()


# ----------------------------------------------------------------- torch convenience
class _CudaView:
    """Zero-copy __cuda_array_interface__ view of library-owned device memory."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


def _view(ptr: int, shape, typestr: str, torch_dtype=None):
    import torch
    t = torch.as_tensor(_CudaView(ptr, shape, typestr), device="cuda")
    if torch_dtype is not None:
        t = t.view(torch_dtype)
    return t.clone()


def _check_tensor(t, name: str, dtype, shape, cuda: bool) -> None:
    """The C ABI sees only a pointer: the dtype, shape, device and layout of
    every tensor are checked here, before the call."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")
    if t.is_cuda != cuda:
        raise ValueError(f"{name} must be a {'CUDA' if cuda else 'host (CPU)'} tensor")
    if t.numel() and t.data_ptr() % 16:
        raise ValueError(f"{name} must start on a 16-byte boundary")


_DTYPE = {"bf16": SFFN_BF16, "fp32": SFFN_FP32}
_MODE = {"relu_threshold": SFFN_MODE_RELU_THRESHOLD, "wina_topk": SFFN_MODE_WINA_TOPK,
         "wina_full_h": SFFN_MODE_WINA_FULL_H}
_ACT = {"relu": SFFN_ACT_RELU, "silu": SFFN_ACT_SILU}
_PATH = {"auto": SFFN_PATH_AUTO, "rows": SFFN_PATH_ROWS, "tiles": SFFN_PATH_TILES}


class SparseFFN:
    """A handle over device tensors (the tensors are kept alive by the object).

    Weights are neuron-major [d_ff][d_model] (W_down is down_proj.weight^T);
    A is [d_model][rank], B is [rank][d_ff]; bias is fp32 [d_ff].
    """

    def __init__(self, W_up, W_down, *, W_gate=None, A=None, B=None, bias=None,
                 mode: str = "relu_threshold", act: str = "relu", threshold: float = 0.0,
                 k: int = 0, tile_capacity: int = 32, max_tokens: int = 8, path: str = "auto",
                 debug_gate: bool = False, separate: bool = False, cooperative: bool = False,
                 input_k: int = 0, V=None, backward: bool = False, stream: Optional[int] = None):
        import torch
        self.h = None
        self._keep = [t for t in (W_up, W_down, W_gate, A, B, bias, V) if t is not None]
        dt = W_up.dtype
        if dt not in (torch.bfloat16, torch.float32):
            raise TypeError("operands must be bf16 or fp32")
        if W_up.dim() != 2:
            raise ValueError("W_up must be [d_ff][d_model]")
        if (W_gate is None) == (A is None):
            raise ValueError("give either W_gate (dense gate) or A and B (low-rank gate)")
        self.dtype = "bf16" if dt == torch.bfloat16 else "fp32"
        self._torch_dtype = dt
        F, d = W_up.shape
        _check_tensor(W_up, "W_up", dt, (F, d), True)
        _check_tensor(W_down, "W_down", dt, (F, d), True)
        if W_gate is not None:
            _check_tensor(W_gate, "W_gate", dt, (F, d), True)
        else:
            if B is None or A.dim() != 2:
                raise ValueError("the low-rank gate needs A [d_model][rank] and B [rank][d_ff]")
            _check_tensor(A, "A", dt, (d, A.shape[1]), True)
            _check_tensor(B, "B", dt, (A.shape[1], F), True)
        if bias is not None:
            _check_tensor(bias, "bias", torch.float32, (F,), True)
        if V is not None:
            _check_tensor(V, "V", dt, (d, d), True)
        self.d_model, self.d_ff, self.max_tokens = d, F, max_tokens
        desc = sffn_desc()
        desc.d_model, desc.d_ff, desc.max_tokens = d, F, max_tokens
        desc.rank = 0 if A is None else A.shape[1]
        desc.dtype = _DTYPE[self.dtype]
        desc.mode = _MODE[mode]
        desc.act = _ACT[act]
        desc.threshold = float(threshold)
        desc.k = int(k)
        desc.tile_capacity = int(tile_capacity)
        desc.path = _PATH[path]
        desc.flags = ((SFFN_FLAG_DEBUG_GATE if debug_gate else 0) | (SFFN_FLAG_SEPARATE if separate else 0)
                      | (SFFN_FLAG_COOPERATIVE if cooperative else 0) | (SFFN_FLAG_BACKWARD if backward else 0))
        ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        desc.W_gate, desc.A, desc.B = ptr(W_gate), ptr(A), ptr(B)
        desc.W_up, desc.W_down, desc.gate_bias = ptr(W_up), ptr(W_down), ptr(bias)
        desc.input_k = int(input_k or 0)
        desc.V = ptr(V)
        self.desc = desc
        self.h = sffn_create(desc, self._stream(stream))

    @staticmethod
    def _stream(stream: Optional[int]) -> int:
        import torch
        return torch.cuda.current_stream().cuda_stream if stream is None else int(stream)

    def _check_io(self, x, out, cuda: bool) -> int:
        import torch
        if not isinstance(x, torch.Tensor) or x.dim() != 2:
            raise ValueError("x must be a [T][d_model] tensor")
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"T = {T} exceeds max_tokens = {self.max_tokens}")
        _check_tensor(x, "x", self._torch_dtype, (T, self.d_model), cuda)
        if out is not None:
            _check_tensor(out, "out", torch.float32, (T, self.d_model), cuda)
            if cuda and out.device != x.device:
                raise ValueError("x and out must be on the same device")
        return T

    def forward(self, x, out=None, stream: Optional[int] = None):
        import torch
        T = self._check_io(x, out, cuda=True)
        if out is None:
            out = torch.empty((T, self.d_model), dtype=torch.float32, device=x.device)
        sffn_forward(self.h, x.data_ptr(), T, out.data_ptr(), self._stream(stream))
        return out

    __call__ = forward

    def backward(self, x, dy, *, dx=None, dW_gate=None, dW_up=None, dW_down=None, d_bias=None,
                 with_bias: bool = True, stream: Optional[int] = None) -> dict:
        """Gradients of the last forward for upstream dy (fp32 [T][d_model]):
        {dx, dW_gate, dW_up, dW_down, d_bias} as fp32 device tensors."""
        import torch
        T = self._check_io(x, None, cuda=True)
        _check_tensor(dy, "dy", torch.float32, (T, self.d_model), True)
        z = lambda shape: torch.empty(shape, dtype=torch.float32, device=x.device)  # noqa: E731
        dx = z((T, self.d_model)) if dx is None else dx
        dW_gate = z((self.d_ff, self.d_model)) if dW_gate is None else dW_gate
        dW_up = z((self.d_ff, self.d_model)) if dW_up is None else dW_up
        dW_down = z((self.d_ff, self.d_model)) if dW_down is None else dW_down
        if with_bias and d_bias is None:
            d_bias = z((self.d_ff,))
        for name, t, shape in (("dx", dx, (T, self.d_model)), ("dW_gate", dW_gate, (self.d_ff, self.d_model)),
                               ("dW_up", dW_up, (self.d_ff, self.d_model)),
                               ("dW_down", dW_down, (self.d_ff, self.d_model))):
            _check_tensor(t, name, torch.float32, shape, True)
        if d_bias is not None:
            _check_tensor(d_bias, "d_bias", torch.float32, (self.d_ff,), True)
        p = lambda t: ctypes.c_void_p(t.data_ptr() if t is not None else None)  # noqa: E731
        _check(load_library().sffn_backward(self.h, p(x), p(dy), T, p(dx), p(dW_gate), p(dW_up), p(dW_down),
                                            p(d_bias), ctypes.c_void_p(self._stream(stream))), "sffn_backward")
        return {"dx": dx, "dW_gate": dW_gate, "dW_up": dW_up, "dW_down": dW_down, "d_bias": d_bias}

    def forward_host(self, x_host, out_host=None, stream: Optional[int] = None):
        import torch
        T = self._check_io(x_host, out_host, cuda=False)
        if out_host is None:
            out_host = torch.empty((T, self.d_model), dtype=torch.float32, pin_memory=True)
        sffn_forward_host(self.h, x_host.data_ptr(), T, out_host.data_ptr(), self._stream(stream))
        return out_host

    def twell(self, T: int) -> dict:
        """Copies of the last forward's TwELL records and overflow flags."""
        lib = load_library()
        vp = ctypes.c_void_p
        c, i, v, o = vp(), vp(), vp(), vp()
        nt, cap = ctypes.c_int(), ctypes.c_int()
        _check(lib.sffn_debug_twell(self.h, ctypes.byref(c), ctypes.byref(i), ctypes.byref(v),
                                    ctypes.byref(o), ctypes.byref(nt), ctypes.byref(cap)), "twell")
        P, C = nt.value, cap.value
        import torch
        vt = ("<u2", torch.bfloat16) if self.dtype == "bf16" else ("<f4", None)
        return {"count": _view(c.value, (T, P), "<i2"), "idx": _view(i.value, (T, P, C), "<i2"),
                "val": _view(v.value, (T, P, C), vt[0], vt[1]),
                "overflow_epoch": _view(o.value, (T,), "<u4")}

    def debug_decode_waits(self, phantom_ctas: int, wait_us: int) -> None:
        """Test hook: single-launch decode forwards await `phantom_ctas` CTAs
        that never run, with waits of `wait_us` µs (0, 0 restores)."""
        _check(load_library().sffn_debug_decode_waits(self.h, phantom_ctas, wait_us), "debug_decode_waits")

    def debug_set_epoch(self, epoch: int) -> None:
        """Test hook: the next forward takes epoch `epoch` + 1 (0 skipped)."""
        _check(load_library().sffn_debug_set_epoch(self.h, epoch), "debug_set_epoch")

    def keep_masks(self, T: int):
        """The last ROWS-path forward's keep masks, uint32 [T][n_tiles][4]."""
        k = ctypes.c_void_p()
        _check(load_library().sffn_debug_keep(self.h, ctypes.byref(k)), "keep_masks")
        return _view(k.value, (T, self.d_ff // 128, 4), "<u4")

    def gate_debug(self, T: int):
        g = ctypes.c_void_p()
        _check(load_library().sffn_debug_gate(self.h, ctypes.byref(g)), "gate_debug")
        return _view(g.value, (T, self.d_ff), "<f4")

    def workspace_bytes(self) -> int:
        """Bytes of device memory the handle allocated (one workspace)."""
        n = ctypes.c_size_t()
        _check(load_library().sffn_workspace_bytes(self.h, ctypes.byref(n)), "workspace_bytes")
        return int(n.value)

    def norms(self):
        n = ctypes.c_void_p()
        _check(load_library().sffn_debug_norms(self.h, ctypes.byref(n)), "norms")
        return _view(n.value, (self.d_ff,), "<f4")

    def stats(self, stream: Optional[int] = None) -> sffn_stats:
        return sffn_get_stats(self.h, self._stream(stream))

    def timing_begin(self, max_forwards: int, stride: int = 1) -> None:
        sffn_timing_begin(self.h, max_forwards, stride)

    def timing_end(self) -> dict:
        return sffn_timing_end(self.h)

    def read_status(self, stream: Optional[int] = None) -> int:
        return sffn_read_status(self.h, self._stream(stream))

    def close(self) -> None:
        if getattr(self, "h", None) is not None and self.h.value:
            sffn_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class GsiLinear:
    """Gated subspace linear layer over device tensors: y = M·bf16(V_k^T x)
    for tokens whose residual ratio is below eps, y = W x for the others.
    W is [d_out][d_in] bf16, V_k is [d_in][k] bf16 (orthonormal columns)."""

    def __init__(self, W, Vk, eps: float, max_tokens: int = 8, stream: Optional[int] = None):
        import torch
        self.h = None
        if W.dim() != 2 or Vk.dim() != 2:
            raise ValueError("W must be [d_out][d_in] and Vk [d_in][k]")
        d_out, d_in = W.shape
        k = Vk.shape[1]
        _check_tensor(W, "W", torch.bfloat16, (d_out, d_in), True)
        _check_tensor(Vk, "Vk", torch.bfloat16, (d_in, k), True)
        self._keep = [W, Vk]
        self.d_in, self.d_out, self.k, self.max_tokens = d_in, d_out, k, max_tokens
        desc = sffn_gsi_desc()
        desc.d_in, desc.d_out, desc.k, desc.max_tokens = d_in, d_out, k, max_tokens
        desc.eps = float(eps)
        desc.W, desc.Vk = W.data_ptr(), Vk.data_ptr()
        h = ctypes.c_void_p()
        _check(load_library().sffn_gsi_create(ctypes.byref(desc), ctypes.c_void_p(SparseFFN._stream(stream)),
                                              ctypes.byref(h)), "sffn_gsi_create")
        self.h = h

    def forward(self, x, y=None, stream: Optional[int] = None):
        import torch
        if not isinstance(x, torch.Tensor) or x.dim() != 2:
            raise ValueError("x must be a [T][d_in] tensor")
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"T = {T} exceeds max_tokens = {self.max_tokens}")
        _check_tensor(x, "x", torch.bfloat16, (T, self.d_in), True)
        if y is None:
            y = torch.empty((T, self.d_out), dtype=torch.float32, device=x.device)
        _check_tensor(y, "y", torch.float32, (T, self.d_out), True)
        _check(load_library().sffn_gsi_forward(self.h, ctypes.c_void_p(x.data_ptr()), T,
                                               ctypes.c_void_p(y.data_ptr()),
                                               ctypes.c_void_p(SparseFFN._stream(stream))), "sffn_gsi_forward")
        return y

    __call__ = forward

    def n_slow(self, stream: Optional[int] = None) -> int:
        n = ctypes.c_int()
        _check(load_library().sffn_gsi_stats(self.h, ctypes.c_void_p(SparseFFN._stream(stream)), ctypes.byref(n)),
               "sffn_gsi_stats")
        return int(n.value)

    def debug(self, T: int) -> dict:
        import torch
        vp = ctypes.c_void_p
        g, part, M = vp(), vp(), vp()
        n = ctypes.c_int()
        _check(load_library().sffn_gsi_debug(self.h, ctypes.byref(g), ctypes.byref(part), ctypes.byref(n),
                                             ctypes.byref(M)), "sffn_gsi_debug")
        p = _view(part.value, (n.value, self.max_tokens, 2), "<f4")[:, :T, :]
        return {"g": _view(g.value, (T, self.k), "<f4"), "rn2": p[:, :, 0].sum(0), "xn2": p[:, :, 1].sum(0),
                "M": _view(M.value, (self.d_out, self.k), "<u2", torch.bfloat16)}

    def timing_begin(self, max_forwards: int, stride: int = 1) -> None:
        _check(load_library().sffn_gsi_timing_begin(self.h, int(max_forwards), int(stride)), "sffn_gsi_timing_begin")

    def timing_end(self) -> dict:
        return sffn_timing_end(self.h, "sffn_gsi_timing_end")

    def close(self) -> None:
        if getattr(self, "h", None) is not None and self.h.value:
            _check(load_library().sffn_gsi_destroy(self.h), "sffn_gsi_destroy")
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class MoeFFN:
    """Mixture of LoPA-gated sparse experts over device tensors.

    experts: a list of dicts with A [d][rank], B [rank][d_ff], W_up and W_down
    [d_ff][d] (bf16) and bias [d_ff] fp32 (<= 0) or None; W_router [E][d]."""

    def __init__(self, W_router, experts: list, top_k: int, *, threshold: float = 0.0,
                 tile_capacity: int = 32, max_tokens: int = 8, stream: Optional[int] = None):
        import torch
        self.h = None
        E = len(experts)
        if E == 0:
            raise ValueError("at least one expert")
        F, d = experts[0]["W_up"].shape
        r = experts[0]["A"].shape[1]
        _check_tensor(W_router, "W_router", torch.bfloat16, (E, d), True)
        for e, ex in enumerate(experts):
            _check_tensor(ex["A"], f"A[{e}]", torch.bfloat16, (d, r), True)
            _check_tensor(ex["B"], f"B[{e}]", torch.bfloat16, (r, F), True)
            _check_tensor(ex["W_up"], f"W_up[{e}]", torch.bfloat16, (F, d), True)
            _check_tensor(ex["W_down"], f"W_down[{e}]", torch.bfloat16, (F, d), True)
            if ex.get("bias") is not None:
                _check_tensor(ex["bias"], f"bias[{e}]", torch.float32, (F,), True)
        self._keep = [W_router] + [t for ex in experts for t in ex.values() if t is not None]
        self.d_model, self.d_ff, self.n_experts, self.top_k, self.max_tokens = d, F, E, top_k, max_tokens
        arr = lambda key: (ctypes.c_void_p * E)(*[  # noqa: E731
            (ex[key].data_ptr() if ex.get(key) is not None else None) for ex in experts])
        self._arrays = {k: arr(k) for k in ("A", "B", "W_up", "W_down", "bias")}
        desc = sffn_moe_desc()
        desc.n_experts, desc.top_k, desc.d_model, desc.d_ff, desc.rank = E, top_k, d, F, r
        desc.max_tokens, desc.tile_capacity, desc.threshold = max_tokens, tile_capacity, float(threshold)
        desc.W_router = W_router.data_ptr()
        cast = lambda a: ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))  # noqa: E731
        desc.A, desc.B = cast(self._arrays["A"]), cast(self._arrays["B"])
        desc.W_up, desc.W_down = cast(self._arrays["W_up"]), cast(self._arrays["W_down"])
        desc.gate_bias = cast(self._arrays["bias"]) if all(ex.get("bias") is not None for ex in experts) else None
        h = ctypes.c_void_p()
        _check(load_library().sffn_moe_create(ctypes.byref(desc), ctypes.c_void_p(SparseFFN._stream(stream)),
                                              ctypes.byref(h)), "sffn_moe_create")
        self.h = h

    def forward(self, x, out=None, stream: Optional[int] = None):
        import torch
        if not isinstance(x, torch.Tensor) or x.dim() != 2:
            raise ValueError("x must be a [T][d_model] tensor")
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"T = {T} exceeds max_tokens = {self.max_tokens}")
        _check_tensor(x, "x", torch.bfloat16, (T, self.d_model), True)
        if out is None:
            out = torch.empty((T, self.d_model), dtype=torch.float32, device=x.device)
        _check_tensor(out, "out", torch.float32, (T, self.d_model), True)
        _check(load_library().sffn_moe_forward(self.h, ctypes.c_void_p(x.data_ptr()), T,
                                               ctypes.c_void_p(out.data_ptr()),
                                               ctypes.c_void_p(SparseFFN._stream(stream))), "sffn_moe_forward")
        return out

    __call__ = forward

    def routing(self, T: int) -> dict:
        vp = ctypes.c_void_p
        sel, w, lg = vp(), vp(), vp()
        _check(load_library().sffn_moe_debug(self.h, ctypes.byref(sel), ctypes.byref(w), ctypes.byref(lg)),
               "sffn_moe_debug")
        return {"sel": _view(sel.value, (T, self.top_k), "<i4"), "w": _view(w.value, (T, self.top_k), "<f4"),
                "logits": _view(lg.value, (T, self.n_experts), "<f4")}

    def expert_twell(self, e: int, T: int) -> dict:
        """Copies of expert e's TwELL records for its last block of T rows."""
        import torch
        eh = ctypes.c_void_p()
        _check(load_library().sffn_moe_expert(self.h, int(e), ctypes.byref(eh)), "sffn_moe_expert")
        view = SparseFFN.__new__(SparseFFN)      # a non-owning view: the MoE handle owns the expert
        view.h, view.dtype, view._torch_dtype = None, "bf16", torch.bfloat16
        view.d_model, view.d_ff, view.max_tokens = self.d_model, self.d_ff, self.max_tokens
        view.h = eh
        try:
            return view.twell(T)
        finally:
            view.h = None

    def read_status(self, stream: Optional[int] = None) -> int:
        return load_library().sffn_moe_read_status(self.h, ctypes.c_void_p(SparseFFN._stream(stream)))

    def timing_begin(self, max_forwards: int, stride: int = 1) -> None:
        _check(load_library().sffn_moe_timing_begin(self.h, int(max_forwards), int(stride)), "sffn_moe_timing_begin")

    def timing_end(self) -> dict:
        return sffn_timing_end(self.h, "sffn_moe_timing_end")

    def close(self) -> None:
        if getattr(self, "h", None) is not None and self.h.value:
            _check(load_library().sffn_moe_destroy(self.h), "sffn_moe_destroy")
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
