"""Activation-sparse gated FFN forward for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library libsffn.so (include/sffn.h) built from
csrc/; this package only marshals arguments to it.
"""
from .binding import (  # noqa: F401
    SFFN_ACT_RELU, SFFN_ACT_SILU, SFFN_BF16, SFFN_ERR_ALLOC, SFFN_ERR_CUDA, SFFN_ERR_DEVICE,
    SFFN_ERR_INVALID_ARG, SFFN_ERR_NO_DEVICE, SFFN_ERR_TIMEOUT, SFFN_ERR_UNSUPPORTED,
    SFFN_FLAG_DEBUG_GATE, SFFN_FP32, SFFN_MODE_RELU_THRESHOLD, SFFN_MODE_WINA_TOPK, SFFN_OK,
    SFFN_PATH_AUTO, SFFN_PATH_ROWS, SFFN_PATH_TILES, GsiLinear, MoeFFN, SffnError, SparseFFN, load_library,
    sffn_create, sffn_desc, sffn_destroy, sffn_forward, sffn_forward_host, sffn_get_stats,
    sffn_read_status, sffn_stats, sffn_timing_begin, sffn_timing_end, sffn_version, status_string,
)
