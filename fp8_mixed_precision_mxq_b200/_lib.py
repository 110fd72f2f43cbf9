"""ctypes binding of libmxq.so (argument marshalling only; every step runs in the
library's CUDA kernels).  Loading fails loudly if the library was not built."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmxq.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_SHAPE = 2
ERR_ALIGN = 3
ERR_UNSUPPORTED = 4
ERR_CUDA = 5
ERR_TIMEOUT = 6
ERR_WORKSPACE = 7
STATUS_NAMES = {0: "MXQ_OK", 1: "MXQ_ERR_INVALID_ARG", 2: "MXQ_ERR_SHAPE", 3: "MXQ_ERR_ALIGN",
                4: "MXQ_ERR_UNSUPPORTED", 5: "MXQ_ERR_CUDA", 6: "MXQ_ERR_TIMEOUT", 7: "MXQ_ERR_WORKSPACE"}

FMT_E2M1 = 0
FMT_E4M3 = 1
ACT_NONE = 0
ACT_GELU = 1
MODE_NATIVE = 0
MODE_QDQ = 1

# Every symbol include/mxq.h declares, with its ctypes signature.
_vp, _i64, _i32, _u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32


class WDesc(ctypes.Structure):
    """mxq_wdesc: one linear layer's quantized weights."""
    _fields_ = [("codes", _vp), ("sf", _vp), ("bias", _vp), ("N", _i64), ("K", _i64)]


SIGNATURES = {
    "mxq_version": ([], _i32),
    "mxq_codes_bytes": ([_i64, _i64, _i32], _i64),
    "mxq_sf_bytes": ([_i64, _i64], _i64),
    "mxq_workspace_bytes": ([_i64, _i64, _i64, _i32, _i32], _i64),
    "mxq_quantize_weight": ([_vp, _i64, _i64, _vp, _vp, _vp], _i32),
    "mxq_quantize_act": ([_vp, _i64, _i64, _i32, _vp, _vp, _vp], _i32),
    "mxq_dequantize": ([_vp, _vp, _i64, _i64, _i32, _vp, _vp], _i32),
    "mxq_gemm": ([_vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp], _i32),
    "mxq_gemm_bf16": ([_vp, _i64, _i64, _vp, _i64, _vp, _vp, _vp], _i32),
    "mxq_gemm_bf16_quant_a": ([_vp, _i64, _i64, _vp, _i64, _vp, _vp, _i32, _vp, _vp, _vp], _i32),
    "mxq_channel_absmax": ([_vp, _i64, _i64, _vp, _vp], _i32),
    "mxq_smooth_scales": ([_vp, _vp, _i64, ctypes.c_float, _vp, _vp, _vp], _i32),
    "mxq_sqnr": ([ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_i64), _i32, _vp, _vp], _i32),
    "mxq_lowrank_split": ([_vp, _i64, _vp, _vp, _i64, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp], _i32),
    "mxq_linear": ([_vp, _i64, _i64, _vp, _vp, _i64, _vp, _i32, _i32, _vp, _i64, _vp, _vp], _i32),
    "mxq_dit_block_linears": ([ctypes.POINTER(WDesc), ctypes.POINTER(_vp), ctypes.POINTER(_i64),
                               ctypes.POINTER(_vp), _u32, _i32, _vp, _i64, _vp], _i32),
    "mxq_block_workspace_bytes": ([ctypes.POINTER(WDesc), ctypes.POINTER(_i64), _u32, _i32], _i64),
    "mxq_block_workspace_min_bytes": ([ctypes.POINTER(WDesc), ctypes.POINTER(_i64), _u32, _i32], _i64),
    "mxq_linear_noalloc": ([_vp, _i64, _i64, _vp, _vp, _i64, _vp, _i32, _vp, _vp], _i32),
    "mxq_linear_noalloc_max_scratch_bytes": ([], _i64),
    "mxq_gemm_gelu_quant": ([_vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _vp], _i32),
    "mxq_gemm_quant": ([_vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _i32, _i32, _vp, _vp, _vp, _vp], _i32),
    "mxq_gelu_bf16": ([_vp, _i64, _vp, _vp], _i32),
    "mxq_ffn": ([_vp, _i64, _i64, ctypes.POINTER(WDesc), ctypes.POINTER(WDesc), _i32, _i32, _vp, _i64, _vp, _vp],
                _i32),
    "mxq_ffn_workspace_bytes": ([_i64, _i64, _i64, _i32, _i32], _i64),
    "mxq_quantize_act_static": ([_vp, _i64, _i64, ctypes.c_float, _vp, _vp, _vp], _i32),
    "mxq_linear_static": ([_vp, _i64, _i64, _vp, _vp, _i64, _vp, ctypes.c_float, _vp, _i64, _vp, _vp], _i32),
    "mxq_absmax": ([_vp, _i64, _vp, _vp], _i32),
    "mxq_select_policy": ([ctypes.c_double, ctypes.c_double, _i32], _i32),
    "mxq_tier_thresholds": ([_i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double),
                             ctypes.POINTER(ctypes.c_double)], _i32),
    "mxq_linear_lowrank": ([_vp, _i64, _i64, _vp, _vp, _i64, _vp, _i32, _vp, _vp, _i64, _vp, _i64, _vp, _vp], _i32),
    "mxq_lowrank_workspace_bytes": ([_i64, _i64, _i64, _i32, _i64], _i64),
    "mxq_quantize_act_transformed": ([_vp, _i64, _i64, _i32, _vp, _i32, _vp, _vp, _vp], _i32),
    "mxq_quantize_weight_transformed": ([_vp, _i64, _i64, _vp, _i32, _vp, _vp, _vp], _i32),
    "mxq_linear_transformed": ([_vp, _i64, _i64, _vp, _vp, _i64, _vp, _i32, _vp, _i32, _vp, _i64, _vp, _vp],
                               _i32),
    "mxq_sf_to_logical": ([_vp, _i64, _i64, _vp, _vp], _i32),
    "mxq_poll_status": ([_vp], _i32),
    "mxq_set_debug": ([_u32], _i32),
    "mxq_last_error": ([], ctypes.c_char_p),
    "mxq_last_path": ([], ctypes.c_char_p),
}

_lib = None


class MxqError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        self.status = status
        super().__init__("%s returned %s: %s" % (where, STATUS_NAMES.get(status, status), message))


def lib():
    """Load libmxq.so (building it first if the sources are newer and nvcc exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            from . import build as _build
            try:
                _build.build()
            except Exception as e:  # noqa: BLE001
                raise ImportError("libmxq.so is missing and could not be built: %s" % e) from e
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def last_error() -> str:
    return lib().mxq_last_error().decode()


def last_path() -> str:
    return lib().mxq_last_path().decode()


def check(status: int, where: str) -> None:
    if status != OK:
        raise MxqError(status, where, last_error())
