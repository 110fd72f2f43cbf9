"""MX block-quantized W4A4 / W4A8 linear layers on B200 (sm_100a).

The compute lives in libmxq.so (hand-written CUDA: the MX quantizer, the dequantizer
and tcgen05 block-scaled GEMMs) behind the C ABI of include/mxq.h; this package is
the Python binding of that ABI.
"""
from ._lib import FMT_E2M1, FMT_E4M3, MODE_NATIVE, MODE_QDQ, MxqError, lib  # noqa: F401
from .ops import (QWeight, block_workspace_bytes, codes_bytes, dequantize, dit_block_linears, gemm,  # noqa: F401
                  last_path, linear, poll_status, quantize_act, quantize_weight, set_debug, sf_bytes,
                  sf_to_logical, workspace_bytes)
