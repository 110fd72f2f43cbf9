"""The C-ABI library loads, exports every symbol include/mxq.h declares, and rejects bad
arguments before touching the GPU (these run without a GPU)."""
import ctypes
import os
import re

import pytest

from fp8_mixed_precision_mxq_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxq.h")

V = ctypes.c_void_p
A16 = V(4096)          # a 16-byte aligned non-null dummy pointer (never dereferenced)
A8 = V(4096 + 8)       # misaligned


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(mxq_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("mxq_quantize_weight", "mxq_quantize_act", "mxq_linear", "mxq_dit_block_linears",
                 "mxq_gemm", "mxq_dequantize", "mxq_last_error"):
        assert must in names


def test_library_exports_every_declared_symbol():
    L = _lib.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in _lib.SIGNATURES, "binding lacks " + name


def test_sizes():
    L = _lib.lib()
    assert L.mxq_codes_bytes(3, 64, 0) == 96
    assert L.mxq_codes_bytes(3, 64, 1) == 192
    assert L.mxq_sf_bytes(1, 32) == 128 * 4
    assert L.mxq_sf_bytes(129, 160) == 256 * 8
    assert L.mxq_sf_bytes(32760, 5120) == 32768 * 160
    assert L.mxq_sf_bytes(5, 48) == -1
    assert L.mxq_workspace_bytes(0, 8, 32, 0, 0) == -1
    assert L.mxq_workspace_bytes(128, 256, 1024, 0, 0) == 128 * 512 + 128 * 32
    assert L.mxq_workspace_bytes(128, 256, 1024, 1, 1) > L.mxq_workspace_bytes(128, 256, 1024, 1, 0)


@pytest.mark.parametrize("args,status", [
    ((None, 4, 64, 0, A16, A16, None), _lib.ERR_INVALID_ARG),      # null input
    ((A16, 0, 64, 0, A16, A16, None), _lib.ERR_INVALID_ARG),       # M = 0
    ((A16, 4, 48, 0, A16, A16, None), _lib.ERR_SHAPE),             # K % 32 != 0
    ((A16, 4, 64, 2, A16, A16, None), _lib.ERR_INVALID_ARG),       # unknown format
    ((A8, 4, 64, 0, A16, A16, None), _lib.ERR_ALIGN),              # misaligned input
    ((A16, 4, 64, 1, A8, A16, None), _lib.ERR_ALIGN),              # misaligned codes
])
def test_quantize_rejects_bad_arguments(args, status):
    L = _lib.lib()
    assert L.mxq_quantize_act(*args) == status
    assert _lib.last_error()


def test_gemm_rejects_bad_arguments():
    L = _lib.lib()
    ok = (A16, A16, 0, 128, 256, A16, A16, 256, None, A16, None)
    bad = [
        ((A16, A16, 0, 128, 256, A16, A16, 250, None, A16, None), _lib.ERR_SHAPE),   # N % 8
        ((A16, A16, 1, 128, 96, A16, A16, 256, None, A16, None), _lib.ERR_SHAPE),    # W4A8 K % 128
        ((A16, A16, 1, 128, 256, A8, A16, 256, None, A16, None), _lib.ERR_ALIGN),    # W4A8 weight 32B
        ((A16, A16, 0, 128, 256, A16, A16, 256, A8, A16, None), _lib.ERR_ALIGN),     # bias
        ((A16, None, 0, 128, 256, A16, A16, 256, None, A16, None), _lib.ERR_INVALID_ARG),
        ((A16, A16, 0, -3, 256, A16, A16, 256, None, A16, None), _lib.ERR_INVALID_ARG),
    ]
    for args, status in bad:
        assert L.mxq_gemm(*args) == status, (args, _lib.last_error())
    # valid arguments get past validation and only then need a device
    rc = L.mxq_gemm(*ok)
    assert rc in (_lib.ERR_CUDA, _lib.ERR_UNSUPPORTED, _lib.OK)


def test_linear_rejects_small_workspace_and_bad_mode():
    L = _lib.lib()
    ws = V(1 << 20)
    assert L.mxq_linear(A16, 128, 256, A16, A16, 256, None, 0, 7, ws, 1 << 30, A16, None) == _lib.ERR_INVALID_ARG
    assert L.mxq_linear(A16, 128, 256, A16, A16, 256, None, 0, 0, V(4096 + 16), 1 << 30, A16,
                        None) == _lib.ERR_ALIGN   # workspace must be 256-byte aligned


def test_block_rejects_bad_mask():
    L = _lib.lib()
    descs = (_lib.WDesc * 8)()
    xs = (ctypes.c_void_p * 8)()
    ms = (ctypes.c_int64 * 8)()
    ys = (ctypes.c_void_p * 8)()
    assert L.mxq_dit_block_linears(descs, xs, ms, ys, 0x100, 0, A16, 0, None) == _lib.ERR_INVALID_ARG
    assert L.mxq_dit_block_linears(None, xs, ms, ys, 0, 0, A16, 0, None) == _lib.ERR_INVALID_ARG


def test_gemm_gelu_quant_rejects_bad_arguments():
    L = _lib.lib()
    #        a_codes a_sf fmt  M    K   w_codes w_sf  N   bias out_fmt codes sf  h  stream
    bad = [
        ((A16, A16, 0, 128, 256, A16, A16, 264, None, 0, A16, A16, None, None), _lib.ERR_SHAPE),  # N % 32
        ((A16, A16, 0, 128, 256, A16, A16, 256, None, 5, A16, A16, None, None), _lib.ERR_INVALID_ARG),  # out_fmt
        ((A16, A16, 0, 128, 256, A16, A16, 256, None, 1, A16, None, None, None), _lib.ERR_INVALID_ARG),  # out_sf
        ((A16, A16, 0, 128, 256, A16, A16, 256, None, 1, A8, A16, None, None), _lib.ERR_ALIGN),  # out_codes
        ((A16, A16, 0, 128, 256, A16, A16, 256, None, 0, A16, A16, A8, None), _lib.ERR_ALIGN),  # h
    ]
    for args, status in bad:
        assert L.mxq_gemm_gelu_quant(*args) == status, (args, _lib.last_error())


def test_gemm_quant_rejects_bad_arguments():
    L = _lib.lib()
    #        a_codes a_sf fmt  M    K   w_codes w_sf  N   bias act out_fmt codes sf  h  stream
    bad = [
        ((A16, A16, 0, 128, 256, A16, A16, 256, None, 2, 0, A16, A16, None, None), _lib.ERR_INVALID_ARG),  # act
        ((A16, A16, 0, 128, 256, A16, A16, 256, None, -1, 0, A16, A16, None, None), _lib.ERR_INVALID_ARG),  # act
        ((A16, A16, 0, 128, 256, A16, A16, 264, None, 0, 0, A16, A16, None, None), _lib.ERR_SHAPE),  # N % 32
        ((A16, A16, 0, 128, 256, A16, A16, 256, None, 0, 5, A16, A16, None, None), _lib.ERR_INVALID_ARG),  # out_fmt
        ((A16, A16, 0, 128, 256, A16, A16, 256, None, 1, 1, A8, A16, None, None), _lib.ERR_ALIGN),  # out_codes
    ]
    for args, status in bad:
        assert L.mxq_gemm_quant(*args) == status, (args, _lib.last_error())


def test_ffn_workspace_and_shape_checks():
    L = _lib.lib()
    assert L.mxq_ffn_workspace_bytes(128, 256, 512, 0, 1) > 0
    assert L.mxq_ffn_workspace_bytes(128, 250, 512, 0, 1) == -1
    assert L.mxq_ffn_workspace_bytes(128, 256, 512, 0, 3) == -1
    up = _lib.WDesc(4096, 4096, None, 512, 256)
    down = _lib.WDesc(4096, 4096, None, 256, 512)
    wrong = _lib.WDesc(4096, 4096, None, 256, 384)  # K differs from the hidden width
    ws = V(1 << 20)
    need = L.mxq_ffn_workspace_bytes(128, 256, 512, 0, 0)
    assert L.mxq_ffn(A16, 128, 256, ctypes.byref(up), ctypes.byref(wrong), 0, 0, ws, need, A16,
                     None) == _lib.ERR_SHAPE
    assert L.mxq_ffn(A16, 128, 128, ctypes.byref(up), ctypes.byref(down), 0, 0, ws, need, A16,
                     None) == _lib.ERR_SHAPE
    assert L.mxq_ffn(A16, 128, 256, ctypes.byref(up), ctypes.byref(down), 0, 0, ws, need - 1, A16,
                     None) == _lib.ERR_WORKSPACE
    assert L.mxq_ffn(A16, 128, 256, None, ctypes.byref(down), 0, 0, ws, need, A16, None) == _lib.ERR_INVALID_ARG


def test_static_entry_points_reject_bad_arguments():
    L = _lib.lib()
    for bad_scale in (0.0, -1.0, float("inf"), float("nan")):
        assert L.mxq_quantize_act_static(A16, 128, 256, bad_scale, A16, A16, None) == _lib.ERR_INVALID_ARG
        assert L.mxq_linear_static(A16, 128, 256, A16, A16, 256, None, bad_scale, V(1 << 20), 1 << 30, A16,
                                   None) == _lib.ERR_INVALID_ARG
    assert L.mxq_quantize_act_static(A16, 128, 250, 0.5, A16, A16, None) == _lib.ERR_SHAPE
    assert L.mxq_linear_static(A16, 128, 96, A16, A16, 256, None, 0.5, V(1 << 20), 1 << 30, A16,
                               None) == _lib.ERR_SHAPE  # W4A8 GEMM needs K % 128
    assert L.mxq_linear_static(A16, 128, 256, A16, A16, 256, None, 0.5, V(1 << 20), 16, A16,
                               None) == _lib.ERR_WORKSPACE
    assert L.mxq_absmax(A16, 12, A16, None) == _lib.ERR_SHAPE
    assert L.mxq_absmax(A8, 16, A16, None) == _lib.ERR_ALIGN


def test_transform_entry_points_reject_bad_arguments():
    L = _lib.lib()
    assert L.mxq_quantize_act_transformed(A16, 128, 256, 0, None, 64, A16, A16, None) == _lib.ERR_INVALID_ARG
    assert L.mxq_quantize_act_transformed(A16, 128, 96, 0, None, 128, A16, A16, None) == _lib.ERR_SHAPE
    assert L.mxq_quantize_act_transformed(A16, 128, 256, 0, A8, 32, A16, A16, None) == _lib.ERR_ALIGN
    assert L.mxq_quantize_weight_transformed(A16, 128, 256, None, 33, A16, A16, None) == _lib.ERR_INVALID_ARG
    assert L.mxq_linear_transformed(A16, 128, 256, A16, A16, 256, None, 0, None, 48, V(1 << 20), 1 << 30, A16,
                                    None) == _lib.ERR_INVALID_ARG
    assert L.mxq_linear_transformed(A16, 128, 256, A16, A16, 256, None, 0, None, 32, V(1 << 20), 16, A16,
                                    None) == _lib.ERR_WORKSPACE


def test_lowrank_entry_point_rejects_bad_arguments():
    L = _lib.lib()
    for bad_rank in (0, 32, 96, 320):
        assert L.mxq_linear_lowrank(A16, 128, 256, A16, A16, 256, None, 0, A16, A16, bad_rank, V(1 << 20), 1 << 30,
                                    A16, None) == _lib.ERR_INVALID_ARG
        assert L.mxq_lowrank_workspace_bytes(128, 256, 256, 0, bad_rank) == -1
    assert L.mxq_linear_lowrank(A16, 128, 256, A16, A16, 256, None, 0, A8, A16, 64, V(1 << 20), 1 << 30, A16,
                                None) == _lib.ERR_ALIGN
    need = L.mxq_lowrank_workspace_bytes(128, 256, 256, 0, 64)
    assert need > L.mxq_workspace_bytes(128, 256, 256, 0, 0)
    assert L.mxq_linear_lowrank(A16, 128, 256, A16, A16, 256, None, 0, A16, A16, 64, V(1 << 20), need - 1, A16,
                                None) == _lib.ERR_WORKSPACE


def test_gemm_quant_binding_rejects_unknown_activation():
    from fp8_mixed_precision_mxq_b200 import ops
    with pytest.raises(ValueError):
        ops.gemm_quant(None, None, "e2m1", 128, 256, None, act="relu")


def test_linear_entry_points_reject_unsupported_shapes_with_their_reason():
    """The shape limits the header states, through every entry point that runs a GEMM:
    N % 8 != 0 and, for native W4A8, K % 128 != 0 return MXQ_ERR_SHAPE with the reason
    in mxq_last_error(), before anything needs a device."""
    L = _lib.lib()
    ws = V(1 << 20)
    for mode in (0, 1):
        assert L.mxq_linear(A16, 128, 256, A16, A16, 250, None, 0, mode, ws, 1 << 30, A16, None) == _lib.ERR_SHAPE
        assert "multiple of 8" in _lib.last_error()
    assert L.mxq_linear(A16, 128, 96, A16, A16, 256, None, 1, 0, ws, 1 << 30, A16, None) == _lib.ERR_SHAPE
    assert "K % 128" in _lib.last_error()
    assert L.mxq_linear_noalloc(A16, 128, 96, A16, A16, 256, None, 1, A16, None) == _lib.ERR_SHAPE
    assert "K % 128" in _lib.last_error()
    assert L.mxq_linear_noalloc(A16, 128, 256, A16, A16, 252, None, 0, A16, None) == _lib.ERR_SHAPE
    assert "multiple of 8" in _lib.last_error()
    # W4A4 takes K = 96 (only native W4A8 expands the weight in 128-element steps)
    rc = L.mxq_linear(A16, 128, 96, A16, A16, 256, None, 0, 0, ws, 1 << 30, A16, None)
    assert rc != _lib.ERR_SHAPE, _lib.last_error()
    descs = (_lib.WDesc * 8)(*[_lib.WDesc(4096, 4096, None, 256, 96)] * 8)
    xs = (ctypes.c_void_p * 8)(*[4096] * 8)
    ms = (ctypes.c_int64 * 8)(*[128] * 8)
    ys = (ctypes.c_void_p * 8)(*[4096] * 8)
    assert L.mxq_dit_block_linears(descs, xs, ms, ys, 0x80, 0, ws, 1 << 30, None) == _lib.ERR_SHAPE
    assert "block linear 7" in _lib.last_error() and "K % 128" in _lib.last_error()


def test_gelu_entry_point_rejects_bad_arguments():
    L = _lib.lib()
    assert L.mxq_gelu_bf16(A16, 0, A16, None) == _lib.ERR_INVALID_ARG
    assert L.mxq_gelu_bf16(None, 8, A16, None) == _lib.ERR_INVALID_ARG
    assert L.mxq_gelu_bf16(V(4096 + 1), 8, A16, None) == _lib.ERR_ALIGN
    assert L.mxq_gelu_bf16(A16, 8, V(4096 + 1), None) == _lib.ERR_ALIGN


def test_bf16_gemm_quantizing_a_rejects_bad_arguments():
    """mxq_gemm_bf16_quant_a checks before any launch: the output is at most 128 wide, a's K
    holds whole MX blocks, the format is known, and the MX buffers are 16-byte aligned."""
    L = _lib.lib()
    args = lambda M=64, K=128, N=64, fmt=_lib.FMT_E2M1, codes=A16, sf=A16: (  # noqa: E731
        A16, M, K, A16, N, None, A16, fmt, codes, sf, None)
    assert L.mxq_gemm_bf16_quant_a(*args(N=136)) == _lib.ERR_SHAPE
    assert "above 128" in _lib.last_error()
    assert L.mxq_gemm_bf16_quant_a(*args(K=40)) == _lib.ERR_SHAPE
    assert L.mxq_gemm_bf16_quant_a(*args(N=12)) == _lib.ERR_SHAPE
    assert L.mxq_gemm_bf16_quant_a(*args(fmt=7)) == _lib.ERR_INVALID_ARG
    assert L.mxq_gemm_bf16_quant_a(*args(M=0)) == _lib.ERR_INVALID_ARG
    assert L.mxq_gemm_bf16_quant_a(*args(codes=V(4096 + 8))) == _lib.ERR_ALIGN
    assert L.mxq_gemm_bf16_quant_a(*args(sf=None)) == _lib.ERR_INVALID_ARG
