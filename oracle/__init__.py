"""CPU oracle for the MX block-quantized linear layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library does not use it, and it
shares no code with the CUDA library.

The arithmetic lives in ``mx_oracle.c`` (plain C, fp64), which restates the MX
format of the blog "Quark Mixed-Precision Quantization for Wan2.2 Video Generation
on AMD Instinct GPUs" (section "Quantization formats": OCP MXFP4 weights, dynamic
MXFP4 or FP8 E4M3 activations, 32-element blocks with an E8M0 shared scale, RTN).
This module only builds that library and marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

E2M1 = 0
E4M3 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mx_oracle.c")
_LIB = os.path.join(_HERE, "libmx_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``mx_oracle.c`` with gcc into ``libmx_oracle.so`` next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
             "-D_GNU_SOURCE", _SRC, "-o", tmp, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        # MXO_LIB_OVERRIDE lets the mutation tests load a deliberately broken copy.
        override = os.environ.get("MXO_LIB_OVERRIDE")
        _lib = ctypes.CDLL(override if override else build())
        L = _lib
        i64, i32, vp, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_double
        L.mxo_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.mxo_bf16_to_double.restype = dbl
        L.mxo_encode_elem.argtypes = [dbl, i32]
        L.mxo_encode_elem.restype = i32
        L.mxo_decode_elem.argtypes = [i32, i32]
        L.mxo_decode_elem.restype = dbl
        L.mxo_scale_code.argtypes = [dbl, i32, i32]
        L.mxo_scale_code.restype = i32
        L.mxo_scale_value.argtypes = [i32]
        L.mxo_scale_value.restype = dbl
        L.mxo_quantize.argtypes = [vp, i64, i64, i32, vp, vp, i32]
        L.mxo_quantize.restype = i32
        L.mxo_dequantize.argtypes = [vp, vp, i64, i64, i32, vp]
        L.mxo_dequantize.restype = i32
        L.mxo_sf_tiled_bytes.argtypes = [i64, i64]
        L.mxo_sf_tiled_bytes.restype = i64
        L.mxo_sf_tiled_offset.argtypes = [i64, i64, i64]
        L.mxo_sf_tiled_offset.restype = i64
        L.mxo_sf_to_tiled.argtypes = [vp, i64, i64, vp]
        L.mxo_sf_to_tiled.restype = i32
        L.mxo_linear_rows.argtypes = [vp, vp, i32, vp, i64, i64, vp, vp, i64, vp, vp, i32]
        L.mxo_linear_rows.restype = i32
        L.mxo_double_to_bf16.argtypes = [dbl]
        L.mxo_double_to_bf16.restype = ctypes.c_uint16
        L.mxo_gelu.argtypes = [dbl]
        L.mxo_gelu.restype = dbl
        L.mxo_round_bf16.argtypes = [vp, i64, vp]
        L.mxo_round_bf16.restype = None
        L.mxo_gelu_bf16.argtypes = [vp, i64, vp]
        L.mxo_gelu_bf16.restype = None
        L.mxo_quantize_static_e4m3.argtypes = [vp, i64, ctypes.c_float, vp]
        L.mxo_quantize_static_e4m3.restype = i32
        L.mxo_linear_rows_scaled.argtypes = [vp, vp, i32, vp, i64, i64, vp, vp, i64, vp, dbl, vp, i32]
        L.mxo_linear_rows_scaled.restype = i32
        L.mxo_quantize_transformed.argtypes = [vp, i64, i64, vp, i32, i32, vp, vp, vp, vp, vp, vp, i32]
        L.mxo_quantize_transformed.restype = i32
        L.mxo_linear_lowrank_rows.argtypes = [vp, vp, i32, vp, i64, i64, vp, vp, i64, vp, vp, vp, i64, vp, vp, i32]
        L.mxo_linear_lowrank_rows.restype = i32
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def encode_elem(y: float, fmt: int) -> int:
    """Element code of y rounded to the E2M1 / E4M3 grid (RNE, saturating)."""
    return lib().mxo_encode_elem(float(y), fmt)


def decode_elem(code: int, fmt: int) -> float:
    return lib().mxo_decode_elem(int(code), fmt)


def scale_code(amax: float, fmt: int, nonfinite: bool = False) -> int:
    return lib().mxo_scale_code(float(amax), int(nonfinite), fmt)


def bf16_to_float(bits: int) -> float:
    return lib().mxo_bf16_to_double(int(bits))


def codes_row_bytes(K: int, fmt: int) -> int:
    return K if fmt == E4M3 else K // 2


def quantize(x_bits: np.ndarray, fmt: int, nthreads: int | None = None):
    """x_bits: uint16 bf16 bit patterns [rows, K].  Returns (codes, sf_logical)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, K = x_bits.shape
    codes = np.zeros((rows, codes_row_bytes(K, fmt)), dtype=np.uint8)
    sf = np.zeros((rows, K // 32), dtype=np.uint8)
    rc = lib().mxo_quantize(_ptr(x_bits), rows, K, fmt, _ptr(codes), _ptr(sf),
                            nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle quantize rejected shape %r" % (x_bits.shape,))
    return codes, sf


def dequantize(codes: np.ndarray, sf: np.ndarray, K: int, fmt: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows = codes.shape[0]
    out = np.zeros((rows, K), dtype=np.float64)
    if lib().mxo_dequantize(_ptr(codes), _ptr(sf), rows, K, fmt, _ptr(out)) != 0:
        raise ValueError("oracle dequantize rejected K=%d" % K)
    return out


def sf_tiled_bytes(rows: int, K: int) -> int:
    return lib().mxo_sf_tiled_bytes(rows, K)


def sf_tiled_offset(r: int, kb: int, K: int) -> int:
    return lib().mxo_sf_tiled_offset(r, kb, K)


def sf_to_tiled(sf: np.ndarray, K: int) -> np.ndarray:
    """Logical scales [rows, K/32] -> bytes of the tiled 128x4 atom layout."""
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows = sf.shape[0]
    out = np.zeros(sf_tiled_bytes(rows, K), dtype=np.uint8)
    lib().mxo_sf_to_tiled(_ptr(sf), rows, K, _ptr(out))
    return out


def linear_rows(a_codes, a_sf, a_fmt, rows, K, w_codes, w_sf, bias_bits=None,
                nthreads: int | None = None) -> np.ndarray:
    """fp64 Y[rows, :] = deq(A)[rows] . deq(W)^T (+ bias) for the listed rows."""
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8)
    a_sf = np.ascontiguousarray(a_sf, dtype=np.uint8)
    w_codes = np.ascontiguousarray(w_codes, dtype=np.uint8)
    w_sf = np.ascontiguousarray(w_sf, dtype=np.uint8)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    N = w_codes.shape[0]
    y = np.zeros((rows.shape[0], N), dtype=np.float64)
    bias_p = None
    if bias_bits is not None:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16)
        bias_p = _ptr(bias_bits)
    rc = lib().mxo_linear_rows(_ptr(a_codes), _ptr(a_sf), a_fmt, _ptr(rows), rows.shape[0], K,
                               _ptr(w_codes), _ptr(w_sf), N, bias_p, _ptr(y),
                               nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle linear failed (rc=%d)" % rc)
    return y


def linear(a_codes, a_sf, a_fmt, K, w_codes, w_sf, bias_bits=None, nthreads=None):
    M = a_codes.shape[0]
    return linear_rows(a_codes, a_sf, a_fmt, np.arange(M, dtype=np.int64), K, w_codes, w_sf,
                       bias_bits, nthreads)


def double_to_bf16(v: float) -> int:
    """bf16 bits of v rounded to nearest, ties to even (overflow -> Inf)."""
    return int(lib().mxo_double_to_bf16(float(v)))


def gelu(x: float) -> float:
    """GELU(x) = x * Phi(x) in fp64 (the plain erf form)."""
    return lib().mxo_gelu(float(x))


def round_bf16(y: np.ndarray) -> np.ndarray:
    """fp64 array -> bf16 bit patterns (uint16), same shape."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, dtype=np.uint16)
    lib().mxo_round_bf16(_ptr(y), y.size, _ptr(out))
    return out


def gelu_bf16(y_bits: np.ndarray) -> np.ndarray:
    """bf16 bits y -> bf16 bits of GELU(y) (fp64 GELU, one rounding to bf16)."""
    y_bits = np.ascontiguousarray(y_bits, dtype=np.uint16)
    out = np.empty(y_bits.shape, dtype=np.uint16)
    lib().mxo_gelu_bf16(_ptr(y_bits), y_bits.size, _ptr(out))
    return out


def ffn_hidden_rows(a_codes, a_sf, a_fmt, rows, K, w1_codes, w1_sf, b1_bits, h_fmt,
                    nthreads: int | None = None):
    """The hidden activation between a FFN's two linears, for the listed rows, as a
    bf16 network computes it and as the next linear consumes it:
    y = x . W1^T + b1 (fp64) -> bf16 -> GELU -> bf16 (h) -> MX quantized in h_fmt.
    Returns (h bits [nrows, N], codes, logical scales)."""
    y = linear_rows(a_codes, a_sf, a_fmt, rows, K, w1_codes, w1_sf, b1_bits, nthreads)
    h = gelu_bf16(round_bf16(y))
    codes, sf = quantize(h, h_fmt, nthreads)
    return h, codes, sf


def quantize_static_e4m3(x_bits: np.ndarray, scale: float) -> np.ndarray:
    """Static per-tensor E4M3 codes of bf16 bits x (same shape, uint8): RNE_sat(x / s)
    for the binary32 scale s (a Python float is first rounded to binary32)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    codes = np.empty(x_bits.shape, dtype=np.uint8)
    lib().mxo_quantize_static_e4m3(_ptr(x_bits), x_bits.size, float(scale), _ptr(codes))
    return codes


def linear_rows_scaled(a_codes, a_sf, a_fmt, rows, K, w_codes, w_sf, alpha, bias_bits=None,
                       nthreads: int | None = None) -> np.ndarray:
    """fp64 Y[rows, :] = alpha * deq(A)[rows] . deq(W)^T (+ bias)."""
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8)
    a_sf = np.ascontiguousarray(a_sf, dtype=np.uint8)
    w_codes = np.ascontiguousarray(w_codes, dtype=np.uint8)
    w_sf = np.ascontiguousarray(w_sf, dtype=np.uint8)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    N = w_codes.shape[0]
    y = np.zeros((rows.shape[0], N), dtype=np.float64)
    bias_p = None
    if bias_bits is not None:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16)
        bias_p = _ptr(bias_bits)
    rc = lib().mxo_linear_rows_scaled(_ptr(a_codes), _ptr(a_sf), a_fmt, _ptr(rows), rows.shape[0], K,
                                      _ptr(w_codes), _ptr(w_sf), N, bias_p, float(alpha), _ptr(y),
                                      nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle scaled linear failed (rc=%d)" % rc)
    return y


def quantize_transformed(x_bits: np.ndarray, fmt: int, B: int, mul: np.ndarray | None = None,
                         nthreads: int | None = None):
    """The transform_on quantizer's definition: t = (x * mul) . blockdiag(H_B) / sqrt(B) in
    fp64, then MX quantization of t.  Returns a dict with
      codes, sf  -- the definition's element codes (packed) and logical scales [rows, K/32];
      t          -- the transformed values [rows, K] (fp64);
      code_lo, code_hi -- per element [rows, K], the codes of t -+ delta, delta the error
                    bound of a binary32 evaluation: equal where the code is certain;
      blk_amb    -- per MX block: 0 scale certain, 1 a binary32 evaluation may take a
                    neighbouring scale, 2 it may overflow binary32."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, K = x_bits.shape
    out = {"codes": np.zeros((rows, codes_row_bytes(K, fmt)), dtype=np.uint8),
           "sf": np.zeros((rows, K // 32), dtype=np.uint8),
           "t": np.zeros((rows, K), dtype=np.float64),
           "code_lo": np.zeros((rows, K), dtype=np.uint8),
           "code_hi": np.zeros((rows, K), dtype=np.uint8),
           "blk_amb": np.zeros((rows, K // 32), dtype=np.uint8)}
    mp = None
    if mul is not None:
        mul = np.ascontiguousarray(mul, dtype=np.float32)
        mp = _ptr(mul)
    rc = lib().mxo_quantize_transformed(_ptr(x_bits), rows, K, mp, B, fmt, _ptr(out["codes"]), _ptr(out["sf"]),
                                        _ptr(out["t"]), _ptr(out["code_lo"]), _ptr(out["code_hi"]),
                                        _ptr(out["blk_amb"]), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle transform failed (rc=%d)" % rc)
    return out


def linear_lowrank_rows(a_codes, a_sf, a_fmt, rows, K, r_codes, r_sf, x_bits, l1t_bits, l2t_bits, bias_bits=None,
                        nthreads: int | None = None) -> np.ndarray:
    """fp64 y[rows] = deq(A)[rows] . deq(R)^T + bf16(x[rows] . l1t^T) . l2t^T (+ bias)."""
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8)
    a_sf = np.ascontiguousarray(a_sf, dtype=np.uint8)
    r_codes = np.ascontiguousarray(r_codes, dtype=np.uint8)
    r_sf = np.ascontiguousarray(r_sf, dtype=np.uint8)
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    l1t_bits = np.ascontiguousarray(l1t_bits, dtype=np.uint16)
    l2t_bits = np.ascontiguousarray(l2t_bits, dtype=np.uint16)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    N, r = l2t_bits.shape
    y = np.zeros((rows.shape[0], N), dtype=np.float64)
    bias_p = None
    if bias_bits is not None:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16)
        bias_p = _ptr(bias_bits)
    rc = lib().mxo_linear_lowrank_rows(_ptr(a_codes), _ptr(a_sf), a_fmt, _ptr(rows), rows.shape[0], K,
                                       _ptr(r_codes), _ptr(r_sf), N, _ptr(x_bits), _ptr(l1t_bits), _ptr(l2t_bits),
                                       r, bias_p, _ptr(y), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle low-rank linear failed (rc=%d)" % rc)
    return y


# ---- the bf16 GEMM and the policy's calibration / load-time arithmetic -----------------
#
# Plain numpy in fp64 on the exact values of the bf16 / fp32 inputs: the standard bf16
# GEMM of the blog's "Kernel note" (the quantize-dequantize emulation's GEMM), SmoothQuant's
# per-channel scales and the whole-block SQNR ("Mixed-Precision selection",
# "Calibration-driven block selection"), and the SVDQuant split of a weight ("Results").

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact values of bf16 bit patterns."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def gemm_bf16(a_bits: np.ndarray, b_bits: np.ndarray, bias_bits: np.ndarray | None = None) -> np.ndarray:
    """fp64 y = a . b^T (+ bias) for bf16 a [M, K], b [N, K]."""
    y = bf16_bits_to_f64(a_bits) @ bf16_bits_to_f64(b_bits).T
    if bias_bits is not None:
        y = y + bf16_bits_to_f64(bias_bits)[None, :]
    return y


def channel_absmax(x_bits: np.ndarray) -> np.ndarray:
    """max over rows of |x[:, k]| (fp64; exact, the values are bf16)."""
    return np.abs(bf16_bits_to_f64(x_bits)).max(axis=0)


def smooth_scales(amax_x: np.ndarray, amax_w: np.ndarray, alpha: float) -> np.ndarray:
    """SmoothQuant's s_k = max(amax_x_k, 1e-5)^alpha / max(amax_w_k, 1e-5)^(1 - alpha) in fp64
    (the 1e-5 floor as the binary32 value the library compares with)."""
    floor = float(np.float32(1e-5))
    ax = np.maximum(np.asarray(amax_x, dtype=np.float64), floor)
    aw = np.maximum(np.asarray(amax_w, dtype=np.float64), floor)
    return ax ** float(alpha) / aw ** (1.0 - float(alpha))


def sqnr(ref_bits: list, test_bits: list):
    """(sum ref^2, sum (ref - test)^2, 10 log10 of their ratio) over pairs of bf16 tensors."""
    num = sum(float(np.sum(bf16_bits_to_f64(r) ** 2)) for r in ref_bits)
    den = sum(float(np.sum((bf16_bits_to_f64(r) - bf16_bits_to_f64(t)) ** 2)) for r, t in zip(ref_bits, test_bits))
    with np.errstate(divide="ignore"):
        db = 10.0 * np.log10(num / den) if den > 0 else float("inf")
    return num, den, db


def lowrank_split(U: np.ndarray, S: np.ndarray, Vh: np.ndarray, w_bits: np.ndarray, rank: int):
    """The SVDQuant split from singular triplets (fp32 U, S, Vh): l2t = bf16(U_r sqrt(S_r)),
    l1t = bf16(sqrt(S_r) Vh_r) and the residual bf16(W - l2t . l1t), each product and sum in
    fp64 and rounded once to bf16.  Returns bf16 bits (l1t, l2t, residual)."""
    rs = np.sqrt(np.asarray(S[:rank], dtype=np.float64))
    l2t = round_bf16(np.asarray(U[:, :rank], dtype=np.float64) * rs[None, :])
    l1t = round_bf16(rs[:, None] * np.asarray(Vh[:rank], dtype=np.float64))
    resid = round_bf16(bf16_bits_to_f64(w_bits) - bf16_bits_to_f64(l2t) @ bf16_bits_to_f64(l1t))
    return l1t, l2t, resid
