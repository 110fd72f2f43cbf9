"""Tensor-level entry points: the same calls as the C ABI (include/mxq.h), taking torch
tensors for device memory and the current torch stream.  Nothing here computes:
each function checks dtypes and devices, allocates outputs with torch, and calls the
library."""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import FMT_E2M1, FMT_E4M3, MODE_NATIVE, MODE_QDQ, WDesc, check

_FMTS = {"e2m1": FMT_E2M1, "e4m3": FMT_E4M3, FMT_E2M1: FMT_E2M1, FMT_E4M3: FMT_E4M3}
_MODES = {"native": MODE_NATIVE, "qdq": MODE_QDQ, MODE_NATIVE: MODE_NATIVE, MODE_QDQ: MODE_QDQ}


def _fmt(f) -> int:
    return _FMTS[f]


def _mode(m) -> int:
    return _MODES[m]


def _stream(stream=None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _p(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _cuda_bf16(t: torch.Tensor, name: str) -> None:
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
        raise ValueError("%s must be a contiguous bf16 CUDA tensor" % name)


def codes_bytes(rows: int, K: int, fmt="e2m1") -> int:
    return int(_lib.lib().mxq_codes_bytes(rows, K, _fmt(fmt)))


def sf_bytes(rows: int, K: int) -> int:
    return int(_lib.lib().mxq_sf_bytes(rows, K))


def workspace_bytes(M: int, N: int, K: int, fmt="e2m1", mode="native") -> int:
    return int(_lib.lib().mxq_workspace_bytes(M, N, K, _fmt(fmt), _mode(mode)))


@dataclass
class QWeight:
    """MXFP4 weight of one linear layer: codes [N, K/2], tiled scales, optional bias."""
    codes: torch.Tensor
    sf: torch.Tensor
    N: int
    K: int
    bias: torch.Tensor | None = None

    def desc(self) -> WDesc:
        return WDesc(self.codes.data_ptr(), self.sf.data_ptr(),
                     0 if self.bias is None else self.bias.data_ptr(), self.N, self.K)


def quantize_act(x: torch.Tensor, fmt="e2m1", codes=None, sf=None, stream=None):
    """x [M, K] bf16 -> (codes, tiled scales) in format fmt."""
    _cuda_bf16(x, "x")
    M, K = x.shape
    f = _fmt(fmt)
    if codes is None:
        codes = torch.empty(max(1, codes_bytes(M, K, f)), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(max(1, sf_bytes(M, K)), dtype=torch.uint8, device=x.device)
    check(_lib.lib().mxq_quantize_act(_p(x), M, K, f, _p(codes), _p(sf), _stream(stream)), "mxq_quantize_act")
    return codes, sf


def quantize_weight(w: torch.Tensor, bias: torch.Tensor | None = None, stream=None) -> QWeight:
    """w [N, K] bf16 -> QWeight (MXFP4 codes [N, K/2] + tiled scales)."""
    _cuda_bf16(w, "w")
    N, K = w.shape
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    sf = torch.empty(max(1, sf_bytes(N, K)), dtype=torch.uint8, device=w.device)
    check(_lib.lib().mxq_quantize_weight(_p(w), N, K, _p(codes), _p(sf), _stream(stream)), "mxq_quantize_weight")
    if bias is not None:
        _cuda_bf16(bias, "bias")
    return QWeight(codes, sf, N, K, bias)


def dequantize(codes: torch.Tensor, sf: torch.Tensor, rows: int, K: int, fmt="e2m1", out=None, stream=None):
    if out is None:
        out = torch.empty((rows, K), dtype=torch.bfloat16, device=codes.device)
    check(_lib.lib().mxq_dequantize(_p(codes), _p(sf), rows, K, _fmt(fmt), _p(out), _stream(stream)),
          "mxq_dequantize")
    return out


def gemm(a_codes, a_sf, fmt, M: int, K: int, w: QWeight, out=None, stream=None):
    """GEMM on an already-quantized activation: y [M, N] bf16."""
    if out is None:
        out = torch.empty((M, w.N), dtype=torch.bfloat16, device=a_codes.device)
    check(_lib.lib().mxq_gemm(_p(a_codes), _p(a_sf), _fmt(fmt), M, K, _p(w.codes), _p(w.sf), w.N, _p(w.bias),
                              _p(out), _stream(stream)), "mxq_gemm")
    return out


def gemm_bf16(a: torch.Tensor, b: torch.Tensor, bias: torch.Tensor | None = None, out=None, stream=None):
    """y [M, N] = a [M, K] . b [N, K]^T (+ bias) in bf16 with fp32 accumulation, on the
    library's tcgen05 kernel (kind::f16)."""
    _cuda_bf16(a, "a")
    _cuda_bf16(b, "b")
    if bias is not None:
        _cuda_bf16(bias, "bias")
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a is [%d, %d] but b is [%d, %d]" % (M, K, N, b.shape[1]))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    check(_lib.lib().mxq_gemm_bf16(_p(a), M, K, _p(b), N, _p(bias), _p(out), _stream(stream)), "mxq_gemm_bf16")
    return out


def gemm_bf16_quant_a(a: torch.Tensor, b: torch.Tensor, fmt="e2m1", bias: torch.Tensor | None = None, out=None,
                      codes=None, sf=None, stream=None):
    """(y, codes, sf): y [M, N] = a [M, K] . b [N, K]^T (+ bias) in bf16 (N <= 128) by the
    bf16 kernel, which also writes a's MX quantization in format fmt (codes, tiled scales:
    the bits quantize_act writes) from the same read of a."""
    _cuda_bf16(a, "a")
    _cuda_bf16(b, "b")
    if bias is not None:
        _cuda_bf16(bias, "bias")
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a is [%d, %d] but b is [%d, %d]" % (M, K, N, b.shape[1]))
    f = _fmt(fmt)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    if codes is None:
        codes = torch.empty(max(1, codes_bytes(M, K, f)), dtype=torch.uint8, device=a.device)
    if sf is None:
        sf = torch.empty(max(1, sf_bytes(M, K)), dtype=torch.uint8, device=a.device)
    check(_lib.lib().mxq_gemm_bf16_quant_a(_p(a), M, K, _p(b), N, _p(bias), _p(out), f, _p(codes), _p(sf),
                                           _stream(stream)), "mxq_gemm_bf16_quant_a")
    return out, codes, sf


def linear(x: torch.Tensor, w: QWeight, fmt="e2m1", mode="native", workspace=None, out=None, stream=None):
    """y = x . deq(w)^T + bias with x quantized on the fly to fmt (E2M1 = W4A4, E4M3 = W4A8)."""
    _cuda_bf16(x, "x")
    M, K = x.shape
    f, m = _fmt(fmt), _mode(mode)
    need = workspace_bytes(M, w.N, K, f, m)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((M, w.N), dtype=torch.bfloat16, device=x.device)
    check(_lib.lib().mxq_linear(_p(x), M, K, _p(w.codes), _p(w.sf), w.N, _p(w.bias), f, m, _p(workspace),
                                workspace.numel() * workspace.element_size(), _p(out), _stream(stream)),
          "mxq_linear")
    return out


def linear_noalloc(x: torch.Tensor, w: QWeight, fmt="e2m1", out=None, stream=None):
    """As linear() in native mode, but the library takes its scratch from a fixed static
    device buffer instead of a workspace (for callers that cannot allocate where they run
    a layer; see mxq_linear_noalloc in include/mxq.h for the size limit and the rule that
    calls must not overlap on the GPU).  Only the output is allocated here, and only when
    `out` is not given."""
    _cuda_bf16(x, "x")
    M, K = x.shape
    if out is None:
        out = torch.empty((M, w.N), dtype=torch.bfloat16, device=x.device)
    check(_lib.lib().mxq_linear_noalloc(_p(x), M, K, _p(w.codes), _p(w.sf), w.N, _p(w.bias), _fmt(fmt), _p(out),
                                        _stream(stream)), "mxq_linear_noalloc")
    return out


def gemm_gelu_quant(a_codes, a_sf, fmt, M: int, K: int, w: QWeight, out_fmt="e2m1", codes=None, sf=None,
                    h=None, stream=None):
    """GEMM whose epilogue applies bias + GELU and writes the result MX-quantized in
    out_fmt (the next layer's input): returns (codes, tiled scales).  Pass a bf16 [M, N]
    tensor as h to also receive the GELU output."""
    f = _fmt(out_fmt)
    if codes is None:
        codes = torch.empty(max(1, codes_bytes(M, w.N, f)), dtype=torch.uint8, device=a_codes.device)
    if sf is None:
        sf = torch.empty(max(1, sf_bytes(M, w.N)), dtype=torch.uint8, device=a_codes.device)
    if h is not None:
        _cuda_bf16(h, "h")
    check(_lib.lib().mxq_gemm_gelu_quant(_p(a_codes), _p(a_sf), _fmt(fmt), M, K, _p(w.codes), _p(w.sf), w.N,
                                         _p(w.bias), f, _p(codes), _p(sf), _p(h), _stream(stream)),
          "mxq_gemm_gelu_quant")
    return codes, sf


def gemm_quant(a_codes, a_sf, fmt, M: int, K: int, w: QWeight, act="none", out_fmt="e2m1", codes=None, sf=None,
               h=None, stream=None):
    """GEMM whose epilogue writes its output MX-quantized in out_fmt, after GELU when
    act is "gelu" (mxq_gemm_gelu_quant) or as it is when act is "none": returns (codes,
    tiled scales).  Pass a bf16 [M, N] tensor as h to also receive the quantizer's input."""
    acts = {"none": _lib.ACT_NONE, "gelu": _lib.ACT_GELU}
    if act not in acts:
        raise ValueError("act must be 'none' or 'gelu', got %r" % (act,))
    f = _fmt(out_fmt)
    if codes is None:
        codes = torch.empty(max(1, codes_bytes(M, w.N, f)), dtype=torch.uint8, device=a_codes.device)
    if sf is None:
        sf = torch.empty(max(1, sf_bytes(M, w.N)), dtype=torch.uint8, device=a_codes.device)
    if h is not None:
        _cuda_bf16(h, "h")
    check(_lib.lib().mxq_gemm_quant(_p(a_codes), _p(a_sf), _fmt(fmt), M, K, _p(w.codes), _p(w.sf), w.N, _p(w.bias),
                                    acts[act], f, _p(codes), _p(sf), _p(h), _stream(stream)), "mxq_gemm_quant")
    return codes, sf


def gelu_bf16(x: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """GELU of bf16 values as the quantizing epilogue applies it (exact, rounded once to bf16)."""
    _cuda_bf16(x, "x")
    if out is None:
        out = torch.empty_like(x)
    _cuda_bf16(out, "out")
    if out.numel() != x.numel():
        raise ValueError("out must have as many elements as x")
    check(_lib.lib().mxq_gelu_bf16(_p(x), x.numel(), _p(out), _stream(stream)), "mxq_gelu_bf16")
    return out


def ffn_workspace_bytes(M: int, K: int, H: int, up_fmt="e2m1", down_fmt="e2m1") -> int:
    return int(_lib.lib().mxq_ffn_workspace_bytes(M, K, H, _fmt(up_fmt), _fmt(down_fmt)))


def ffn(x: torch.Tensor, up: QWeight, down: QWeight, up_fmt="e2m1", down_fmt="e2m1", workspace=None, out=None,
        stream=None):
    """y = quant(GELU(x . up^T + b_up)) . down^T + b_down with the hidden activation kept
    MX-quantized between the two linears."""
    _cuda_bf16(x, "x")
    M, K = x.shape
    if workspace is None:
        workspace = torch.empty(ffn_workspace_bytes(M, K, up.N, up_fmt, down_fmt), dtype=torch.uint8,
                                device=x.device)
    if out is None:
        out = torch.empty((M, down.N), dtype=torch.bfloat16, device=x.device)
    du, dd = up.desc(), down.desc()
    check(_lib.lib().mxq_ffn(_p(x), M, K, ctypes.byref(du), ctypes.byref(dd), _fmt(up_fmt), _fmt(down_fmt),
                             _p(workspace), workspace.numel(), _p(out), _stream(stream)), "mxq_ffn")
    return out


def absmax(x: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """max |x| over a bf16 tensor, as a one-element fp32 CUDA tensor (calibration)."""
    _cuda_bf16(x, "x")
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    check(_lib.lib().mxq_absmax(_p(x), x.numel(), _p(out), _stream(stream)), "mxq_absmax")
    return out


def quantize_act_static(x: torch.Tensor, scale: float, codes=None, sf=None, stream=None):
    """x [M, K] bf16 -> static per-tensor E4M3 codes [M, K] and tiled scales (all 127)."""
    _cuda_bf16(x, "x")
    M, K = x.shape
    if codes is None:
        codes = torch.empty(max(1, codes_bytes(M, K, FMT_E4M3)), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(max(1, sf_bytes(M, K)), dtype=torch.uint8, device=x.device)
    check(_lib.lib().mxq_quantize_act_static(_p(x), M, K, float(scale), _p(codes), _p(sf), _stream(stream)),
          "mxq_quantize_act_static")
    return codes, sf


def linear_static(x: torch.Tensor, w: QWeight, act_scale: float, workspace=None, out=None, stream=None):
    """y = act_scale * (static E4M3 codes of x) . deq(w)^T + bias (W4A8, static activations)."""
    _cuda_bf16(x, "x")
    M, K = x.shape
    if workspace is None:
        workspace = torch.empty(workspace_bytes(M, w.N, K, FMT_E4M3, MODE_NATIVE), dtype=torch.uint8,
                                device=x.device)
    if out is None:
        out = torch.empty((M, w.N), dtype=torch.bfloat16, device=x.device)
    check(_lib.lib().mxq_linear_static(_p(x), M, K, _p(w.codes), _p(w.sf), w.N, _p(w.bias), float(act_scale),
                                       _p(workspace), workspace.numel(), _p(out), _stream(stream)),
          "mxq_linear_static")
    return out


def _f32_or_none(t, name):
    if t is None:
        return None
    if not (t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()):
        raise ValueError("%s must be a contiguous float32 CUDA tensor" % name)
    return t


def quantize_act_transformed(x: torch.Tensor, fmt="e2m1", block=32, mul=None, codes=None, sf=None, stream=None):
    """x [M, K] bf16 -> MX codes and tiled scales of (x * mul) rotated by the block Hadamard."""
    _cuda_bf16(x, "x")
    M, K = x.shape
    f = _fmt(fmt)
    mul = _f32_or_none(mul, "mul")
    if codes is None:
        codes = torch.empty(max(1, codes_bytes(M, K, f)), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(max(1, sf_bytes(M, K)), dtype=torch.uint8, device=x.device)
    check(_lib.lib().mxq_quantize_act_transformed(_p(x), M, K, f, _p(mul), int(block), _p(codes), _p(sf),
                                                  _stream(stream)), "mxq_quantize_act_transformed")
    return codes, sf


def quantize_weight_transformed(w: torch.Tensor, bias=None, block=32, mul=None, stream=None) -> QWeight:
    """w [N, K] bf16 -> QWeight of (w * mul) rotated by the block Hadamard (mul = s)."""
    _cuda_bf16(w, "w")
    N, K = w.shape
    mul = _f32_or_none(mul, "mul")
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    sf = torch.empty(max(1, sf_bytes(N, K)), dtype=torch.uint8, device=w.device)
    check(_lib.lib().mxq_quantize_weight_transformed(_p(w), N, K, _p(mul), int(block), _p(codes), _p(sf),
                                                     _stream(stream)), "mxq_quantize_weight_transformed")
    if bias is not None:
        _cuda_bf16(bias, "bias")
    return QWeight(codes, sf, N, K, bias)


def linear_transformed(x: torch.Tensor, w: QWeight, fmt="e2m1", block=32, act_mul=None, workspace=None, out=None,
                       stream=None):
    """The linear on the transformed path (w from quantize_weight_transformed, same block)."""
    _cuda_bf16(x, "x")
    M, K = x.shape
    f = _fmt(fmt)
    act_mul = _f32_or_none(act_mul, "act_mul")
    if workspace is None:
        workspace = torch.empty(workspace_bytes(M, w.N, K, f, MODE_NATIVE), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((M, w.N), dtype=torch.bfloat16, device=x.device)
    check(_lib.lib().mxq_linear_transformed(_p(x), M, K, _p(w.codes), _p(w.sf), w.N, _p(w.bias), f, _p(act_mul),
                                            int(block), _p(workspace), workspace.numel(), _p(out), _stream(stream)),
          "mxq_linear_transformed")
    return out


def lowrank_split(w: torch.Tensor, U: torch.Tensor, S: torch.Tensor, Vh: torch.Tensor, rank: int, stream=None):
    """The SVDQuant split of w [N, K] bf16 from its singular triplets (U [N, >= rank],
    S [>= rank], Vh [>= rank, K], fp32 CUDA tensors, the first `rank` used), in the library:
    l2t = bf16(U sqrt(S)) [N, rank], l1t = bf16(sqrt(S) Vh) [rank, K] and the residual
    bf16(w - l2t . l1t) [N, K].  Returns (l1t, l2t, residual)."""
    _cuda_bf16(w, "w")
    N, K = w.shape
    for t, name in ((U, "U"), (S, "S"), (Vh, "Vh")):
        if not (t.is_cuda and t.dtype == torch.float32 and t.stride(-1) == 1):
            raise ValueError("%s must be a float32 CUDA tensor with unit inner stride" % name)
    if U.shape[0] != N or Vh.shape[1] != K or min(U.shape[1], S.shape[0], Vh.shape[0]) < rank:
        raise ValueError("factors of shapes %s, %s, %s do not fit w [%d, %d] at rank %d" % (
            tuple(U.shape), tuple(S.shape), tuple(Vh.shape), N, K, rank))
    l2t = torch.empty((N, rank), dtype=torch.bfloat16, device=w.device)
    l1t = torch.empty((rank, K), dtype=torch.bfloat16, device=w.device)
    resid = torch.empty((N, K), dtype=torch.bfloat16, device=w.device)
    check(_lib.lib().mxq_lowrank_split(_p(U), U.stride(0), _p(S), _p(Vh), Vh.stride(0), _p(w), N, K, rank, _p(l2t),
                                       _p(l1t), _p(resid), _stream(stream)), "mxq_lowrank_split")
    return l1t, l2t, resid


def svd_split(w: torch.Tensor, rank: int, stream=None):
    """Offline weight preparation of the SVDQuant branch (load time, not the layer's path):
    the singular value decomposition of w in fp32 is a library factorization (torch's),
    the split into l2t = U_r sqrt(S_r), l1t = sqrt(S_r) V_r^T and the bf16 residual
    w - l2t . l1t runs in this library (lowrank_split).  Returns (l1t, l2t, residual)."""
    _cuda_bf16(w, "w")
    U, S, Vh = torch.linalg.svd(w.float(), full_matrices=False)
    return lowrank_split(w, U.contiguous(), S.contiguous(), Vh.contiguous(), rank, stream=stream)


def channel_absmax(x: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """max over rows of |x[:, k]| for a bf16 [rows, K] tensor, as K float32 values."""
    _cuda_bf16(x, "x")
    rows, K = x.shape
    if out is None:
        out = torch.empty(K, dtype=torch.float32, device=x.device)
    check(_lib.lib().mxq_channel_absmax(_p(x), rows, K, _p(out), _stream(stream)), "mxq_channel_absmax")
    return out


def smooth_scales(amax_x: torch.Tensor, amax_w: torch.Tensor, alpha: float = 0.5, with_inverse: bool = False,
                  stream=None):
    """SmoothQuant's s_k = max(amax_x_k, 1e-5)^alpha / max(amax_w_k, 1e-5)^(1 - alpha);
    with_inverse: also 1 / s_k (the activation's multiplier), returned as (s, 1/s)."""
    amax_x = _f32_or_none(amax_x, "amax_x")
    amax_w = _f32_or_none(amax_w, "amax_w")
    K = amax_x.numel()
    if amax_w.numel() != K:
        raise ValueError("channel counts differ: %d vs %d" % (K, amax_w.numel()))
    s = torch.empty(K, dtype=torch.float32, device=amax_x.device)
    inv = torch.empty(K, dtype=torch.float32, device=amax_x.device) if with_inverse else None
    check(_lib.lib().mxq_smooth_scales(_p(amax_x), _p(amax_w), K, float(alpha), _p(s), _p(inv), _stream(stream)),
          "mxq_smooth_scales")
    return (s, inv) if with_inverse else s


def sqnr(refs, tests, out=None, stream=None) -> torch.Tensor:
    """SQNR over pairs of bf16 tensors: a float64 CUDA tensor [sum ref^2, sum (ref - test)^2,
    dB]."""
    refs, tests = list(refs), list(tests)
    if len(refs) != len(tests) or not refs:
        raise ValueError("need as many test tensors as reference tensors, at least one")
    for r, t in zip(refs, tests):
        _cuda_bf16(r, "ref")
        _cuda_bf16(t, "test")
        if r.numel() != t.numel():
            raise ValueError("a reference and its test tensor differ in size")
    if out is None:
        out = torch.empty(3, dtype=torch.float64, device=refs[0].device)
    n = len(refs)
    rp = (ctypes.c_void_p * n)(*[r.data_ptr() for r in refs])
    tp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in tests])
    ns = (ctypes.c_int64 * n)(*[r.numel() for r in refs])
    check(_lib.lib().mxq_sqnr(rp, tp, ns, n, _p(out), _stream(stream)), "mxq_sqnr")
    return out


def lowrank_workspace_bytes(M: int, N: int, K: int, fmt="e2m1", rank=64) -> int:
    return int(_lib.lib().mxq_lowrank_workspace_bytes(M, N, K, _fmt(fmt), int(rank)))


def linear_lowrank(x: torch.Tensor, residual: QWeight, l1t: torch.Tensor, l2t: torch.Tensor, fmt="e2m1",
                   workspace=None, out=None, stream=None):
    """y = deq(xq) . deq(Rq)^T + bf16(x . l1t^T) . l2t^T + bias (SVDQuant branch in the
    same accumulator)."""
    _cuda_bf16(x, "x")
    _cuda_bf16(l1t, "l1t")
    _cuda_bf16(l2t, "l2t")
    M, K = x.shape
    rank = l1t.shape[0]
    f = _fmt(fmt)
    if workspace is None:
        workspace = torch.empty(lowrank_workspace_bytes(M, residual.N, K, f, rank), dtype=torch.uint8,
                                device=x.device)
    if out is None:
        out = torch.empty((M, residual.N), dtype=torch.bfloat16, device=x.device)
    check(_lib.lib().mxq_linear_lowrank(_p(x), M, K, _p(residual.codes), _p(residual.sf), residual.N,
                                        _p(residual.bias), f, _p(l1t), _p(l2t), rank, _p(workspace),
                                        workspace.numel(), _p(out), _stream(stream)), "mxq_linear_lowrank")
    return out


def block_workspace_bytes(weights, rows, w4a8_bits: int, mode="native", minimum: bool = False) -> int:
    """Workspace of dit_block_linears: by default the size that lets the quantizers overlap
    the GEMMs (native mode); minimum=True gives the least it accepts."""
    descs = (WDesc * 8)(*[w.desc() for w in weights])
    ms = (ctypes.c_int64 * 8)(*rows)
    fn = _lib.lib().mxq_block_workspace_min_bytes if minimum else _lib.lib().mxq_block_workspace_bytes
    return int(fn(descs, ms, w4a8_bits, _mode(mode)))


def dit_block_linears(weights, xs, w4a8_bits: int, mode="native", workspace=None, outs=None, stream=None):
    """The eight linears of one DiT block (QKV, attn-out, cross-Q/K/V/out, FFN-up,
    FFN-down); bit i of w4a8_bits selects W4A8 for linear i."""
    assert len(weights) == 8 and len(xs) == 8
    rows = [int(x.shape[0]) for x in xs]
    for x in xs:
        _cuda_bf16(x, "block input")
    if outs is None:
        outs = [torch.empty((r, w.N), dtype=torch.bfloat16, device=xs[0].device) for r, w in zip(rows, weights)]
    need = block_workspace_bytes(weights, rows, w4a8_bits, mode)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=xs[0].device)
    descs = (WDesc * 8)(*[w.desc() for w in weights])
    xin = (ctypes.c_void_p * 8)(*[x.data_ptr() for x in xs])
    ms = (ctypes.c_int64 * 8)(*rows)
    yout = (ctypes.c_void_p * 8)(*[y.data_ptr() for y in outs])
    check(_lib.lib().mxq_dit_block_linears(descs, xin, ms, yout, w4a8_bits, _mode(mode), _p(workspace),
                                           workspace.numel(), _stream(stream)), "mxq_dit_block_linears")
    return outs


def sf_to_logical(sf: torch.Tensor, rows: int, K: int, stream=None) -> torch.Tensor:
    out = torch.empty((rows, K // 32), dtype=torch.uint8, device=sf.device)
    check(_lib.lib().mxq_sf_to_logical(_p(sf), rows, K, _p(out), _stream(stream)), "mxq_sf_to_logical")
    return out


def poll_status(stream=None) -> int:
    """Synchronizes the stream and returns the device status word (0 = fine)."""
    return int(_lib.lib().mxq_poll_status(_stream(stream)))


def set_debug(flags: int) -> None:
    _lib.lib().mxq_set_debug(flags)


def last_path() -> str:
    return _lib.last_path()
