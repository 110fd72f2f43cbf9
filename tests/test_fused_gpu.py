"""The GEMM whose epilogue emits the next layer's MX-quantized input (bias -> bf16 ->
GELU -> bf16 -> MX block quantization), and the FFN built on it.

The oracle computes the same chain from the same bf16 inputs in fp64
(oracle.ffn_hidden_rows).  The GPU accumulates in fp32 in another order, so its bf16
rounding of the linear output differs from the oracle's on a small fraction of
elements; the checks are therefore:
  * the GELU itself is exact: on every bf16 value (mxq_gelu_bf16, the epilogue's table),
    and inside the epilogue, where h is bit for bit the oracle's bf16 GELU of the GPU's own
    pre-activation (the no-activation epilogue's h);
  * h (the GELU output, returned for checking) equals the oracle's on >= 99 % of the
    elements and stays within the GEMM tolerance everywhere;
  * codes and scales are bit-exact against the oracle's chain on every block whose 32 h
    values agree with the oracle's;
  * on every block, padding of the tiled layout included, codes and scales are bit-exact
    against the oracle's quantizer applied to the h the GPU produced (the epilogue's
    quantization step checked on its own input);
  * the FFN output is within the GEMM tolerance of the oracle's FFN chain.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _mx

pytestmark = pytest.mark.gpu


def _ops():
    from fp8_mixed_precision_mxq_b200 import ops
    return ops


def _bits_np(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_hidden(x, w1, b1, a_fmt, h_fmt):
    """Oracle h (bf16 bits), codes and logical scales for all rows of x."""
    xc, xs, _ = _mx.oracle_quantize(x, a_fmt)
    wc, ws, _ = _mx.oracle_quantize(w1, "e2m1")
    rows = np.arange(x.shape[0], dtype=np.int64)
    bb = _mx.bits(b1) if b1 is not None else None
    return oracle.ffn_hidden_rows(xc, xs, _mx.FMT[a_fmt], rows, x.shape[1], wc, ws, bb, _mx.FMT[h_fmt])


def check_hidden(M, N, h_gpu, codes, sf, h_ref, c_ref, s_ref, h_fmt, what):
    hg = _bits_np(h_gpu).reshape(M, N)
    eq = hg == h_ref
    assert eq.mean() >= 0.99, "%s: only %.4f of h equals the oracle's" % (what, eq.mean())
    _mx.assert_gemm_close(_mx.bf16_to_f64(h_gpu),
                          torch.from_numpy(h_ref.view(np.int16)).view(torch.bfloat16).double().numpy(), what + " h")
    # bit-exact against the oracle's chain on every block whose h agrees with the oracle's
    KB = N // 32
    blk_eq = eq.reshape(M, KB, 32).all(axis=2)
    sf_np = sf.cpu().numpy()
    s_gpu = _mx.tiled_to_logical(sf_np, M, N)
    assert np.array_equal(s_gpu[blk_eq], s_ref[blk_eq]), what + ": scales differ on agreeing blocks"
    per = 32 if h_fmt == "e4m3" else 16
    c_np = codes.cpu().numpy()
    c_gpu = c_np[: M * KB * per].reshape(M, KB, per)
    assert np.array_equal(c_gpu[blk_eq], c_ref.reshape(M, KB, per)[blk_eq]), what + ": codes differ on agreeing blocks"
    # every block, and the tiled layout's padding: the oracle's quantizer on the GPU's h
    c_o, s_o = oracle.quantize(hg, _mx.FMT[h_fmt])
    assert np.array_equal(c_np[: c_o.size], c_o.reshape(-1)), what + ": codes differ from the oracle's quantize(h)"
    assert np.array_equal(sf_np, oracle.sf_to_tiled(s_o, N)), what + ": tiled scales differ from the oracle's"


CASES = [  # M, N, K, a_fmt, h_fmt
    (128, 256, 512, "e2m1", "e2m1"),
    (128, 256, 512, "e2m1", "e4m3"),
    (300, 544, 512, "e2m1", "e2m1"),   # ragged M (CTA pairs) and N (last tile 32 columns)
    (300, 544, 512, "e4m3", "e4m3"),   # W4A8 GEMM feeding an E4M3 hidden activation
    (1, 32, 128, "e2m1", "e2m1"),      # one row, one output block (k-blocks padded to 4)
    (513, 1056, 1024, "e4m3", "e2m1"),
]


@pytest.mark.parametrize("M,N,K,a_fmt,h_fmt", CASES)
def test_gemm_gelu_quant_against_oracle(M, N, K, a_fmt, h_fmt):
    ops = _ops()
    x = synth.activation(M, K, "normal", seed=M + N, device="cuda", outlier_frac=0.02, outlier_scale=30.0)
    w = synth.weight(N, K, seed=N + K, device="cuda")
    b = synth.bias(N, seed=N, device="cuda")
    qw = ops.quantize_weight(w, bias=b)
    xc, xs = ops.quantize_act(x, a_fmt)
    h = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    codes, sf = ops.gemm_gelu_quant(xc, xs, a_fmt, M, K, qw, out_fmt=h_fmt, h=h)
    assert ops.poll_status() == 0
    assert "+gelu->" + h_fmt in ops.last_path()
    h_ref, c_ref, s_ref = oracle_hidden(x, w, b, a_fmt, h_fmt)
    check_hidden(M, N, h, codes, sf, h_ref, c_ref, s_ref, h_fmt, "M=%d N=%d %s->%s" % (M, N, a_fmt, h_fmt))
    # without the h output the codes and scales are the same
    codes2, sf2 = ops.gemm_gelu_quant(xc, xs, a_fmt, M, K, qw, out_fmt=h_fmt)
    assert torch.equal(codes2, codes) and torch.equal(sf2, sf)


@pytest.mark.parametrize("M,N,K,a_fmt,h_fmt", CASES)
def test_gemm_quant_identity_is_quantize_of_gemm(M, N, K, a_fmt, h_fmt):
    """With no activation the quantizing epilogue's h is, bit for bit, the plain
    GEMM's bf16 output, and its codes and tiled scales (padding included) are the oracle's
    quantization of that output, bit for bit; the GELU choice equals mxq_gemm_gelu_quant."""
    ops = _ops()
    x = synth.activation(M, K, "normal", seed=M + 7 * N, device="cuda", outlier_frac=0.02, outlier_scale=30.0)
    w = synth.weight(N, K, seed=N + 3 * K, device="cuda")
    b = synth.bias(N, seed=N + 1, device="cuda")
    qw = ops.quantize_weight(w, bias=b)
    xc, xs = ops.quantize_act(x, a_fmt)
    y = ops.gemm(xc, xs, a_fmt, M, K, qw)
    h = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    codes, sf = ops.gemm_quant(xc, xs, a_fmt, M, K, qw, act="none", out_fmt=h_fmt, h=h)
    assert ops.poll_status() == 0
    assert "+quant->" + h_fmt in ops.last_path()
    assert torch.equal(h, y)
    # the epilogue's quantization of its own output, checked by the oracle's quantizer
    c_o, s_o = oracle.quantize(_bits_np(y).reshape(M, N), _mx.FMT[h_fmt])
    assert np.array_equal(codes.cpu().numpy()[: c_o.size], c_o.reshape(-1))
    assert np.array_equal(sf.cpu().numpy(), oracle.sf_to_tiled(s_o, N))
    # and the product is the oracle's linear within the GEMM tolerance
    xo, xso, _ = _mx.oracle_quantize(x, a_fmt)
    wo, wso, _ = _mx.oracle_quantize(w, "e2m1")
    ref = oracle.linear_rows(xo, xso, _mx.FMT[a_fmt], np.arange(M), K, wo, wso, _mx.bits(b))
    _mx.assert_gemm_close(_mx.bf16_to_f64(h), ref, "identity-quant epilogue M=%d N=%d" % (M, N))
    hg = torch.empty_like(h)
    cg, sg = ops.gemm_quant(xc, xs, a_fmt, M, K, qw, act="gelu", out_fmt=h_fmt, h=hg)
    cg2, sg2 = ops.gemm_gelu_quant(xc, xs, a_fmt, M, K, qw, out_fmt=h_fmt)
    assert torch.equal(cg, cg2) and torch.equal(sg, sg2)
    # the GELU step inside the epilogue: exactly the oracle's bf16 GELU of the same y
    assert np.array_equal(_bits_np(hg).reshape(M, N), oracle.gelu_bf16(_bits_np(y).reshape(M, N)))


def _is_nan_bf16(b):
    return ((b & 0x7F80) == 0x7F80) & ((b & 0x007F) != 0)


def test_gelu_bf16_every_pattern():
    """All 65536 bf16 bit patterns: the library's GELU (the epilogue's table and closed
    forms) equals the oracle's fp64 GELU rounded once to bf16, bit for bit; where the
    oracle gives NaN (NaN inputs, -Inf) the library gives NaN."""
    ops = _ops()
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = torch.from_numpy(allb.view(np.int16)).view(torch.bfloat16).cuda()
    y = _bits_np(ops.gelu_bf16(x))
    assert ops.poll_status() == 0
    ref = oracle.gelu_bf16(allb)
    nan_ref = _is_nan_bf16(ref)
    assert np.array_equal(_is_nan_bf16(y), nan_ref)
    bad = np.nonzero((y != ref) & ~nan_ref)[0]
    assert bad.size == 0, "GELU differs on %d bf16 values, e.g. %s" % (
        bad.size, [(hex(int(allb[i])), hex(int(y[i])), hex(int(ref[i]))) for i in bad[:5]])
    # in place gives the same
    ops.gelu_bf16(x, out=x)
    assert np.array_equal(_bits_np(x), y)


def test_gemm_gelu_quant_padding_rows_are_zero():
    """Rows between M and the next multiple of 128 get scale 0 in the tiled layout,
    whatever the buffer held before."""
    ops = _ops()
    M, N, K = 200, 256, 256
    x = synth.activation(M, K, "normal", seed=3, device="cuda")
    qw = ops.quantize_weight(synth.weight(N, K, seed=4, device="cuda"))
    xc, xs = ops.quantize_act(x, "e2m1")
    sf = torch.full((ops.sf_bytes(M, N),), 0x77, dtype=torch.uint8, device="cuda")
    codes = torch.empty((ops.codes_bytes(M, N, "e2m1"),), dtype=torch.uint8, device="cuda")
    ops.gemm_gelu_quant(xc, xs, "e2m1", M, K, qw, out_fmt="e2m1", codes=codes, sf=sf)
    assert ops.poll_status() == 0
    h = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ops.gemm_gelu_quant(xc, xs, "e2m1", M, K, qw, out_fmt="e2m1", h=h)
    _, s_o = oracle.quantize(_bits_np(h).reshape(M, N), oracle.E2M1)
    assert np.array_equal(sf.cpu().numpy(), oracle.sf_to_tiled(s_o, N))
    assert not (sf == 0x77).any()


def oracle_ffn_rows(x, w1, b1, w2, b2, up_fmt, down_fmt, rows):
    """The unfused FFN in fp64 on the listed rows: linear -> bf16 -> GELU -> bf16 ->
    MX quantize -> linear."""
    xr = x[torch.as_tensor(rows, device=x.device)]
    h, hc, hs = oracle_hidden(xr, w1, b1, up_fmt, down_fmt)
    wc, ws, _ = _mx.oracle_quantize(w2, "e2m1")
    return oracle.linear_rows(hc, hs, _mx.FMT[down_fmt], np.arange(len(rows), dtype=np.int64), w1.shape[0], wc, ws,
                              _mx.bits(b2))


@pytest.mark.parametrize("up_fmt,down_fmt", [("e2m1", "e2m1"), ("e2m1", "e4m3"), ("e4m3", "e2m1"),
                                             ("e4m3", "e4m3")])
def test_ffn_against_oracle(up_fmt, down_fmt):
    ops = _ops()
    M, K, H, N2 = 300, 512, 1024, 256
    x = synth.activation(M, K, "normal", seed=5, device="cuda", outlier_frac=0.02, outlier_scale=30.0)
    w1, b1 = synth.weight(H, K, seed=6, device="cuda"), synth.bias(H, seed=6, device="cuda")
    w2, b2 = synth.weight(N2, H, seed=7, device="cuda"), synth.bias(N2, seed=7, device="cuda")
    up, down = ops.quantize_weight(w1, bias=b1), ops.quantize_weight(w2, bias=b2)
    y = ops.ffn(x, up, down, up_fmt, down_fmt)
    assert ops.poll_status() == 0
    assert "ffn" in ops.last_path()
    ref = oracle_ffn_rows(x, w1, b1, w2, b2, up_fmt, down_fmt, np.arange(M))
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "ffn %s->%s" % (up_fmt, down_fmt))
    # the same chain through the separate entry points gives the same bits
    xc, xs = ops.quantize_act(x, up_fmt)
    hc, hs = ops.gemm_gelu_quant(xc, xs, up_fmt, M, K, up, out_fmt=down_fmt)
    y2 = ops.gemm(hc, hs, down_fmt, M, H, down)
    assert torch.equal(y, y2)


@pytest.mark.slow
@pytest.mark.parametrize("down_fmt", ["e2m1", "e4m3"])
def test_ffn_full_720p_sampled_rows(down_fmt):
    """The block's FFN at full size (M = 75600 tokens, dim 5120, hidden 13824), FFN-down in
    W4A4 or W4A8; h and the output checked on one row per 1024-row span plus the ends."""
    ops = _ops()
    c = synth.BLOCK_720P
    M = c["M"]
    ws, bs = synth.block_weights(c["seed"], device="cuda")
    i_up = [n for n, *_ in synth.BLOCK_LINEARS].index("ffn_up")
    i_dn = [n for n, *_ in synth.BLOCK_LINEARS].index("ffn_down")
    w1, b1, w2, b2 = ws[i_up], bs[i_up], ws[i_dn], bs[i_dn]
    x = synth.activation(M, w1.shape[1], "normal", seed=c["seed"] * 100 + i_up, device="cuda",
                         outlier_frac=0.01, outlier_scale=30.0)
    up, down = ops.quantize_weight(w1, bias=b1), ops.quantize_weight(w2, bias=b2)
    y = ops.ffn(x, up, down, "e2m1", down_fmt)
    assert ops.poll_status() == 0
    rows = synth.sample_rows(M, tile=1024).numpy()
    ref = oracle_ffn_rows(x, w1, b1, w2, b2, "e2m1", down_fmt, rows)
    _mx.assert_gemm_close(_mx.bf16_to_f64(y[torch.from_numpy(rows).cuda()]), ref, "ffn 720p ->" + down_fmt)
    # the hidden activation of the same launch configuration, on the sampled rows
    xc, xs = ops.quantize_act(x, "e2m1")
    h = torch.empty((M, w1.shape[0]), dtype=torch.bfloat16, device="cuda")
    codes, sf = ops.gemm_gelu_quant(xc, xs, "e2m1", M, w1.shape[1], up, out_fmt=down_fmt, h=h)
    assert ops.poll_status() == 0
    r = torch.from_numpy(rows).cuda()
    h_ref, _, _ = oracle_hidden(x[r], w1, b1, "e2m1", down_fmt)
    eq = _bits_np(h[r]) == h_ref
    assert eq.mean() >= 0.99
    # the whole hidden activation: codes and tiled scales against the oracle's quantizer
    # applied to the GPU's h
    c_o, s_o = oracle.quantize(_bits_np(h).reshape(M, -1), _mx.FMT[down_fmt])
    assert np.array_equal(codes.cpu().numpy()[: c_o.size], c_o.reshape(-1))
    assert np.array_equal(sf.cpu().numpy(), oracle.sf_to_tiled(s_o, w1.shape[0]))
