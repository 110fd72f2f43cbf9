"""The library's bf16 GEMM (the tcgen05 kernel with kind::f16 stages): y = a . b^T + bias
against the oracle's fp64 product within the GEMM tolerance, on ragged shapes (M below and
across the 128 / 256-row tiles, N across the 256-column tiles, K not a multiple of the
64-element stage); the QDQ linear and the low-rank branch activation run on it."""
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


@pytest.mark.parametrize("M,N,K", [(1, 8, 32), (127, 264, 96), (128, 256, 64), (300, 520, 1000), (513, 1288, 2048),
                                   (1000, 64, 5120)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemm_bf16_against_oracle(M, N, K, with_bias):
    ops = _ops()
    a = synth.activation(M, K, "normal", seed=M + K, device="cuda", outlier_frac=0.02, outlier_scale=20.0)
    b = synth.weight(N, K, seed=N + K, device="cuda")
    bias = synth.bias(N, seed=N, device="cuda") if with_bias else None
    y = ops.gemm_bf16(a, b, bias)
    assert ops.poll_status() == 0
    assert ops.last_path().startswith("bf16 kind::f16")
    ref = oracle.gemm_bf16(_mx.bits(a), _mx.bits(b), None if bias is None else _mx.bits(bias))
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "bf16 gemm %dx%dx%d" % (M, N, K))


def _quant_a(ops, a, b, fmt):
    """mxq_gemm_bf16_quant_a into guarded buffers: (y, codes, tiled scales) as numpy, the
    guard bands checked untouched."""
    M, K = a.shape
    nc, ns = ops.codes_bytes(M, K, fmt), ops.sf_bytes(M, K)
    codes = torch.full((nc + 64,), 0xA5, dtype=torch.uint8, device="cuda")
    sf = torch.full((ns + 64,), 0x5A, dtype=torch.uint8, device="cuda")
    y, _, _ = ops.gemm_bf16_quant_a(a, b, fmt, codes=codes, sf=sf)
    assert ops.poll_status() == 0
    assert ops.last_path().endswith("+quantize a->" + fmt)
    c, s = codes.cpu().numpy(), sf.cpu().numpy()
    assert (c[nc:] == 0xA5).all(), "codes guard band overwritten"
    assert (s[ns:] == 0x5A).all(), "scale guard band overwritten"
    return y, c[:nc], s[:ns]


def _assert_quant_equal(c, s, a, fmt, what):
    c_ref, _, s_ref = _mx.oracle_quantize(a, fmt)
    c_ref = c_ref.reshape(-1)
    if not np.array_equal(c, c_ref):
        i = int(np.nonzero(c != c_ref)[0][0])
        raise AssertionError("%s: %d code bytes differ, first at byte %d: gpu %#x oracle %#x" % (
            what, int((c != c_ref).sum()), i, c[i], c_ref[i]))
    if not np.array_equal(s, s_ref):
        i = int(np.nonzero(s != s_ref)[0][0])
        raise AssertionError("%s: tiled scales differ at byte %d: gpu %d oracle %d" % (what, i, s[i], s_ref[i]))


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
@pytest.mark.parametrize("M,N,K", [(1, 8, 32), (127, 64, 96), (257, 128, 320), (300, 72, 160), (600, 120, 2080),
                                   (1000, 64, 5120)])
def test_gemm_bf16_quant_a_against_oracle(fmt, M, N, K):
    """The bf16 GEMM that also quantizes its A: y against the oracle's fp64 product, and a's
    codes and tiled scales bit for bit against the oracle's quantizer, padding included.
    Ragged M (the tile's padding rows write scale 0 and no codes), K % 64 == 32 (the last
    stage's second block lies past K), K / 32 not a multiple of 4 (padding k-blocks after
    the last stage), N from 8 to 128 (MMAs 16 to 128 wide)."""
    ops = _ops()
    a = synth.activation(M, K, "student_t", seed=M + K + 1, device="cuda", outlier_frac=0.03, outlier_scale=40.0)
    b = synth.weight(N, K, seed=N + K, device="cuda")
    y, c, s = _quant_a(ops, a, b, fmt)
    _assert_quant_equal(c, s, a, fmt, "quant_a %dx%d %s" % (M, K, fmt))
    ref = oracle.gemm_bf16(_mx.bits(a), _mx.bits(b))
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "bf16 gemm quant_a %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_gemm_bf16_quant_a_every_bf16_pattern(fmt):
    """Every bf16 bit pattern (Inf and NaN blocks included), 31 to a block behind an amax
    carrier at 2^0 .. 2^19 times the block's largest magnitude, through the fused quantizer:
    codes and scales bit for bit against the oracle (the product is not checked: NaN and Inf
    rows are meant to poison it)."""
    from tests.test_quant_gpu import exhaustive_blocks
    ops = _ops()
    b = synth.weight(64, 256, seed=5, device="cuda")
    for shift in (0, 1, 2, 3, 8, 19):
        x = exhaustive_blocks(shift)
        n = x.shape[0] // 8 * 8
        x = x[:n].reshape(-1, 256).contiguous().cuda()
        _, c, s = _quant_a(ops, x, b, fmt)
        _assert_quant_equal(c, s, x, fmt, "every pattern, shift %d %s" % (shift, fmt))


def test_gemm_bf16_quant_a_rejects_bad_arguments():
    ops = _ops()
    a = torch.zeros((64, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError, match="above 128"):
        ops.gemm_bf16_quant_a(a, torch.zeros((136, 128), dtype=torch.bfloat16, device="cuda"), "e2m1")
    with pytest.raises(RuntimeError, match="multiple of 32"):
        ops.gemm_bf16_quant_a(torch.zeros((64, 40), dtype=torch.bfloat16, device="cuda"),
                              torch.zeros((64, 40), dtype=torch.bfloat16, device="cuda"), "e2m1")


def test_gemm_bf16_exact_case():
    """Operands whose products and partial sums are exact in fp32 (small integers times
    powers of two): the output is the exact sum rounded once to bf16, bit for bit."""
    ops = _ops()
    g = torch.Generator().manual_seed(3)
    M, N, K = 260, 264, 192
    a = (torch.randint(-8, 9, (M, K), generator=g).float() * 0.25).to(torch.bfloat16).cuda()
    b = torch.randint(-4, 5, (N, K), generator=g).float().to(torch.bfloat16).cuda()
    y = ops.gemm_bf16(a, b)
    ref = oracle.gemm_bf16(_mx.bits(a), _mx.bits(b))
    assert np.all(np.abs(ref) < 2 ** 11)  # multiples of 1/4 below 2^11: every partial sum exact in fp32
    assert np.array_equal(_mx.bits(y), oracle.round_bf16(ref))


def test_qdq_linear_runs_on_the_library_gemm():
    ops = _ops()
    M, N, K = 300, 520, 1024
    x = synth.activation(M, K, "gelu", seed=9, device="cuda", outlier_frac=0.01, outlier_scale=50.0)
    w = synth.weight(N, K, seed=10, device="cuda")
    b = synth.bias(N, seed=10, device="cuda")
    qw = ops.quantize_weight(w, bias=b)
    y = ops.linear(x, qw, "e4m3", mode="qdq")
    assert ops.poll_status() == 0
    path = ops.last_path()
    assert path.startswith("qdq e4m3 dequant + bf16 kind::f16") and "cublas" not in path.lower()
    xc, xs, _ = _mx.oracle_quantize(x, "e4m3")
    wc, ws, _ = _mx.oracle_quantize(w, "e2m1")
    ref = oracle.linear_rows(xc, xs, oracle.E4M3, np.arange(M), K, wc, ws, _mx.bits(b))
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "qdq linear")
