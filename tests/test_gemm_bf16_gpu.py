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
