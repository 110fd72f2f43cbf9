"""GPU GEMM / linear parity against the CPU oracle (fp64 GEMM on the dequantized
operands).  Bounds: relative Frobenius error <= 2e-3 and, per output row,
max |y - y_ref| <= 1e-2 * max |y_ref|.  The operands the oracle multiplies come from
the oracle's own quantizer run on the same bf16 inputs; the GPU quantizer is checked
bit-exact against them first."""
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


def make_case(M, N, K, fmt, seed, bias=True, act="student_t"):
    x = synth.activation(M, K, act, seed=seed, device="cuda", outlier_frac=0.02, outlier_scale=40.0)
    w = synth.weight(N, K, seed=seed, device="cuda")
    b = synth.bias(N, seed=seed, device="cuda") if bias else None
    return x, w, b


def oracle_linear(x, w, b, fmt, rows=None):
    xc, xs, _ = _mx.oracle_quantize(x, fmt)
    wc, ws, _ = _mx.oracle_quantize(w, "e2m1")
    K = x.shape[1]
    bb = _mx.bits(b) if b is not None else None
    if rows is None:
        rows = np.arange(x.shape[0])
    return oracle.linear_rows(xc, xs, _mx.FMT[fmt], rows, K, wc, ws, bb)


SHAPES_W4A4 = [(128, 256, 256), (300, 520, 1056), (1, 8, 32), (127, 200, 64), (129, 264, 96),
               (513, 768, 2048), (256, 512, 5120)]
SHAPES_W4A8 = [(128, 256, 128), (300, 520, 1024), (1, 8, 128), (129, 200, 640), (513, 768, 2048)]


@pytest.mark.parametrize("M,N,K", SHAPES_W4A4)
def test_gemm_w4a4_full_compare(M, N, K):
    ops = _ops()
    x, w, b = make_case(M, N, K, "e2m1", seed=M + N + K)
    qw = ops.quantize_weight(w, bias=b)
    xc, xs = ops.quantize_act(x, "e2m1")
    y = ops.gemm(xc, xs, "e2m1", M, K, qw)
    assert "mxf4" in ops.last_path()
    assert ops.poll_status() == 0
    ref = oracle_linear(x, w, b, "e2m1")
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "w4a4 %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("M,N,K", SHAPES_W4A8)
def test_gemm_w4a8_full_compare(M, N, K):
    ops = _ops()
    x, w, b = make_case(M, N, K, "e4m3", seed=M + N + K + 1, act="gelu")
    qw = ops.quantize_weight(w, bias=b)
    xc, xs = ops.quantize_act(x, "e4m3")
    y = ops.gemm(xc, xs, "e4m3", M, K, qw)
    assert "mxf8f6f4" in ops.last_path()
    assert ops.poll_status() == 0
    ref = oracle_linear(x, w, b, "e4m3")
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "w4a8 %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_gemm_no_bias_and_guard_band(fmt):
    ops = _ops()
    M, N, K = 200, 264, 512
    x, w, _ = make_case(M, N, K, fmt, seed=5, bias=False)
    qw = ops.quantize_weight(w)
    xc, xs = ops.quantize_act(x, fmt)
    canary = 1232.0  # exact in bf16
    buf = torch.full(((M + 2) * N,), canary, dtype=torch.bfloat16, device="cuda")
    y = buf[: M * N].view(M, N)
    ops.gemm(xc, xs, fmt, M, K, qw, out=y)
    torch.cuda.synchronize()
    assert (buf[M * N:].float() == canary).all(), "GEMM wrote past the end of y"
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), oracle_linear(x, w, None, fmt), "no-bias " + fmt)


def test_gemm_lossless_operands_match_exact_product():
    """X and W built from random MX codes are exactly representable, so the GEMM must
    reproduce the fp64 product of the bf16 inputs to within bf16 output rounding."""
    ops = _ops()
    rng = np.random.default_rng(0)
    M, N, K = 256, 256, 512
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])

    def mx_matrix(rows):
        codes = rng.integers(0, 8, (rows, K))
        codes[:, ::32] = 7
        vals = grid[codes] * np.where(rng.integers(0, 2, (rows, K)), -1, 1) * \
            2.0 ** (np.repeat(rng.integers(-6, 3, (rows, K // 32)), 32, 1))
        return vals

    xv, wv = mx_matrix(M), mx_matrix(N)
    x = torch.from_numpy(xv).float().to(torch.bfloat16).cuda()
    w = torch.from_numpy(wv).float().to(torch.bfloat16).cuda()
    qw = ops.quantize_weight(w)
    xc, xs = ops.quantize_act(x, "e2m1")
    y = _mx.bf16_to_f64(ops.gemm(xc, xs, "e2m1", M, K, qw))
    ref = xv @ wv.T
    assert np.array_equal(y, torch.from_numpy(ref).float().to(torch.bfloat16).double().numpy()) or \
        np.abs(y - ref).max() <= 2 ** -8 * np.abs(ref).max()


@pytest.mark.parametrize("fmt,mode", [("e2m1", "native"), ("e4m3", "native"), ("e2m1", "qdq"), ("e4m3", "qdq")])
def test_linear_modes(fmt, mode):
    ops = _ops()
    M, N, K = 384, 512, 1024
    x, w, b = make_case(M, N, K, fmt, seed=11)
    qw = ops.quantize_weight(w, bias=b)
    y = ops.linear(x, qw, fmt=fmt, mode=mode)
    assert ops.poll_status() == 0
    ref = oracle_linear(x, w, b, fmt)
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "linear %s %s" % (fmt, mode))


def test_gemm_deterministic():
    ops = _ops()
    M, N, K = 640, 1024, 2048
    x, w, b = make_case(M, N, K, "e2m1", seed=21)
    qw = ops.quantize_weight(w, bias=b)
    ys = [ops.linear(x, qw, "e2m1") for _ in range(3)]
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16))


def test_w4a8_beats_w4a4_sqnr_on_outliers():
    """Diagnostic modelled on the blog's block SQNR (section "Calibration-driven block
    selection"): on heavy-tailed activations FP8 activations keep more signal."""
    ops = _ops()
    M, N, K = 512, 512, 2048
    x, w, _ = make_case(M, N, K, "e2m1", seed=31, bias=False)
    qw = ops.quantize_weight(w)
    y_ref = _mx.bf16_to_f64(x) @ _mx.bf16_to_f64(w).T
    s4 = _mx.sqnr_db(y_ref, _mx.bf16_to_f64(ops.linear(x, qw, "e2m1")))
    s8 = _mx.sqnr_db(y_ref, _mx.bf16_to_f64(ops.linear(x, qw, "e4m3")))
    assert s8 > s4


@pytest.mark.slow
@pytest.mark.parametrize("name", ["ffn_up_480p_w4a4", "ffn_down_720p_w4a8"])
def test_linear_full_workload_sampled_rows(name):
    """Full-size workloads in the launch configuration the benchmark times; the oracle
    checks one random row per 128-row tile plus the first and last rows."""
    ops = _ops()
    wl = synth.workload(name, device="cuda", with_bias=True)
    x, w, b, fmt = wl["x"], wl["w"], wl["bias"], wl["fmt"]
    qw = ops.quantize_weight(w, bias=b)
    y = ops.linear(x, qw, fmt=fmt)
    assert ops.poll_status() == 0
    rows = synth.sample_rows(wl["M"]).numpy()
    ref = oracle_linear(x, w, b, fmt, rows=rows)
    _mx.assert_gemm_close(_mx.bf16_to_f64(y[torch.from_numpy(rows).cuda()]), ref, name)
