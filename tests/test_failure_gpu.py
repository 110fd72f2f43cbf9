"""Failure detection of the GEMM kernel without a GPU fault: with debug bit 0 set the
producer leaves the first pipeline stage of the first tile unfilled, so the MMA issuer's
bounded wait (one second) runs out.  The kernel must record MXQ_ERR_TIMEOUT in its
device status word, wind down on its own (no hang, TMEM freed), and leave the context
usable: the next call with the flag cleared gives the same output as a clean run."""
import time

import pytest
import torch

import synth
from tests import _mx

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,M", [("e2m1", 128), ("e4m3", 300)])
def test_gemm_bounded_wait_reports_timeout(fmt, M):
    from fp8_mixed_precision_mxq_b200 import _lib, ops
    K, N = 512, 512
    x = synth.activation(M, K, "normal", seed=11, device="cuda")
    qw = ops.quantize_weight(synth.weight(N, K, seed=12, device="cuda"))
    codes, sf = ops.quantize_act(x, fmt)
    assert ops.poll_status() == _lib.OK
    y_clean = ops.gemm(codes, sf, fmt, M, K, qw)
    assert ops.poll_status() == _lib.OK

    y_bad = torch.zeros_like(y_clean)
    ops.set_debug(1)
    try:
        t0 = time.monotonic()
        ops.gemm(codes, sf, fmt, M, K, qw, out=y_bad)  # launch succeeds; the wait runs out on the device
        status = ops.poll_status()
        elapsed = time.monotonic() - t0
    finally:
        ops.set_debug(0)
    assert status == _lib.ERR_TIMEOUT, _lib.STATUS_NAMES.get(status, status)
    assert "bounded wait" in _lib.last_error()
    assert elapsed < 30.0, "the kernel took %.1f s to wind down" % elapsed
    # the status word was cleared by the poll; the context still computes
    assert ops.poll_status() == _lib.OK
    y_again = ops.gemm(codes, sf, fmt, M, K, qw)
    assert ops.poll_status() == _lib.OK
    assert torch.equal(y_again, y_clean)
    assert torch.isfinite(y_again.float()).all()


def test_quantize_and_gemm_still_match_oracle_after_timeout():
    """After a timed-out launch, a fresh linear is still within the GEMM tolerance of
    the oracle."""
    import oracle
    from fp8_mixed_precision_mxq_b200 import _lib, ops
    M, K, N = 256, 1024, 384
    x = synth.activation(M, K, "student_t", seed=21, device="cuda", outlier_frac=0.01, outlier_scale=30.0)
    w = synth.weight(N, K, seed=22, device="cuda")
    qw = ops.quantize_weight(w)
    codes, sf = ops.quantize_act(x, "e2m1")
    ops.set_debug(1)
    try:
        ops.gemm(codes, sf, "e2m1", M, K, qw)
        assert ops.poll_status() == _lib.ERR_TIMEOUT
    finally:
        ops.set_debug(0)
    y = ops.linear(x, qw, "e2m1")
    assert ops.poll_status() == _lib.OK
    xc, xs, _ = _mx.oracle_quantize(x, "e2m1")
    wc, ws, _ = _mx.oracle_quantize(w, "e2m1")
    y_ref = oracle.linear(xc, xs, _mx.FMT["e2m1"], K, wc, ws)
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), y_ref, "linear after a timed-out launch")


@pytest.mark.parametrize("block", [32, 128])
def test_transform_quantizer_bounded_wait_reports_timeout(block):
    """Debug bit 1: the transform quantizer's first warp never issues its first span's
    copy, so that warp's bounded wait (one second) runs out; the kernel records
    MXQ_ERR_TIMEOUT, waits for its other copies and returns, and the next call with the
    flag cleared gives the clean result."""
    from fp8_mixed_precision_mxq_b200 import _lib, ops
    M, K = 300, 1024
    x = synth.activation(M, K, "student_t", seed=31, device="cuda")
    mul = torch.rand(K, device="cuda", dtype=torch.float32) + 0.5
    c_clean, s_clean = ops.quantize_act_transformed(x, "e2m1", block, mul)
    assert ops.poll_status() == _lib.OK
    ops.set_debug(2)
    try:
        t0 = time.monotonic()
        ops.quantize_act_transformed(x, "e2m1", block, mul)
        status = ops.poll_status()
        elapsed = time.monotonic() - t0
    finally:
        ops.set_debug(0)
    assert status == _lib.ERR_TIMEOUT, _lib.STATUS_NAMES.get(status, status)
    assert "quantizer" in _lib.last_error()
    assert elapsed < 30.0, "the kernel took %.1f s to wind down" % elapsed
    assert ops.poll_status() == _lib.OK
    c_again, s_again = ops.quantize_act_transformed(x, "e2m1", block, mul)
    assert ops.poll_status() == _lib.OK
    assert torch.equal(c_again, c_clean) and torch.equal(s_again, s_clean)
