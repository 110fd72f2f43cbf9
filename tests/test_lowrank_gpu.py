"""The SVDQuant low-rank branch (blog sections "Results", "Calibration-driven block
selection"): y = deq(xq) . deq(Rq)^T + bf16(x . l1t^T) . l2t^T + bias, the branch's bf16
MMAs accumulating into the same TMEM accumulator as the block-scaled product."""
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


def oracle_lowrank(x, l1t, l2t, res, b, fmt, rows=None):
    xr = x if rows is None else x[torch.as_tensor(rows, device=x.device)]
    xc, xs, _ = _mx.oracle_quantize(xr, fmt)
    rc, rs, _ = _mx.oracle_quantize(res, "e2m1")
    n = np.arange(xr.shape[0], dtype=np.int64)
    return oracle.linear_lowrank_rows(xc, xs, _mx.FMT[fmt], n, x.shape[1], rc, rs, _mx.bits(xr), _mx.bits(l1t),
                                      _mx.bits(l2t), None if b is None else _mx.bits(b))


@pytest.mark.parametrize("M,N,K,rank,fmt", [(128, 256, 512, 64, "e2m1"), (300, 520, 1024, 128, "e2m1"),
                                            (129, 264, 1024, 64, "e4m3"), (513, 768, 2048, 256, "e2m1"),
                                            (1, 8, 128, 64, "e2m1"), (300, 544, 512, 192, "e4m3")])
def test_linear_lowrank_against_oracle(M, N, K, rank, fmt):
    ops = _ops()
    x = synth.activation(M, K, "student_t", seed=M + K, device="cuda", outlier_frac=0.01, outlier_scale=40.0)
    l1t, l2t, res = synth.lowrank_weight(N, K, rank, seed=N + rank, device="cuda")
    b = synth.bias(N, seed=N, device="cuda")
    qr = ops.quantize_weight(res, bias=b)
    y = ops.linear_lowrank(x, qr, l1t, l2t, fmt)
    assert ops.poll_status() == 0
    assert "+lowrank" in ops.last_path()
    ref = oracle_lowrank(x, l1t, l2t, res, b, fmt)
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "low-rank %dx%dx%d r=%d %s" % (M, N, K, rank, fmt))


def test_zero_branch_gives_the_plain_gemm_bit_for_bit():
    """With l1t = 0 the branch MMAs add exact zeros, so the output equals the plain GEMM
    of the residual bit for bit (the block-scaled accumulation order is unchanged)."""
    ops = _ops()
    M, N, K = 300, 520, 1024
    x = synth.activation(M, K, "normal", seed=5, device="cuda")
    l1t, l2t, res = synth.lowrank_weight(N, K, 64, seed=6, device="cuda")
    qr = ops.quantize_weight(res, bias=synth.bias(N, seed=6, device="cuda"))
    y = ops.linear_lowrank(x, qr, torch.zeros_like(l1t), l2t, "e2m1")
    y_plain = ops.linear(x, qr, "e2m1")
    assert ops.poll_status() == 0
    assert torch.equal(y, y_plain)


def test_svd_split_reconstructs_and_helps_w4a4():
    """ops.svd_split (offline preparation) reconstructs W to bf16 accuracy, and on a weight
    with a dominant low-rank part the branch raises the W4A4 SQNR against the unquantized
    product (the point of SVDQuant)."""
    ops = _ops()
    M, N, K, rank = 512, 512, 1024, 64
    l1t0, l2t0, res0 = synth.lowrank_weight(N, K, rank, seed=8, device="cuda", lr_scale=8.0)
    w = (l2t0.float() @ l1t0.float() + res0.float()).to(torch.bfloat16)
    l1t, l2t, res = ops.svd_split(w, rank)
    recon = l2t.float() @ l1t.float() + res.float()
    assert (recon - w.float()).norm() / w.float().norm() < 1e-2
    x = synth.activation(M, K, "student_t", seed=9, device="cuda", outlier_frac=0.01, outlier_scale=20.0)
    exact = (x.double() @ w.double().T).cpu().numpy()
    s_plain = _mx.sqnr_db(exact, _mx.bf16_to_f64(ops.linear(x, ops.quantize_weight(w), "e2m1")))
    s_lr = _mx.sqnr_db(exact, _mx.bf16_to_f64(ops.linear_lowrank(x, ops.quantize_weight(res), l1t, l2t, "e2m1")))
    print("W4A4 SQNR (dB): plain %.2f, with the rank-%d branch %.2f" % (s_plain, rank, s_lr))
    assert s_lr > s_plain


@pytest.mark.slow
def test_linear_lowrank_full_ffn_up_480p_sampled_rows():
    """FFN-up at 480p (M = 32760, K = 5120, N = 13824) with a rank-128 branch, in the
    launch configuration the benchmark times; sampled rows against the oracle."""
    ops = _ops()
    c = synth.WORKLOADS["ffn_up_480p_w4a4"]
    M, K, N = c["M"], c["K"], c["N"]
    x = synth.activation(M, K, c["act"], seed=c["seed"], device="cuda", outlier_frac=c["outlier_frac"],
                         outlier_scale=c["outlier_scale"])
    l1t, l2t, res = synth.lowrank_weight(N, K, 128, seed=c["seed"], device="cuda")
    b = synth.bias(N, seed=c["seed"], device="cuda")
    y = ops.linear_lowrank(x, ops.quantize_weight(res, bias=b), l1t, l2t, "e2m1")
    assert ops.poll_status() == 0
    rows = synth.sample_rows(M).numpy()
    ref = oracle_lowrank(x, l1t, l2t, res, b, "e2m1", rows=rows)
    _mx.assert_gemm_close(_mx.bf16_to_f64(y[torch.from_numpy(rows).cuda()]), ref, "low-rank FFN-up 480p")
