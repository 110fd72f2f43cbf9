"""The policy's calibration and load-time arithmetic in the library: per-channel abs-max,
SmoothQuant scales, the whole-block SQNR and the SVDQuant split, each against the oracle's
fp64 restatement."""
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


@pytest.mark.parametrize("M,K", [(1, 8), (130, 96), (3000, 5120), (70000, 64)])
def test_channel_absmax_is_exact(M, K):
    ops = _ops()
    x = synth.activation(M, K, "student_t", seed=M + K, device="cuda", outlier_frac=0.05, outlier_scale=40.0)
    got = ops.channel_absmax(x).cpu().numpy().astype(np.float64)
    assert np.array_equal(got, oracle.channel_absmax(_mx.bits(x)))


def test_channel_absmax_propagates_nan_and_inf():
    ops = _ops()
    x = torch.randn(64, 32).to(torch.bfloat16)
    x[5, 3] = float("nan")
    x[7, 9] = float("-inf")
    got = ops.channel_absmax(x.cuda()).cpu().numpy()
    assert np.isnan(got[3]) and np.isposinf(got[9]) and np.isfinite(np.delete(got, [3, 9])).all()


@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 0.85, 1.0])
def test_smooth_scales_against_oracle(alpha):
    ops = _ops()
    g = torch.Generator().manual_seed(int(alpha * 100))
    K = 5120
    ax = (torch.rand(K, generator=g) * 50.0) ** 2
    aw = torch.rand(K, generator=g) * 0.1
    ax[:4] = torch.tensor([0.0, 1e-9, 3.0, 1e-5])
    aw[4:8] = torch.tensor([0.0, 1e-9, 2.0, 1e-5])
    s, inv = ops.smooth_scales(ax.cuda(), aw.cuda(), alpha, with_inverse=True)
    want = oracle.smooth_scales(ax.numpy(), aw.numpy(), alpha)
    got = s.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - want) <= 8 * 2.0 ** -24 * np.abs(want)), np.abs(got / want - 1).max()
    gi = inv.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(gi - 1.0 / want) <= 9 * 2.0 ** -24 * np.abs(1.0 / want))


def test_sqnr_against_oracle():
    ops = _ops()
    refs, tests = [], []
    for i, (M, N) in enumerate([(300, 512), (512, 1024), (64, 8)]):
        r = synth.activation(M, N, "normal", seed=i, device="cuda")
        noise = synth.activation(M, N, "normal", seed=100 + i, device="cuda")
        refs.append(r)
        tests.append((r.float() + 0.01 * noise.float()).to(torch.bfloat16))
    out = ops.sqnr(refs, tests).cpu().numpy()
    num, den, db = oracle.sqnr([_mx.bits(r) for r in refs], [_mx.bits(t) for t in tests])
    assert abs(out[0] - num) <= 1e-12 * num and abs(out[1] - den) <= 1e-12 * den
    assert abs(out[2] - db) <= 1e-9
    same = ops.sqnr(refs[:1], refs[:1]).cpu().numpy()
    assert same[1] == 0.0 and np.isposinf(same[2])


def _bf16_f32(t):
    return t.to(torch.bfloat16).float()


def test_lowrank_split_exact_factors():
    """Factors whose products with sqrt(S) are bf16 values (S powers of 4, U and Vh bf16
    values): l2t and l1t bit-exact; the residual equal to the oracle's on nearly all
    elements and everywhere within one bf16 step plus the fp32 accumulation bound of the
    rank-r sum (r 2^-24 sum_j |l2t l1t|, twice over: accumulation and the subtraction)."""
    ops = _ops()
    g = torch.Generator().manual_seed(8)
    N, K, r = 520, 1000, 64
    U = _bf16_f32(torch.randn(N, r, generator=g))
    Vh = _bf16_f32(torch.randn(r, K, generator=g))
    S = (4.0 ** torch.randint(-3, 4, (r,), generator=g)).float()
    w = synth.weight(N, K, seed=8)
    l1t, l2t, res = ops.lowrank_split(w.cuda(), U.cuda(), S.cuda(), Vh.cuda(), r)
    o1, o2, orr = oracle.lowrank_split(U.numpy(), S.numpy(), Vh.numpy(), _mx.bits(w), r)
    assert np.array_equal(_mx.bits(l1t), o1) and np.array_equal(_mx.bits(l2t), o2)
    got, want = _mx.bits(res), orr
    eq = got == want
    assert eq.mean() >= 0.99, eq.mean()
    gv, wv = oracle.bf16_bits_to_f64(got), oracle.bf16_bits_to_f64(want)
    ulp = np.maximum(np.abs(wv), 2.0 ** -126) * 2.0 ** -7
    s_abs = np.abs(oracle.bf16_bits_to_f64(o2)) @ np.abs(oracle.bf16_bits_to_f64(o1))
    acc = 2 * r * 2.0 ** -24 * s_abs
    assert np.all(np.abs(gv - wv) <= ulp + acc)


def test_svd_split_recomposes_the_weight():
    """ops.svd_split (torch's SVD, then the library's split) on a random weight with a
    low-rank part: l2t . l1t + residual gives back w to bf16 rounding, and the residual of
    rank 64 is much smaller than the weight."""
    ops = _ops()
    N, K, r = 512, 768, 64
    l1t0, l2t0, resid0 = synth.lowrank_weight(N, K, r, seed=4, device="cuda")
    w = (l2t0.float() @ l1t0.float() + resid0.float()).to(torch.bfloat16)
    l1t, l2t, res = ops.svd_split(w, r)
    back = l2t.double() @ l1t.double() + res.double()
    err = (back - w.double()).abs()
    assert float(err.max()) <= 2.0 ** -7 * float(w.double().abs().max())
    assert float(res.double().norm()) < 0.5 * float(w.double().norm())
