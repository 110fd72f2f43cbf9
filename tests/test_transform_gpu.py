"""The transform_on path (blog section "Mixed-Precision selection": smoothing and a fixed
Hadamard rotation before quantization), checked against the oracle's definition
t = (x * mul) . blockdiag(H_B) / sqrt(B) taken in fp64: scales and codes bit-exact wherever
the definition's value is farther from a decision boundary than the error bound of a
binary32 evaluation, one of the two neighbouring codes within it (tests/_mx.py,
check_transformed); the transformed linear within the GEMM tolerance of the oracle's
product of the transformed operands."""
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


def smooth_scales(x, alpha=0.5, seed=0):
    """SmoothQuant-style per-channel scales s_k = max|x_k|^alpha (a calibration stand-in)."""
    s = x.abs().amax(dim=0).float().clamp_min(1e-3) ** alpha
    return s.contiguous()


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
@pytest.mark.parametrize("block", [32, 128])
@pytest.mark.parametrize("smooth", [False, True])
@pytest.mark.parametrize("M,K", [(1, 128), (129, 256), (300, 1024)])
def test_quantize_transformed_against_definition(fmt, block, smooth, M, K):
    ops = _ops()
    x = synth.activation(M, K, "student_t", seed=M + K + block, device="cuda", outlier_frac=0.02, outlier_scale=40.0)
    mul = (1.0 / smooth_scales(x)).contiguous() if smooth else None
    codes, sf = ops.quantize_act_transformed(x, fmt, block, mul)
    torch.cuda.synchronize()
    ref = oracle.quantize_transformed(_mx.bits(x), _mx.FMT[fmt], block, None if mul is None else mul.cpu().numpy())
    _mx.check_transformed(codes, sf, M, K, fmt, ref, "%s B=%d smooth=%s %dx%d" % (fmt, block, smooth, M, K),
                          max_uncertain=_mx.UNCERTAIN_LIMIT[fmt] * (1 if M * K >= 10000 else 10))


@pytest.mark.parametrize("block", [32, 128])
def test_transformed_linear_against_oracle(block):
    ops = _ops()
    M, N, K = 300, 520, 1024
    x = synth.activation(M, K, "student_t", seed=11, device="cuda", outlier_frac=0.01, outlier_scale=50.0)
    w = synth.weight(N, K, seed=12, device="cuda")
    b = synth.bias(N, seed=12, device="cuda")
    s = smooth_scales(x)
    inv_s = (1.0 / s).contiguous()
    qw = ops.quantize_weight_transformed(w, bias=b, block=block, mul=s)
    y = ops.linear_transformed(x, qw, "e2m1", block, inv_s)
    assert ops.poll_status() == 0
    assert "hadamard%d smooth" % block in ops.last_path()
    xo = oracle.quantize_transformed(_mx.bits(x), oracle.E2M1, block, inv_s.cpu().numpy())
    wo = oracle.quantize_transformed(_mx.bits(w), oracle.E2M1, block, s.cpu().numpy())
    ref = oracle.linear_rows(xo["codes"], xo["sf"], oracle.E2M1, np.arange(M), K, wo["codes"], wo["sf"], _mx.bits(b))
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "transformed linear, block %d" % block)
    # the transforms cancel: the result approximates the unquantized product
    exact = (x.double() @ w.double().T + b.double()).cpu().numpy()
    assert _mx.sqnr_db(exact, _mx.bf16_to_f64(y)) > 15.0


def test_transform_sqnr_report():
    """W4A4 SQNR against the unquantized product on the outlier recipe, plain vs rotated
    vs smoothed + rotated (a diagnostic; the values are printed, only a floor is asserted)."""
    ops = _ops()
    M, N, K = 512, 512, 2048
    x = synth.activation(M, K, "student_t", seed=21, device="cuda", outlier_frac=0.01, outlier_scale=50.0)
    w = synth.weight(N, K, seed=22, device="cuda")
    exact = (x.double() @ w.double().T).cpu().numpy()
    plain = _mx.sqnr_db(exact, _mx.bf16_to_f64(ops.linear(x, ops.quantize_weight(w), "e2m1")))
    res = {"plain": plain}
    for block in (32, 128):
        rot = ops.linear_transformed(x, ops.quantize_weight_transformed(w, block=block), "e2m1", block)
        res["hadamard%d" % block] = _mx.sqnr_db(exact, _mx.bf16_to_f64(rot))
        s = smooth_scales(x)
        sm = ops.linear_transformed(x, ops.quantize_weight_transformed(w, block=block, mul=s), "e2m1", block,
                                    (1.0 / s).contiguous())
        res["smooth+hadamard%d" % block] = _mx.sqnr_db(exact, _mx.bf16_to_f64(sm))
    print("W4A4 SQNR (dB):", {k: round(v, 2) for k, v in res.items()})
    assert min(res.values()) > 10.0


def special_input(M, K, seed):
    """bf16 rows whose 32-value blocks take magnitudes from 2^-140 (bf16 subnormals) to
    2^126 (the butterflies overflow to Inf there), plus NaN, +-Inf, +-0 and blocks of
    equal values (their rotation is exact zeros but one)."""
    g = torch.Generator().manual_seed(seed)
    exps = torch.tensor([-140, -134, -130, -127, -124, -120, -117, -115, -100, 0, 100, 115, 118, 120, 122, 124, 125,
                         126], dtype=torch.float64)
    pick = exps[torch.randint(len(exps), (M, K // 32), generator=g)]
    x = torch.randn(M, K, generator=g, dtype=torch.float64) * torch.repeat_interleave(2.0 ** pick, 32, dim=1)
    x = x.to(torch.bfloat16)
    x[0, 5] = float("nan")
    x[1, 77] = float("inf")
    x[2, 300 % K] = float("-inf")
    x[3] = 0.0
    x[4, : K // 2] = -0.0
    x[5, :32] = 1.0
    x[5, 7] = 1.0 + 2.0 ** -7
    x[6, 32:64] = 2.0 ** -125
    return x


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
@pytest.mark.parametrize("block", [32, 128])
@pytest.mark.parametrize("smooth", [False, True])
def test_quantize_transformed_special_values(fmt, block, smooth):
    """Subnormal, overflowing and non-finite inputs against the definition: non-finite
    blocks get scale 255 and zero codes on both sides; blocks whose rotation could overflow
    binary32, or whose values sit in the subnormal range where binary32 rounds absolutely,
    fall in the oracle's uncertain set, and every certain scale and code is exact."""
    ops = _ops()
    M, K = 48, 512
    x = special_input(M, K, seed=block + (7 if smooth else 0))
    mul = None
    if smooth:
        g = torch.Generator().manual_seed(5)
        mul = (2.0 ** (torch.rand(K, generator=g) * 8.0 - 4.0)).float().contiguous()
    xd = x.cuda()
    codes, sf = ops.quantize_act_transformed(xd, fmt, block, None if mul is None else mul.cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_transformed(_mx.bits(x), _mx.FMT[fmt], block, None if mul is None else mul.numpy())
    assert (ref["sf"] == 255).any() and (ref["sf"] == 0).any()  # the input reaches both ends of the scale range
    _mx.check_transformed(codes, sf, M, K, fmt, ref, "special values", max_uncertain=None)


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
@pytest.mark.parametrize("block", [32, 128])
@pytest.mark.parametrize("M,K", [(9000, 2176), (4000, 5120)])
def test_quantize_transformed_multi_span(fmt, block, M, K):
    """Tensors of more MX blocks than the launch has lanes (148 SMs x 32 CTAs x 128), so
    every warp takes several spans and the per-channel multipliers it holds must stay the
    ones of its channels; K = 2176 and 5120 make the launch round its grid to multiples of
    17 and 5 CTAs.  Whole tensor against the definition."""
    ops = _ops()
    x = synth.activation(M, K, "student_t", seed=M + block, device="cuda", outlier_frac=0.02, outlier_scale=40.0)
    mul = (1.0 / smooth_scales(x)).contiguous()
    codes, sf = ops.quantize_act_transformed(x, fmt, block, mul)
    torch.cuda.synchronize()
    ref = oracle.quantize_transformed(_mx.bits(x), _mx.FMT[fmt], block, mul.cpu().numpy())
    _mx.check_transformed(codes, sf, M, K, fmt, ref, "multi-span %dx%d" % (M, K))


@pytest.mark.slow
@pytest.mark.parametrize("block", [32, 128])
def test_transform_full_ffn_up_480p(block):
    """The bench's transform_on workload at full size (M = 32760, K = 5120, SmoothQuant-style
    multipliers): the quantizer's codes and scales against the definition on the whole
    tensor, in the launch configuration the bench times; the transformed linear (N = 13824)
    within the GEMM tolerance on one row per 128-row tile plus the ends."""
    ops = _ops()
    wl = synth.workload("ffn_up_480p_w4a4", device="cuda", with_bias=True)
    x, w, b, M, K = wl["x"], wl["w"], wl["bias"], wl["M"], wl["K"]
    s = smooth_scales(x)
    inv_s = (1.0 / s).contiguous()
    codes, sf = ops.quantize_act_transformed(x, "e2m1", block, inv_s)
    torch.cuda.synchronize()
    xb = _mx.bits(x)
    ref = oracle.quantize_transformed(xb, oracle.E2M1, block, inv_s.cpu().numpy())
    n_unc = _mx.check_transformed(codes, sf, M, K, "e2m1", ref, "480p B=%d" % block)
    print("480p transform B=%d: %d uncertain elements of %d" % (block, n_unc, M * K))
    qw = ops.quantize_weight_transformed(w, bias=b, block=block, mul=s)
    y = ops.linear_transformed(x, qw, "e2m1", block, inv_s)
    assert ops.poll_status() == 0
    rows = synth.sample_rows(M).numpy()
    wo = oracle.quantize_transformed(_mx.bits(w), oracle.E2M1, block, s.cpu().numpy())
    K2 = K // 2
    ref_y = oracle.linear_rows(ref["codes"].reshape(M, K2)[rows], ref["sf"][rows], oracle.E2M1, np.arange(len(rows)),
                               K, wo["codes"], wo["sf"], _mx.bits(b))
    _mx.assert_gemm_close(_mx.bf16_to_f64(y[torch.from_numpy(rows).cuda()]), ref_y, "transformed linear 480p")


@pytest.mark.slow
@pytest.mark.parametrize("block", [32, 128])
def test_transform_720p_sampled_rows(block):
    """The bench's headline transform_on shape (M = 75600, K = 5120) in the launch
    configuration the bench times: the whole tensor quantized on the GPU, one row per
    128-row tile plus the ends checked against the definition."""
    ops = _ops()
    wl = synth.workload("ffn_up_720p_w4a4", device="cuda", with_bias=False)
    x, M, K = wl["x"], wl["M"], wl["K"]
    s = smooth_scales(x)
    inv_s = (1.0 / s).contiguous()
    codes, sf = ops.quantize_act_transformed(x, "e2m1", block, inv_s)
    assert ops.poll_status() == 0
    rows = synth.sample_rows(M).numpy()
    xs = _mx.bits(x[torch.from_numpy(rows).cuda()])
    ref = oracle.quantize_transformed(xs, oracle.E2M1, block, inv_s.cpu().numpy())
    cg = codes.view(M, K // 2)[torch.from_numpy(rows).cuda()].cpu().numpy()
    sg = _mx.tiled_to_logical(sf.cpu().numpy(), M, K)[rows]
    n_unc = _mx.check_transformed(cg, sg, len(rows), K, "e2m1", ref, "720p B=%d sampled rows" % block)
    print("720p transform B=%d: %d uncertain elements of %d sampled" % (block, n_unc, len(rows) * K))
