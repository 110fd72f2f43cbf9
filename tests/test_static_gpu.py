"""Static per-tensor FP8 E4M3 activations (the blog's W4A8 as its "Quantization formats"
table names it): calibration by abs-max, codes bit-exact against the oracle's exact
quotient RNE_sat(x / s) -- including inputs whose code a binary32 evaluation of x / s would
get wrong, and scales across the whole binary32 range -- block scales all 127 in the tiled
layout, and the scaled W4A8 linear within the GEMM tolerance."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _exact, _mx

pytestmark = pytest.mark.gpu


def _ops():
    from fp8_mixed_precision_mxq_b200 import ops
    return ops


@pytest.mark.parametrize("M,K", [(1, 32), (127, 64), (300, 1024), (513, 2080)])
def test_absmax_is_exact(M, K):
    ops = _ops()
    x = synth.activation(M, K, "student_t", seed=M, device="cuda", outlier_frac=0.02, outlier_scale=40.0)
    got = ops.absmax(x).item()
    assert got == x.abs().max().float().item()


@pytest.mark.parametrize("M,K", [(1, 32), (127, 64), (129, 96), (300, 1024), (513, 2080)])
@pytest.mark.parametrize("scale_kind", ["calibrated", "small", "large"])
def test_quantize_static_bitexact(M, K, scale_kind):
    ops = _ops()
    x = synth.activation(M, K, "gelu", seed=M + K, device="cuda", outlier_frac=0.02, outlier_scale=50.0)
    amax = ops.absmax(x).item()
    scale = {"calibrated": amax / 448.0, "small": amax / 4000.0, "large": amax / 3.0}[scale_kind]
    codes, sf = ops.quantize_act_static(x, scale)
    torch.cuda.synchronize()
    want = oracle.quantize_static_e4m3(_mx.bits(x), scale).reshape(-1)
    got = codes.cpu().numpy()[: M * K]
    if not np.array_equal(got, want):
        i = int(np.nonzero(got != want)[0][0])
        raise AssertionError("code %d of %d differs: gpu %#x oracle %#x (x bits %#x)" % (
            i, int((got != want).sum()), got[i], want[i], _mx.bits(x).reshape(-1)[i]))
    logical = np.full((M, K // 32), 127, dtype=np.uint8)
    assert np.array_equal(sf.cpu().numpy(), oracle.sf_to_tiled(logical, K))


def _check_static(x_cpu, scale, what):
    ops = _ops()
    codes, sf = ops.quantize_act_static(x_cpu.cuda(), scale)
    torch.cuda.synchronize()
    want = oracle.quantize_static_e4m3(_mx.bits(x_cpu), scale).reshape(-1)
    got = codes.cpu().numpy()[: x_cpu.numel()]
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, "%s: %d codes differ, first %d: gpu %#x oracle %#x (x bits %#x, s %r)" % (
        what, bad.size, bad[0], got[bad[0]], want[bad[0]], _mx.bits(x_cpu).reshape(-1)[bad[0]], scale)


def test_quantize_static_near_ties():
    """Inputs whose E4M3 code is decided by less than a binary32 rounding: for each scale s
    of the exhaustive search in tests/_exact.py, the bf16 values x whose binary32 quotient
    or binary32 product x * fl32(1/s) lies on or across an E4M3 midpoint from x / s,
    scaled by powers of two across the E4M3 range, both signs, amid random fill."""
    cases = _exact.static_near_ties()
    by_scale = {}
    for s, x in cases:
        by_scale.setdefault(s, []).append(x)
    scales = sorted(by_scale)[:: max(1, len(by_scale) // 24)]
    g = torch.Generator().manual_seed(7)
    for s in scales:
        vals = [x * Fraction(2) ** j for x in by_scale[s] for j in range(-6, 9)]
        vals = [v for v in vals if Fraction(2) ** -9 <= v / s <= 448]
        bits = [_exact.bf16_bits(v) for v in vals] + [_exact.bf16_bits(v) | 0x8000 for v in vals]
        K = 64
        n = (len(bits) + K - 1) // K * K
        fill = (torch.randn(n, generator=g) * float(s) * 30).to(torch.bfloat16)
        fb = fill.view(torch.int16).numpy().view(np.uint16).copy()
        fb[: len(bits)] = np.array(bits, dtype=np.uint16)
        x = torch.from_numpy(fb.view(np.int16)).view(torch.bfloat16).reshape(n // K, K)
        _check_static(x, float(s), "near ties, s=%r" % float(s))


@pytest.mark.parametrize("scale", [2.0 ** -149, 3.0 * 2.0 ** -140, 1.1e-30, 0.7, 5.5e20, 3.0e38])
def test_quantize_static_extreme_scales_and_special_values(scale):
    """Scales from the smallest binary32 subnormal to near the largest finite value, with
    inputs from bf16 subnormals to the largest bf16, infinities (saturate to +-448) and
    NaN (the E4M3 NaN code)."""
    g = torch.Generator().manual_seed(int(np.log2(scale) + 200))
    M, K = 64, 256
    e = torch.randint(-140, 128, (M, K), generator=g).double()
    x = (torch.randn(M, K, generator=g, dtype=torch.float64) * 2.0 ** e).clamp(-3.0e38, 3.0e38).to(torch.bfloat16)
    x[0, 0], x[0, 1], x[0, 2], x[0, 3] = float("inf"), float("-inf"), float("nan"), -0.0
    x[1, :8] = torch.tensor([3.3895e38, -3.3895e38, 2.0 ** -133, -(2.0 ** -133), 2.0 ** -126, 1.0, -1.0, 0.0])
    # values near the scale itself, where the codes are neither zero nor saturated
    x[2:10] = (torch.randn(8, K, generator=g, dtype=torch.float64) * scale * 100).clamp(-3.0e38, 3.0e38).to(
        torch.bfloat16)
    _check_static(x, scale, "extreme scale")


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (300, 520, 1024), (1, 8, 128), (513, 768, 2048)])
def test_linear_static_against_oracle(M, N, K):
    ops = _ops()
    x = synth.activation(M, K, "gelu", seed=M + N, device="cuda", outlier_frac=0.01, outlier_scale=50.0)
    w = synth.weight(N, K, seed=N + K, device="cuda")
    b = synth.bias(N, seed=N, device="cuda")
    qw = ops.quantize_weight(w, bias=b)
    scale = ops.absmax(x).item() / 448.0
    y = ops.linear_static(x, qw, scale)
    assert ops.poll_status() == 0
    assert "static-scale" in ops.last_path()
    codes = oracle.quantize_static_e4m3(_mx.bits(x), scale)
    sf = np.full((M, K // 32), 127, dtype=np.uint8)
    wc, ws, _ = _mx.oracle_quantize(w, "e2m1")
    ref = oracle.linear_rows_scaled(codes, sf, oracle.E4M3, np.arange(M), K, wc, ws, scale, _mx.bits(b))
    _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "static W4A8 %dx%dx%d" % (M, N, K))


def test_w4a8_activation_forms_sqnr():
    """Both W4A8 activation forms against the product with unquantized activations, on
    GELU data with 1 % outlier channels x50 (the FFN-down recipe): each keeps an SQNR above
    25 dB.  The calibrated static scale does better here (about 31.7 vs 27.6 dB): under
    the floor rule a block's maximum lands in [256, 512) x its scale and E4M3 saturates at
    448, so blocks whose maximum falls in (448, 512) x scale clip it, which a scale of
    amax / 448 never does; the tensor's range fits E4M3's."""
    ops = _ops()
    M, N, K = 512, 512, 1024
    x = synth.activation(M, K, "gelu", seed=3, device="cuda", outlier_frac=0.01, outlier_scale=50.0)
    w = synth.weight(N, K, seed=4, device="cuda")
    qw = ops.quantize_weight(w)
    exact = (x.double() @ ops.dequantize(qw.codes, qw.sf, N, K).double().T).cpu().numpy()
    s_mx = _mx.sqnr_db(exact, _mx.bf16_to_f64(ops.linear(x, qw, "e4m3")))
    s_st = _mx.sqnr_db(exact, _mx.bf16_to_f64(ops.linear_static(x, qw, ops.absmax(x).item() / 448.0)))
    assert s_mx > 25.0 and s_st > 25.0, (s_mx, s_st)


def test_mx_e4m3_block_saturation_is_the_floor_rule():
    """A block whose maximum is 480: floor(log2 480) = 8, so the floor rule gives the
    scale 2^(8 - 8) = 1 (code 127); 480 / 1 is above 448 and the maximum saturates to 448
    under MX-E4M3, while a static scale of 480 / 448 maps it onto 448 exactly."""
    ops = _ops()
    x = torch.full((1, 32), 1.0, dtype=torch.bfloat16, device="cuda")
    x[0, 0] = 480.0
    codes, sf = ops.quantize_act(x, "e4m3")
    sc = ops.sf_to_logical(sf, 1, 32).cpu().numpy()[0, 0]
    deq_max = ops.dequantize(codes, sf, 1, 32, "e4m3")[0, 0].item()
    assert sc == 127 + 8 - 8 and deq_max == 448.0  # floor(log2 480) = 8, minus emax 8
    c_st, _ = ops.quantize_act_static(x, 480.0 / 448.0)
    assert c_st.cpu().numpy()[0] == 0x7E  # 480 / (480/448) = 448, the largest code


@pytest.mark.slow
def test_linear_static_full_ffn_down_720p_sampled_rows():
    """The FFN-down linear at 720p (M = 75600, K = 13824, N = 5120) with a calibrated static
    scale; one row per 128-row tile plus the first and last rows against the oracle."""
    ops = _ops()
    wl = synth.workload("ffn_down_720p_w4a8", device="cuda", with_bias=True)
    x, w, b, M, K = wl["x"], wl["w"], wl["bias"], wl["M"], wl["K"]
    qw = ops.quantize_weight(w, bias=b)
    scale = ops.absmax(x).item() / 448.0
    y = ops.linear_static(x, qw, scale)
    assert ops.poll_status() == 0
    rows = synth.sample_rows(M).numpy()
    xr = x[torch.from_numpy(rows).cuda()]
    codes = oracle.quantize_static_e4m3(_mx.bits(xr), scale)
    sf = np.full((len(rows), K // 32), 127, dtype=np.uint8)
    wc, ws, _ = _mx.oracle_quantize(w, "e2m1")
    ref = oracle.linear_rows_scaled(codes, sf, oracle.E4M3, np.arange(len(rows)), K, wc, ws, scale, _mx.bits(b))
    _mx.assert_gemm_close(_mx.bf16_to_f64(y[torch.from_numpy(rows).cuda()]), ref, "static FFN-down 720p")
