"""GPU quantizer / dequantizer parity: codes and tiled scales bit-exact against the CPU
oracle on the same bf16 bytes (MX format of the blog's section "Quantization
formats": 32-element blocks, E8M0 scale, E2M1 / E4M3 elements, RTN)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _mx

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def gpu_quantize(x, fmt, canary=True):
    """Quantize through the C ABI into buffers pre-filled with a canary pattern and a
    64-byte guard band; returns (codes, sf) without the guard bands."""
    from fp8_mixed_precision_mxq_b200 import ops
    M, K = x.shape
    nc, ns = ops.codes_bytes(M, K, fmt), ops.sf_bytes(M, K)
    codes = torch.full((nc + 64,), 0xA5, dtype=torch.uint8, device=x.device)
    sf = torch.full((ns + 64,), 0x5A, dtype=torch.uint8, device=x.device)
    ops.quantize_act(x, fmt, codes=codes, sf=sf)
    torch.cuda.synchronize()
    c, s = codes.cpu().numpy(), sf.cpu().numpy()
    assert (c[nc:] == 0xA5).all(), "codes guard band overwritten"
    assert (s[ns:] == 0x5A).all(), "scale guard band overwritten"
    return c[:nc], s[:ns]


def assert_bitexact(x, fmt):
    M, K = x.shape
    c_gpu, s_gpu = gpu_quantize(x, fmt)
    c_ref, _, s_ref = _mx.oracle_quantize(x, fmt)
    c_ref = c_ref.reshape(-1)
    if not np.array_equal(c_gpu, c_ref):
        i = int(np.nonzero(c_gpu != c_ref)[0][0])
        rb = oracle.codes_row_bytes(K, _mx.FMT[fmt])
        raise AssertionError("%s codes differ: %d bytes, first at row %d byte %d: gpu %#x oracle %#x" % (
            fmt, int((c_gpu != c_ref).sum()), i // rb, i % rb, c_gpu[i], c_ref[i]))
    if not np.array_equal(s_gpu, s_ref):
        i = int(np.nonzero(s_gpu != s_ref)[0][0])
        raise AssertionError("%s tiled scales differ at byte %d: gpu %d oracle %d" % (fmt, i, s_gpu[i], s_ref[i]))


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
@pytest.mark.parametrize("M,K", [(1, 32), (127, 64), (129, 96), (300, 1024), (128, 160), (513, 2080)])
def test_quantize_bitexact_shapes(fmt, M, K):
    x = synth.activation(M, K, "student_t", seed=M + K, device="cuda", outlier_frac=0.03, outlier_scale=40.0)
    assert_bitexact(x, fmt)


def exhaustive_blocks(shift):
    """All 65536 bf16 bit patterns, 31 per block in pattern order, each block led by an
    amax carrier equal to the block's largest finite magnitude times 2^shift (capped
    at the largest finite bf16).  Blocks that hold Inf / NaN patterns test the
    non-finite convention."""
    pats = np.arange(65536, dtype=np.uint32)
    nblk = (65536 + 30) // 31
    pad = nblk * 31 - 65536
    pats = np.concatenate([pats, np.zeros(pad, dtype=np.uint32)]).reshape(nblk, 31)
    mags = (pats & 0x7FFF)
    finite = mags < 0x7F80
    mmax = np.where(finite, mags, 0).max(axis=1)
    exp = (mmax >> 7) + shift
    carrier = np.where(exp >= 255, 0x7F7F, np.minimum(exp, 254) << 7 | (mmax & 0x7F))
    carrier = np.where(mmax == 0, 0, carrier)
    blocks = np.concatenate([carrier[:, None], pats], axis=1).astype(np.uint16)
    return torch.from_numpy(blocks.reshape(-1, 32).view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_quantize_exhaustive_bf16_patterns(fmt):
    for shift in range(0, 20):
        x = exhaustive_blocks(shift)
        # 2115 blocks of 32 -> lay them out as rows of 8 blocks (K = 256)
        n = x.shape[0] // 8 * 8
        x = x[:n].reshape(-1, 256).contiguous().cuda()
        assert_bitexact(x, fmt)


def _expand(runs):
    out = []
    for v, n in runs:
        out += [float.fromhex(v) if isinstance(v, str) else v] * n
    return out


def test_quantize_hand_worked_blocks():
    blocks = json.load(open(os.path.join(GOLDEN, "hand_blocks.json")))["blocks"]
    for blk in blocks:
        x = torch.tensor(_expand(blk["x"]), dtype=torch.float32).to(torch.bfloat16).reshape(1, 32).cuda()
        c, s = gpu_quantize(x, blk["fmt"])
        assert int(s[0]) == blk["sf"], blk["name"]
        want = _expand(blk["codes"])
        got = list(c) if blk["fmt"] == "e4m3" else [v for b in c for v in (int(b) & 0xF, int(b) >> 4)]
        assert got == want, blk["name"]


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_sf_to_logical_and_dequantize(fmt):
    from fp8_mixed_precision_mxq_b200 import ops
    M, K = 257, 352
    x = synth.activation(M, K, "normal", seed=7, device="cuda", outlier_frac=0.05, outlier_scale=30.0)
    codes, sf = ops.quantize_act(x, fmt)
    logical = ops.sf_to_logical(sf, M, K).cpu().numpy()
    c_ref, s_ref, _ = _mx.oracle_quantize(x, fmt)
    assert np.array_equal(logical, s_ref)
    deq = ops.dequantize(codes, sf, M, K, fmt)
    want = torch.from_numpy(oracle.dequantize(c_ref, s_ref, K, _mx.FMT[fmt])).float().to(torch.bfloat16)
    assert torch.equal(deq.cpu().view(torch.int16), want.view(torch.int16))


def test_quantize_weight_matches_e2m1_activation_path():
    from fp8_mixed_precision_mxq_b200 import ops
    w = synth.weight(520, 1056, seed=3, device="cuda")
    qw = ops.quantize_weight(w)
    c_ref, _, s_ref = _mx.oracle_quantize(w, "e2m1")
    assert np.array_equal(qw.codes.cpu().numpy(), c_ref)
    assert np.array_equal(qw.sf.cpu().numpy(), s_ref)


def test_quantize_deterministic():
    from fp8_mixed_precision_mxq_b200 import ops
    x = synth.activation(1000, 2048, "student_t", seed=9, device="cuda", outlier_frac=0.01, outlier_scale=50.0)
    outs = [ops.quantize_act(x, "e2m1") for _ in range(3)]
    for c, s in outs[1:]:
        assert torch.equal(c, outs[0][0]) and torch.equal(s, outs[0][1])


@pytest.mark.slow
@pytest.mark.parametrize("name", ["ffn_up_480p_w4a4", "ffn_down_720p_w4a8"])
def test_quantize_bitexact_full_workload(name):
    c = synth.WORKLOADS[name]
    x = synth.activation(c["M"], c["K"], c["act"], seed=c["seed"], device="cuda",
                         outlier_frac=c.get("outlier_frac", 0.0), outlier_scale=c["outlier_scale"])
    assert_bitexact(x, c["fmt"])


@pytest.mark.slow
@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
@pytest.mark.parametrize("K", [32, 64])
def test_quantize_max_rows_sampled_tiles(fmt, K):
    """More than 2^24 rows at the smallest K: the kernel's row = block / (K/32) division
    needs more than 64 bits of product there.  Every 128-row tile of the tiled scales is
    a contiguous run of ceil(K/128) atoms, so sampled tiles (the first, the one starting
    at row 2^24, the ragged last one and random ones) are checked byte for byte, codes and
    scales, against the oracle on the same rows."""
    from fp8_mixed_precision_mxq_b200 import ops
    M = (1 << 24) + 200
    x = synth.activation(M, K, "student_t", seed=K, device="cuda", outlier_frac=0.01, outlier_scale=40.0)
    codes, sf = ops.quantize_act(x, fmt)
    torch.cuda.synchronize()
    rb = oracle.codes_row_bytes(K, _mx.FMT[fmt])
    tile_bytes = oracle.sf_tiled_bytes(128, K)
    n_tiles = (M + 127) // 128
    g = torch.Generator().manual_seed(K)
    tiles = {0, (1 << 24) // 128, n_tiles - 1} | {int(t) for t in torch.randint(n_tiles, (5,), generator=g)}
    for t in sorted(tiles):
        r0, r1 = 128 * t, min(M, 128 * t + 128)
        c_ref, s_ref, _ = _mx.oracle_quantize(x[r0:r1], fmt)
        c_gpu = codes[r0 * rb: r1 * rb].cpu().numpy().reshape(r1 - r0, rb)
        assert np.array_equal(c_gpu, c_ref), "codes of rows %d..%d differ" % (r0, r1 - 1)
        s_gpu = sf[t * tile_bytes: (t + 1) * tile_bytes].cpu().numpy()
        assert np.array_equal(s_gpu, oracle.sf_to_tiled(s_ref, K)), "scales of rows %d..%d differ" % (r0, r1 - 1)


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_dequantize_every_code_at_extreme_scales(fmt):
    """Every element code under scale codes 0-12, 120-130 and 240-255: the dequantized bf16
    equals the oracle's exact value rounded to nearest even (the binary32 product the
    kernel forms is exact, so one rounding to bf16 remains: E4M3 products below bf16's
    2^-133 step at scale codes 0-2 round, large scales overflow to Inf); NaN codes and the
    NaN scale give NaN."""
    from fp8_mixed_precision_mxq_b200 import ops
    scales = list(range(0, 13)) + list(range(120, 131)) + list(range(240, 256))
    M, K = len(scales), 512
    if fmt == "e4m3":
        row = np.tile(np.arange(256, dtype=np.uint8), K // 256)
    else:
        row = np.arange(256, dtype=np.uint8)  # every pair of E2M1 codes, K / 2 bytes
    codes = np.tile(row, (M, 1))
    logical = np.repeat(np.array(scales, dtype=np.uint8)[:, None], K // 32, axis=1)
    sf = oracle.sf_to_tiled(logical, K)
    deq = ops.dequantize(torch.from_numpy(codes.reshape(-1)).cuda(), torch.from_numpy(sf).cuda(), M, K, fmt)
    want = torch.from_numpy(oracle.dequantize(codes, logical, K, _mx.FMT[fmt])).to(torch.bfloat16)
    got = deq.cpu()
    nan_w, nan_g = torch.isnan(want), torch.isnan(got)
    assert torch.equal(nan_w, nan_g)
    assert torch.equal(got[~nan_g].view(torch.int16), want[~nan_w].view(torch.int16))
