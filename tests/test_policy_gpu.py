"""Calibration replay of the block policy on synthetic blocks (blog "Calibration-driven block
selection"): OFF / ON SQNR from the library's kernels, decisions by the tier rule, and the
emitted per-(expert, block) masks driving the block entry point."""
import math

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _inputs(M, ctx, seed, outlier_scale):
    xs = []
    for i, (name, N, K, src) in enumerate(synth.BLOCK_LINEARS):
        rows = M if src == "x" else ctx
        kind = "gelu" if name == "ffn_down" else "normal"
        xs.append(synth.activation(rows, K, kind, seed=seed * 100 + i, device="cuda", outlier_frac=0.01,
                                   outlier_scale=outlier_scale))
    return xs


def test_calibrate_two_experts():
    from fp8_mixed_precision_mxq_b200 import ops, policy
    M, ctx = 256, 64
    severities = [3.0, 40.0, 400.0]  # outlier-channel scales of the blocks' inputs
    experts, inputs = [], []
    for e in range(2):
        blocks, xin = [], []
        for b, sev in enumerate(severities):
            ws, bs = synth.block_weights(1000 + 10 * e + b, device="cuda")
            blocks.append((ws, bs))
            xin.append(_inputs(M, ctx, 2000 + 10 * e + b, sev))
        experts.append(blocks)
        inputs.append(xin)
    pol = policy.calibrate(experts, inputs, tier="high")
    print("decisions:", pol.decisions)
    print("sqnr off/on:", [[(round(s.sqnr_off, 1), round(s.sqnr_on, 1)) for s in row] for row in pol.scores])
    for e in range(2):
        for s in pol.scores[e]:
            # MXFP4 W4A4 on these synthetic blocks sits near the format's own SQNR
            assert math.isfinite(s.sqnr_off) and math.isfinite(s.sqnr_on)
            assert 5.0 < s.sqnr_off < 40.0 and 5.0 < s.sqnr_on < 40.0
        for b in range(3):
            s = pol.scores[e][b]
            assert pol.decisions[e][b] == policy.select(s.sqnr_off, s.sqnr_on, "high")
    # the policy's masks drive the block entry point: a promoted block runs W4A8 everywhere
    for e in range(2):
        for b in range(3):
            if pol.decisions[e][b] not in ("w4a8", "plain_mxfp4"):
                continue
            ws, bs = experts[e][b]
            qws = [ops.quantize_weight(w, bias=bb) for w, bb in zip(ws, bs)]
            bits = pol.w4a8_bits(e, b)
            ys = ops.dit_block_linears(qws, inputs[e][b], bits)
            fmt = "e4m3" if bits else "e2m1"
            for i in (0, 7):
                assert torch.equal(ys[i], ops.linear(inputs[e][b][i], qws[i], fmt))
    assert ops.poll_status() == 0
