"""The DiT-block entry point: eight linears of one Wan-A14B-shaped block with a W4A4 /
W4A8 precision mask, and a two-expert stack driven by a per-expert, per-block mask
(the policy of the blog's sections "Mixed-Precision selection" and "Practical
workflow", step 6).  Every linear's output is checked against the CPU oracle."""
import numpy as np
import pytest
import torch

import synth
from tests import _mx
from tests.test_gemm_gpu import oracle_linear

pytestmark = pytest.mark.gpu


def _ops():
    from fp8_mixed_precision_mxq_b200 import ops
    return ops


def block(seed, device="cuda"):
    ops = _ops()
    ws, bs = synth.block_weights(seed, device=device)
    return [ops.quantize_weight(w, bias=b) for w, b in zip(ws, bs)], ws, bs


@pytest.mark.parametrize("bits", [0x00, 0xFF, 0x80, 0x5A])
def test_block_linears_against_oracle(bits):
    ops = _ops()
    M, ctx = 192, 64
    qws, ws, bs = block(seed=3)
    xs = synth.block_inputs(M, seed=3, device="cuda", ctx=ctx)
    ys = ops.dit_block_linears(qws, xs, bits)
    assert ops.poll_status() == 0
    assert ("0x%02x" % bits) in ops.last_path()
    rows = {M: synth.sample_rows(M, tile=32).numpy(), ctx: np.arange(ctx)}
    for i, (name, N, K, src) in enumerate(synth.BLOCK_LINEARS):
        fmt = "e4m3" if (bits >> i) & 1 else "e2m1"
        r = rows[xs[i].shape[0]]
        ref = oracle_linear(xs[i], ws[i], bs[i], fmt, rows=r)
        got = _mx.bf16_to_f64(ys[i][torch.from_numpy(r).cuda()])
        _mx.assert_gemm_close(got, ref, "block linear %s (%s)" % (name, fmt))


def test_block_qdq_mode_matches_native_within_tolerance():
    ops = _ops()
    M, ctx = 128, 32
    qws, ws, bs = block(seed=4)
    xs = synth.block_inputs(M, seed=4, device="cuda", ctx=ctx)
    bits = 0x80
    y_nat = ops.dit_block_linears(qws, xs, bits, mode="native")
    y_qdq = ops.dit_block_linears(qws, xs, bits, mode="qdq")
    assert ops.poll_status() == 0
    for i in (0, 6, 7):
        fmt = "e4m3" if (bits >> i) & 1 else "e2m1"
        r = np.arange(xs[i].shape[0])
        ref = oracle_linear(xs[i], ws[i], bs[i], fmt, rows=r)
        _mx.assert_gemm_close(_mx.bf16_to_f64(y_nat[i]), ref, "native %d" % i)
        _mx.assert_gemm_close(_mx.bf16_to_f64(y_qdq[i]), ref, "qdq %d" % i)


def test_two_expert_stack_follows_the_mask():
    """Two experts x three blocks with a per-(expert, block) mask: each block runs its
    linears with the precision its mask bit names; the W4A8 blocks differ from what the
    same weights give under W4A4, and each output matches the oracle in its own format."""
    ops = _ops()
    M, ctx = 96, 32
    mask = synth.expert_masks(n_experts=2, n_blocks=3, n_w4a8=1, seed=7)
    xs = synth.block_inputs(M, seed=9, device="cuda", ctx=ctx)
    for e in range(2):
        for blk in range(3):
            qws, ws, bs = block(seed=100 + 10 * e + blk)
            bits = 0xFF if mask[e, blk] else 0x00
            ys = ops.dit_block_linears(qws, xs, bits)
            fmt = "e4m3" if bits else "e2m1"
            for i in (1, 7):
                r = np.arange(xs[i].shape[0])
                ref = oracle_linear(xs[i], ws[i], bs[i], fmt, rows=r)
                _mx.assert_gemm_close(_mx.bf16_to_f64(ys[i]), ref, "expert %d block %d linear %d" % (e, blk, i))
    assert ops.poll_status() == 0


def test_block_rejects_wrong_workspace():
    ops = _ops()
    qws, _, _ = block(seed=5)
    xs = synth.block_inputs(64, seed=5, device="cuda", ctx=16)
    need = ops.block_workspace_bytes(qws, [x.shape[0] for x in xs], 0xFF, minimum=True)
    small = torch.empty(need // 2, dtype=torch.uint8, device="cuda")
    with pytest.raises(Exception) as ei:
        ops.dit_block_linears(qws, xs, 0xFF, workspace=small)
    assert "WORKSPACE" in str(ei.value)


@pytest.mark.parametrize("bits", [0x00, 0xFF, 0x5A])
def test_block_overlapped_equals_sequential(bits):
    """With a workspace that holds every linear's quantized input the block quantizes them
    on the library's side stream while the GEMMs run; with the minimum workspace it runs
    the linears one after another.  Both give the same bits, on two calls in a row."""
    ops = _ops()
    qws, _, _ = block(seed=9)
    xs = synth.block_inputs(300, seed=9, device="cuda", ctx=40)
    rows = [x.shape[0] for x in xs]
    big = torch.empty(ops.block_workspace_bytes(qws, rows, bits), dtype=torch.uint8, device="cuda")
    small = torch.empty(ops.block_workspace_bytes(qws, rows, bits, minimum=True), dtype=torch.uint8, device="cuda")
    assert big.numel() > small.numel()
    for _ in range(2):
        y_seq = ops.dit_block_linears(qws, xs, bits, workspace=small)
        assert "overlapped" not in ops.last_path()
        y_ovl = ops.dit_block_linears(qws, xs, bits, workspace=big)
        assert "overlapped" in ops.last_path()
        assert ops.poll_status() == 0
        for i, (a, b) in enumerate(zip(y_seq, y_ovl)):
            assert torch.equal(a, b), "linear %d differs" % i


@pytest.mark.slow
@pytest.mark.parametrize("mask_name", list(synth.BLOCK_MASKS))
def test_block_linears_full_720p_sampled_rows(mask_name):
    """One block at full size (M = 75600 video tokens, 512 text tokens) under each of
    the three masks; every linear's output is checked on one random row per 1024-row
    span plus the first and last rows (the oracle quantizes just those rows: the MX
    blocks of a row depend on nothing else)."""
    ops = _ops()
    c = synth.BLOCK_720P
    bits = synth.BLOCK_MASKS[mask_name]
    ws, bs = synth.block_weights(c["seed"], device="cuda")
    qws = [ops.quantize_weight(w, bias=b) for w, b in zip(ws, bs)]
    xs = synth.block_inputs(c["M"], seed=c["seed"], device="cuda", ctx=c["ctx"])
    ys = ops.dit_block_linears(qws, xs, bits)
    assert ops.poll_status() == 0
    rows = {c["M"]: synth.sample_rows(c["M"], tile=1024), c["ctx"]: synth.sample_rows(c["ctx"], tile=64)}
    for i, (name, N, K, src) in enumerate(synth.BLOCK_LINEARS):
        fmt = "e4m3" if (bits >> i) & 1 else "e2m1"
        r = rows[xs[i].shape[0]].cuda()
        ref = oracle_linear(xs[i][r], ws[i], bs[i], fmt)
        _mx.assert_gemm_close(_mx.bf16_to_f64(ys[i][r]), ref, "%s: linear %s (%s)" % (mask_name, name, fmt))


@pytest.mark.slow
def test_two_expert_stack_full_480p_sampled_linears():
    """The two-expert, 40-block stack at full size: all 80 blocks quantized and resident
    (~15 GB of MXFP4), 8 random blocks per expert promoted to W4A8 by the mask, and the
    forward of each expert issued block by block through the block entry point.  Four
    (block, linear) pairs per expert, two from W4A8 blocks and two from W4A4 blocks, are
    checked against the oracle on sampled rows (the oracle re-derives their bf16 weights
    from the same seeds)."""
    ops = _ops()
    c = synth.STACK_480P
    M, ctx = c["M"], c["ctx"]
    mask = synth.expert_masks(c["n_experts"], c["n_blocks"], c["n_w4a8"], seed=c["seed"])
    xs = synth.block_inputs(M, seed=c["seed"], device="cuda", ctx=ctx)
    stack = []
    for e in range(c["n_experts"]):
        blocks = []
        for blk in range(c["n_blocks"]):
            ws, bs = synth.block_weights(synth.stack_block_seed(e, blk), device="cuda")
            blocks.append([ops.quantize_weight(w, bias=b) for w, b in zip(ws, bs)])
            del ws, bs
        stack.append(blocks)
    g = torch.Generator().manual_seed(c["seed"])
    samples = {}
    for e in range(c["n_experts"]):
        hi = [int(b) for b in torch.nonzero(mask[e]).flatten()]
        lo = [int(b) for b in torch.nonzero(mask[e] == 0).flatten()]
        for pool in (hi, lo):
            for j in torch.randperm(len(pool), generator=g)[:2]:
                samples[(e, pool[int(j)])] = int(torch.randint(8, (1,), generator=g))
    rows = {M: synth.sample_rows(M, tile=1024).cuda(), ctx: synth.sample_rows(ctx, tile=64).cuda()}
    rows_i = [rows[x.shape[0]] for x in xs]
    ws_bytes = ops.block_workspace_bytes(stack[0][0], [x.shape[0] for x in xs], 0xFF)
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    outs = [torch.empty((x.shape[0], w.N), dtype=torch.bfloat16, device="cuda") for x, w in zip(xs, stack[0][0])]
    got = {}
    for e in range(c["n_experts"]):
        for blk in range(c["n_blocks"]):
            bits = 0xFF if mask[e, blk] else 0x00
            ops.dit_block_linears(stack[e][blk], xs, bits, workspace=workspace, outs=outs)
            if (e, blk) in samples:
                i = samples[(e, blk)]
                got[(e, blk, i)] = outs[i][rows_i[i]].clone()
    assert ops.poll_status() == 0
    assert len(got) == 4 * c["n_experts"]
    for (e, blk, i), y in sorted(got.items()):
        ws, bs = synth.block_weights(synth.stack_block_seed(e, blk), device="cuda")
        fmt = "e4m3" if mask[e, blk] else "e2m1"
        ref = oracle_linear(xs[i][rows_i[i]], ws[i], bs[i], fmt)
        _mx.assert_gemm_close(_mx.bf16_to_f64(y), ref, "expert %d block %d linear %s (%s)" % (
            e, blk, synth.BLOCK_LINEARS[i][0], fmt))
