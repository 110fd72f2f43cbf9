"""Calibration-driven block selection (the blog's section of that name, step 4-6 of its
"Practical workflow"): replay a block's captured inputs through plain MXFP4 W4A4 ("OFF")
and through MXFP4 with a transform ("ON": SmoothQuant scales and a fixed block Hadamard
rotation), measure the whole-block output SQNR of each against the bf16 block, and choose
a policy per (expert, block) with the tier rule (mxq_select_policy in the library).

The block's output here is the concatenation of its eight linears' outputs (attention and
norms are not part of this path).  The quantized outputs, the bf16 reference (the
library's bf16 GEMM, as a bf16 network computes the linear), the SmoothQuant scales and the
SQNR all come from the library's kernels."""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field

import torch

from . import _lib, ops

POLICIES = {0: "plain_mxfp4", 1: "transform_on", 2: "w4a8", 3: "bf16"}
TIERS = {"low": 0, "mid": 1, "high": 2}


def select(sqnr_off: float, sqnr_on: float, tier="high") -> str:
    """The tier rule for one block (see mxq_select_policy)."""
    p = _lib.lib().mxq_select_policy(float(sqnr_off), float(sqnr_on), TIERS[tier])
    if p < 0:
        raise ValueError("no policy for sqnr_off=%r sqnr_on=%r tier=%r" % (sqnr_off, sqnr_on, tier))
    return POLICIES[p]


def thresholds(tier="high"):
    f, w, m = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    _lib.check(_lib.lib().mxq_tier_thresholds(TIERS[tier], ctypes.byref(f), ctypes.byref(w), ctypes.byref(m)),
               "mxq_tier_thresholds")
    return f.value, w.value, m.value


def smoothquant_scales(x: torch.Tensor, w: torch.Tensor, alpha: float = 0.5):
    """SmoothQuant's per-channel scales s_k = max|X_k|^alpha / max|W_k|^(1 - alpha) and their
    reciprocals, the channel maxima and the scales computed by the library
    (mxq_channel_absmax, mxq_smooth_scales).  Returns (s, 1/s)."""
    return ops.smooth_scales(ops.channel_absmax(x), ops.channel_absmax(w), alpha, with_inverse=True)


def _sqnr_db(ref: list, out: list) -> float:
    """Whole-block SQNR (dB) of the outputs against the reference, by the library."""
    return float(ops.sqnr(ref, out)[2].item())


@dataclass
class BlockScore:
    sqnr_off: float
    sqnr_on: float
    policy: str = ""


def score_block(weights, biases, xs, hadamard_block: int = 128, alpha: float = 0.5) -> BlockScore:
    """OFF / ON whole-block SQNR of one block: weights and biases are the eight bf16
    linears (w [N, K], b [N] or None), xs their captured bf16 inputs."""
    ref, off, on = [], [], []
    for w, b, x in zip(weights, biases, xs):
        ref.append(ops.gemm_bf16(x, w, b))  # the bf16 block's linear
        qw = ops.quantize_weight(w, bias=b)
        off.append(ops.linear(x, qw, "e2m1"))
        s, inv_s = smoothquant_scales(x, w, alpha)
        qt = ops.quantize_weight_transformed(w, bias=b, block=hadamard_block, mul=s)
        on.append(ops.linear_transformed(x, qt, "e2m1", hadamard_block, inv_s))
    return BlockScore(_sqnr_db(ref, off), _sqnr_db(ref, on))


@dataclass
class Policy:
    """A per-expert, per-block policy: decisions[e][b] in POLICIES' values."""
    tier: str
    decisions: list = field(default_factory=list)
    scores: list = field(default_factory=list)

    def w4a8_bits(self, e: int, b: int) -> int:
        """The mxq_dit_block_linears mask of a block: all linears W4A8 when promoted."""
        return 0xFF if self.decisions[e][b] == "w4a8" else 0x00

    def counts(self):
        out = {}
        for row in self.decisions:
            for d in row:
                out[d] = out.get(d, 0) + 1
        return out


def calibrate(experts, inputs, tier="high", hadamard_block: int = 128, alpha: float = 0.5) -> Policy:
    """experts[e][b] = (weights, biases) of block b of expert e; inputs[e][b] = that block's
    eight captured inputs.  Returns the policy the tier rule picks for every block."""
    pol = Policy(tier)
    for e, blocks in enumerate(experts):
        dec, sc = [], []
        for b, (ws, bs) in enumerate(blocks):
            score = score_block(ws, bs, inputs[e][b], hadamard_block, alpha)
            score.policy = select(score.sqnr_off, score.sqnr_on, tier)
            dec.append(score.policy)
            sc.append(score)
        pol.decisions.append(dec)
        pol.scores.append(sc)
    return pol
