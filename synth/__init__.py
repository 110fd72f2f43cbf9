"""Seeded synthetic inputs shaped like the Wan2.2-A14B linear layers.

This module only draws random numbers; it holds none of the quantization
arithmetic.  Both the CUDA path and the CPU oracle are fed the exact same bf16
bytes produced here.

Shapes follow the blog "Quark Mixed-Precision Quantization for Wan2.2 Video
Generation on AMD Instinct GPUs" (section "Experimental setup": 832x480, 81 frames;
two experts of 40 transformer blocks each, section "Mixed-Precision selection")
with the Wan-A14B block dimensions (model dim 5120, 40 heads x 128, FFN 13824).
Token counts: 32760 at 480p/81 frames, 75600 at 720p/81 frames, text context 512.

Distributions: weights ~ N(0, 0.02^2); activations N(0,1), Student-t(nu=4) or
GELU(N(0,1)), with a few whole K-channels scaled up to make the outliers that
make MXFP4 activations hard.  All draws use torch generators seeded per tensor,
so a tensor can be produced on the GPU or on the CPU with the same recipe.
"""
from __future__ import annotations

import torch

# Dimensions of one Wan-A14B DiT block.
DIM = 5120
FFN = 13824
CTX = 512
TOKENS_480P = 32760
TOKENS_720P = 75600

# The eight linears of one DiT block, in issue order: (name, N, K, rows source).
# "x" rows are the video tokens, "ctx" rows the text context.
BLOCK_LINEARS = [
    ("qkv", 3 * DIM, DIM, "x"),
    ("attn_out", DIM, DIM, "x"),
    ("cross_q", DIM, DIM, "x"),
    ("cross_k", DIM, DIM, "ctx"),
    ("cross_v", DIM, DIM, "ctx"),
    ("cross_out", DIM, DIM, "x"),
    ("ffn_up", FFN, DIM, "x"),
    ("ffn_down", DIM, FFN, "x"),
]

WORKLOADS = {
    "small_w4a4": dict(M=128, K=1024, N=1024, act="normal", n_outlier=4, outlier_scale=30.0,
                       fmt="e2m1", seed=0),
    "ffn_up_480p_w4a4": dict(M=TOKENS_480P, K=DIM, N=FFN, act="student_t", outlier_frac=0.01,
                             outlier_scale=50.0, fmt="e2m1", seed=1),
    "ffn_down_720p_w4a8": dict(M=TOKENS_720P, K=FFN, N=DIM, act="gelu", outlier_frac=0.01,
                               outlier_scale=50.0, fmt="e4m3", seed=2),
    "ffn_up_720p_w4a4": dict(M=TOKENS_720P, K=DIM, N=FFN, act="student_t", outlier_frac=0.01,
                             outlier_scale=50.0, fmt="e2m1", seed=5),
}


# Block-level workloads.  BLOCK_720P: one DiT block's eight linears at 720p / 81 frames,
# run under three precision masks (bit i set = linear i in W4A8): all W4A4, all W4A8, and
# mixed with the FFN-down linear (whose post-GELU input is the heavy-tailed one) in W4A8.
# STACK_480P: two experts of 40 blocks each, all weights resident in MXFP4, at 480p /
# 81 frames, with n_w4a8 random blocks per expert promoted to W4A8; the per-linear inputs
# are fixed buffers (attention and norms are not part of the path).
BLOCK_720P = dict(M=TOKENS_720P, ctx=CTX, seed=40)
BLOCK_MASKS = {"all_w4a4": 0x00, "all_w4a8": 0xFF, "mixed_ffn_down_w4a8": 0x80}
STACK_480P = dict(M=TOKENS_480P, ctx=CTX, n_experts=2, n_blocks=40, n_w4a8=8, seed=50)


def stack_block_seed(expert: int, block: int, base: int = STACK_480P["seed"]) -> int:
    """Seed of block `block` of expert `expert` in the two-expert stack."""
    return base * 1000 + expert * 100 + block


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def outlier_channels(K: int, n: int, seed: int) -> torch.Tensor:
    """n distinct K-indices drawn without replacement (CPU generator, any device)."""
    g = _gen(seed * 7919 + 17, "cpu")
    return torch.randperm(K, generator=g)[:n]


def activation(M: int, K: int, kind: str = "normal", seed: int = 0, device="cpu",
               n_outlier: int | None = None, outlier_frac: float = 0.0,
               outlier_scale: float = 30.0, chunk_rows: int = 8192) -> torch.Tensor:
    """bf16 [M, K] activation.  kind: "normal", "student_t" (nu=4) or "gelu"."""
    if n_outlier is None:
        n_outlier = int(round(outlier_frac * K))
    cols = outlier_channels(K, n_outlier, seed).to(device) if n_outlier > 0 else None
    out = torch.empty((M, K), dtype=torch.bfloat16, device=device)
    g = _gen(seed, device)
    for r0 in range(0, M, chunk_rows):
        r1 = min(M, r0 + chunk_rows)
        z = torch.randn((r1 - r0, K), generator=g, device=device, dtype=torch.float32)
        if kind == "student_t":
            chi2 = torch.zeros_like(z)
            for _ in range(4):
                chi2 += torch.randn(z.shape, generator=g, device=device, dtype=torch.float32) ** 2
            z = z / torch.sqrt(chi2 / 4.0)
        elif kind == "gelu":
            z = torch.nn.functional.gelu(z, approximate="none")
        elif kind != "normal":
            raise ValueError(kind)
        if cols is not None:
            z[:, cols] *= outlier_scale
        out[r0:r1] = z.to(torch.bfloat16)
    return out


def weight(N: int, K: int, seed: int = 0, device="cpu", std: float = 0.02) -> torch.Tensor:
    """bf16 [N, K] weight ~ N(0, std^2)."""
    g = _gen(seed + 1_000_003, device)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * std
    return w.to(torch.bfloat16)


def bias(N: int, seed: int = 0, device="cpu", std: float = 0.1) -> torch.Tensor:
    g = _gen(seed + 2_000_029, device)
    return (torch.randn((N,), generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def workload(name: str, device="cpu", with_bias: bool = False, M: int | None = None):
    """The inputs of a named workload: dict(x, w, bias, fmt, M, K, N)."""
    c = dict(WORKLOADS[name])
    if M is not None:
        c["M"] = M
    x = activation(c["M"], c["K"], c["act"], seed=c["seed"], device=device,
                   n_outlier=c.get("n_outlier"), outlier_frac=c.get("outlier_frac", 0.0),
                   outlier_scale=c["outlier_scale"])
    w = weight(c["N"], c["K"], seed=c["seed"], device=device)
    b = bias(c["N"], seed=c["seed"], device=device) if with_bias else None
    return dict(x=x, w=w, bias=b, fmt=c["fmt"], M=c["M"], K=c["K"], N=c["N"])


def block_inputs(M: int, seed: int, device="cpu", ctx: int = CTX):
    """Per-linear inputs of one DiT block: N(0,1) with 1% outlier channels x30,
    except the FFN-down input, which is GELU(N(0,1)) with 1% channels x50."""
    xs = []
    for i, (name, N, K, src) in enumerate(BLOCK_LINEARS):
        rows = M if src == "x" else ctx
        if name == "ffn_down":
            xs.append(activation(rows, K, "gelu", seed=seed * 100 + i, device=device,
                                 outlier_frac=0.01, outlier_scale=50.0))
        else:
            xs.append(activation(rows, K, "normal", seed=seed * 100 + i, device=device,
                                 outlier_frac=0.01, outlier_scale=30.0))
    return xs


def block_weights(seed: int, device="cpu", with_bias: bool = True):
    ws, bs = [], []
    for i, (name, N, K, src) in enumerate(BLOCK_LINEARS):
        ws.append(weight(N, K, seed=seed * 100 + i, device=device))
        bs.append(bias(N, seed=seed * 100 + i, device=device) if with_bias else None)
    return ws, bs


def expert_masks(n_experts: int = 2, n_blocks: int = 40, n_w4a8: int = 8, seed: int = 4):
    """uint8 [n_experts, n_blocks]: n_w4a8 random blocks per expert set to 1 (W4A8)."""
    g = _gen(seed, "cpu")
    mask = torch.zeros((n_experts, n_blocks), dtype=torch.uint8)
    for e in range(n_experts):
        mask[e, torch.randperm(n_blocks, generator=g)[:n_w4a8]] = 1
    return mask


def block_flops(M: int, ctx: int = CTX) -> float:
    total = 0.0
    for name, N, K, src in BLOCK_LINEARS:
        rows = M if src == "x" else ctx
        total += 2.0 * rows * N * K
    return total


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")


def sample_rows(M: int, seed: int = 0, tile: int = 128) -> torch.Tensor:
    """Row 0, row M-1 and one random row inside every `tile`-row M-tile."""
    g = _gen(seed + 31, "cpu")
    rows = {0, M - 1}
    for t0 in range(0, M, tile):
        span = min(tile, M - t0)
        rows.add(t0 + int(torch.randint(span, (1,), generator=g)))
    return torch.tensor(sorted(rows), dtype=torch.int64)



def lowrank_weight(N: int, K: int, rank: int, seed: int = 0, device="cpu", std: float = 0.02,
                   lr_scale: float = 4.0):
    """A weight with a dominant rank-`rank` part, returned already split as the SVDQuant
    branch uses it: l1t [rank, K] and l2t [N, rank] (bf16) with l2t . l1t of entry std
    about lr_scale * std, and a residual [N, K] ~ N(0, std^2) (bf16); W = l2t . l1t + residual."""
    g = _gen(seed + 3_000_017, device)
    s = (lr_scale * std / rank ** 0.5) ** 0.5
    l1t = (torch.randn((rank, K), generator=g, device=device, dtype=torch.float32) * s).to(torch.bfloat16)
    l2t = (torch.randn((N, rank), generator=g, device=device, dtype=torch.float32) * s).to(torch.bfloat16)
    residual = (torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)
    return l1t, l2t, residual
