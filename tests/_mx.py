"""Helpers shared by the GPU parity tests: run the CPU oracle on the exact bytes the
GPU path consumed, and apply the acceptance bounds of the GEMM."""
import numpy as np
import torch

import oracle

FMT = {"e2m1": oracle.E2M1, "e4m3": oracle.E4M3}

# GEMM acceptance: relative Frobenius error <= 2e-3, and per output row
# max |y - y_ref| <= 1e-2 * max |y_ref| (the row's infinity norm).  The Frobenius
# bound is a statistical one: bf16 round-to-nearest-even alone has a relative error
# of up to 2^-8 per element, so an output of a handful of elements can exceed 2e-3
# even when every element is correctly rounded.  Outputs with fewer than
# SMALL_OUTPUT elements are held instead to a per-element bound: the bf16 unit
# roundoff of the reference value plus a small fp32-accumulation allowance.
REL_FRO = 2e-3
ROW_INF = 1e-2
SMALL_OUTPUT = 4096
BF16_U = 2.0 ** -8


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_quantize(x: torch.Tensor, fmt: str):
    """(codes, logical scales, tiled scales) from the oracle for the bf16 tensor x."""
    xb = bits(x)
    codes, sf = oracle.quantize(xb, FMT[fmt])
    return codes, sf, oracle.sf_to_tiled(sf, xb.shape[1])


def assert_gemm_close(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = ""):
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    assert np.isfinite(y_gpu).all(), what + ": non-finite output"
    diff = y_gpu - y_ref
    fro = np.linalg.norm(diff) / max(np.linalg.norm(y_ref), 1e-300)
    if y_ref.size >= SMALL_OUTPUT:
        assert fro <= REL_FRO, "%s: relative Frobenius error %.3e > %.1e" % (what, fro, REL_FRO)
    else:
        lim = BF16_U * np.abs(y_ref) + 1e-6 * np.abs(y_ref).max()
        bad = np.nonzero(np.abs(diff) > lim)
        assert bad[0].size == 0, "%s: element %s off by %.3e (bound %.3e)" % (
            what, tuple(int(b[0]) for b in bad), np.abs(diff)[bad][0], lim[bad][0])
    row_err = np.abs(diff).max(axis=1)
    row_inf = np.abs(y_ref).max(axis=1)
    bad = np.nonzero(row_err > ROW_INF * row_inf)[0]
    assert bad.size == 0, "%s: %d rows exceed the row bound, first %d: err %.3e vs inf-norm %.3e" % (
        what, bad.size, bad[0], row_err[bad[0]], row_inf[bad[0]])
    return fro


def sqnr_db(y_ref: np.ndarray, y: np.ndarray) -> float:
    return 10.0 * np.log10(np.sum(y_ref ** 2) / max(np.sum((y_ref - y) ** 2), 1e-300))
