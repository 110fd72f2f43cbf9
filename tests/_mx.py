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


def tiled_to_logical(tiled: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Tiled scale bytes -> logical [rows, K/32], through the oracle's (pinned) layout: the
    oracle scatters the 1-based logical index of every scale, one byte plane at a time."""
    KB = K // 32
    idx = np.arange(1, rows * KB + 1, dtype=np.int64)
    where = np.zeros(oracle.sf_tiled_bytes(rows, K), dtype=np.int64)
    for plane in range(4):
        b = ((idx >> (8 * plane)) & 0xFF).astype(np.uint8).reshape(rows, KB)
        where |= oracle.sf_to_tiled(b, K).astype(np.int64) << (8 * plane)
    out = np.zeros(rows * KB, dtype=np.uint8)
    live = where > 0
    out[where[live] - 1] = np.asarray(tiled)[: where.size][live]
    return out.reshape(rows, KB)


def unpack_codes(codes: np.ndarray, rows: int, K: int, fmt: str) -> np.ndarray:
    """Packed element codes -> one byte per element [rows, K]."""
    c = np.asarray(codes).reshape(-1)
    if fmt == "e4m3":
        return c[: rows * K].reshape(rows, K)
    c = c[: rows * K // 2]
    return np.stack([c & 0xF, c >> 4], axis=-1).reshape(rows, K)


_DECODE = {}


def decode_table(fmt: str) -> np.ndarray:
    """Values of every element code of the format (oracle.decode_elem), indexed by code."""
    if fmt not in _DECODE:
        n = 256 if fmt == "e4m3" else 16
        _DECODE[fmt] = np.array([oracle.decode_elem(c, FMT[fmt]) for c in range(n)], dtype=np.float64)
    return _DECODE[fmt]


# Share of the elements a binary32 evaluation of the transform may round either way: the
# error bound is a fixed fraction of the rotation block's L1 norm, so the finer E4M3 grid
# (three mantissa bits) leaves more elements within it than E2M1's.
UNCERTAIN_LIMIT = {"e2m1": 1e-3, "e4m3": 5e-3}


def check_transformed(codes_gpu, sf_gpu, rows: int, K: int, fmt: str, ref: dict, what: str,
                      max_uncertain: float | None | str = "default"):
    """The transform_on quantizer against the oracle's definition (oracle.quantize_transformed):
      * every block whose scale the oracle reports certain has the definition's scale, and on
        it every element whose code is certain has the definition's code, bit for bit;
      * the other elements of such blocks (within a binary32 error bound of a decision
        boundary) have a code whose value lies between the values of the two codes the
        oracle reports for the ends of that bound (on E4M3's fine grid the bound can span
        more than two codes);
      * a block reported uncertain has a scale at most one away (or 255 where binary32 may
        overflow);
      * at most max_uncertain of the elements are uncertain (the format's UNCERTAIN_LIMIT by
        default; None: no limit).
    Returns the number of uncertain elements."""
    if max_uncertain == "default":
        max_uncertain = UNCERTAIN_LIMIT[fmt]
    sf_np = sf_gpu.cpu().numpy() if hasattr(sf_gpu, "cpu") else sf_gpu
    # scales in the tiled layout, or already logical [rows, K / 32] (a row subset)
    sf_l = sf_np if sf_np.ndim == 2 else tiled_to_logical(sf_np, rows, K)
    cg = unpack_codes(codes_gpu.cpu().numpy() if hasattr(codes_gpu, "cpu") else codes_gpu, rows, K, fmt)
    cd = unpack_codes(ref["codes"], rows, K, fmt)
    amb = ref["blk_amb"]
    sure = amb == 0
    bad = np.nonzero(sure & (sf_l != ref["sf"]))
    assert bad[0].size == 0, "%s: %d certain scales differ, first (%d, %d): gpu %d oracle %d" % (
        what, bad[0].size, bad[0][0], bad[1][0], sf_l[bad][0], ref["sf"][bad][0])
    d = np.abs(sf_l.astype(int) - ref["sf"].astype(int))
    unsure_ok = (d <= 1) | ((amb == 2) & (sf_l == 255))
    assert unsure_ok[~sure].all(), what + ": an uncertain block's scale is off by more than one"
    blk_sure = np.repeat(sure, 32, axis=1)
    certain = blk_sure & (ref["code_lo"] == ref["code_hi"])
    bad = np.nonzero(certain & (cg != cd))
    assert bad[0].size == 0, "%s: %d certain codes differ, first (%d, %d): gpu %#x oracle %#x" % (
        what, bad[0].size, bad[0][0], bad[1][0], cg[bad][0], cd[bad][0])
    unc = blk_sure & ~certain
    tab = decode_table(fmt)
    vg, vlo, vhi = tab[cg[unc]], tab[ref["code_lo"][unc]], tab[ref["code_hi"][unc]]
    ok = (np.minimum(vlo, vhi) <= vg) & (vg <= np.maximum(vlo, vhi))
    assert ok.all(), what + ": an uncertain code lies outside its two candidates"
    n_unc = int(unc.sum())
    if max_uncertain is not None:
        assert n_unc <= max_uncertain * cg.size, "%s: %d uncertain elements" % (what, n_unc)
    return n_unc
