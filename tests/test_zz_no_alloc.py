"""mxq_linear_noalloc: the native linear for callers that cannot allocate device memory
where they run a layer (for example under a memory manager that owns the device pool, or
in a plugin handed only its input and output buffers).  Its scratch is a fixed static
device array, so these tests check, through the C ABI, that it gives bit for bit the
result of mxq_linear with a caller workspace on two calls in a row (the second call
reuses the array the first one left behind), that the result is the oracle's linear
within the GEMM tolerance, that the largest inputs the array holds work and the next
larger ones are refused."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _mx

pytestmark = pytest.mark.gpu


def _abi():
    from fp8_mixed_precision_mxq_b200 import _lib
    return _lib


def _call_noalloc(L, x, qw, fmt, y):
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(0 if t is None else t.data_ptr())  # noqa: E731
    return L.mxq_linear_noalloc(p(x), x.shape[0], x.shape[1], p(qw.codes), p(qw.sf), qw.N, p(qw.bias),
                                0 if fmt == "e2m1" else 1, p(y), st)


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_noalloc_matches_workspace_linear_on_two_calls(fmt):
    from fp8_mixed_precision_mxq_b200 import ops
    lib = _abi()
    L = lib.lib()
    M, N, K = 1000, 1288, 2048
    w = synth.weight(N, K, seed=41, device="cuda")
    b = synth.bias(N, seed=41, device="cuda")
    qw = ops.quantize_weight(w, bias=b)
    wc, ws, _ = _mx.oracle_quantize(w, "e2m1")
    for call, seed in enumerate((42, 43)):
        x = synth.activation(M, K, "student_t" if fmt == "e2m1" else "gelu", seed=seed, device="cuda",
                             outlier_frac=0.02, outlier_scale=40.0)
        y_ref = ops.linear(x, qw, fmt=fmt)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = _call_noalloc(L, x, qw, fmt, y)
        assert rc == lib.OK, lib.last_error()
        assert ops.poll_status() == 0
        # the same kernels on the same bytes: identical output
        assert torch.equal(y, y_ref), "noalloc %s call %d differs from mxq_linear" % (fmt, call)
        if call == 0:
            xc, xs, _ = _mx.oracle_quantize(x, fmt)
            rows = np.arange(0, M, 7)
            ref = oracle.linear_rows(xc, xs, _mx.FMT[fmt], rows, K, wc, ws, _mx.bits(b))
            _mx.assert_gemm_close(_mx.bf16_to_f64(y[torch.from_numpy(rows).cuda()]), ref, "noalloc %s" % fmt)


def _largest_rows(ops, K, N, fmt, cap):
    """The largest M whose native workspace fits the static scratch."""
    lo, hi = 1, cap
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if ops.workspace_bytes(mid, N, K, fmt) <= cap:
            lo = mid
        else:
            hi = mid - 1
    return lo


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_noalloc_largest_accepted_input_and_the_next_one(fmt):
    """At the largest M whose scratch fits the array exactly (K = 5120) the entry point runs
    and equals mxq_linear bit for bit; M + 1 needs more and is refused with nothing
    launched.  The header's limits (about 63 M elements of M*K for E2M1, 32 M for E4M3)
    follow from it."""
    from fp8_mixed_precision_mxq_b200 import ops
    lib = _abi()
    L = lib.lib()
    cap = L.mxq_linear_noalloc_max_scratch_bytes()
    K, N = 5120, 256
    M = _largest_rows(ops, K, N, fmt, cap)
    assert ops.workspace_bytes(M, N, K, fmt) <= cap < ops.workspace_bytes(M + 1, N, K, fmt)
    limit = 63e6 if fmt == "e2m1" else 32e6
    assert abs(M * K - limit) < 0.05 * limit, M * K
    qw = ops.quantize_weight(synth.weight(N, K, seed=2, device="cuda"), bias=synth.bias(N, seed=2, device="cuda"))
    x = synth.activation(M + 1, K, "normal", seed=3, device="cuda", outlier_frac=0.01, outlier_scale=30.0)
    xm = x[:M]
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(L, xm, qw, fmt, y) == lib.OK, lib.last_error()
    assert torch.equal(y, ops.linear(xm, qw, fmt=fmt))
    y1 = torch.zeros((M + 1, N), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(L, x, qw, fmt, y1) == lib.ERR_WORKSPACE
    assert "static scratch" in lib.last_error()
    torch.cuda.synchronize()
    assert not y1.any()  # nothing was launched
