"""mxq_linear_noalloc: the native linear for callers that cannot allocate device memory
where they run a layer (for example under a memory manager that owns the device pool, or
in a plugin handed only its input and output buffers).  Its scratch is a fixed static
device array, so these tests check, through the C ABI, that it gives the same result as
mxq_linear with a caller workspace on two calls in a row (the second call reuses the
array the first one left behind), and that inputs too large for the array are refused."""
import ctypes

import numpy as np
import pytest
import torch

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
    qw = ops.quantize_weight(w, bias=synth.bias(N, seed=41, device="cuda"))
    for call, seed in enumerate((42, 43)):
        x = synth.activation(M, K, "student_t" if fmt == "e2m1" else "gelu", seed=seed, device="cuda",
                             outlier_frac=0.02, outlier_scale=40.0)
        y_ref = ops.linear(x, qw, fmt=fmt)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = _call_noalloc(L, x, qw, fmt, y)
        assert rc == lib.OK, lib.last_error()
        assert ops.poll_status() == 0
        _mx.assert_gemm_close(_mx.bf16_to_f64(y), _mx.bf16_to_f64(y_ref), "noalloc %s call %d" % (fmt, call))


def test_noalloc_rejects_inputs_beyond_the_static_scratch():
    from fp8_mixed_precision_mxq_b200 import ops
    lib = _abi()
    L = lib.lib()
    cap = L.mxq_linear_noalloc_max_scratch_bytes()
    assert cap > 0
    K, N = 5120, 256
    M = int(cap // K) + 256  # E4M3 needs a little over M*K bytes: beyond the array
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    qw = ops.quantize_weight(synth.weight(N, K, seed=1, device="cuda"))
    y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    rc = _call_noalloc(L, x, qw, "e4m3", y)
    assert rc == lib.ERR_WORKSPACE
    assert "static scratch" in lib.last_error()
    torch.cuda.synchronize()
    assert not y.any()  # nothing was launched
