"""The checking helpers the GPU parity tests use, exercised on the CPU: the tiled-scale
unscrambling and the transform_on checker (which must accept the definition's own output
and reject a wrong certain code or scale planted into it)."""
import numpy as np
import pytest

import oracle
from tests import _mx


@pytest.mark.parametrize("rows,K", [(1, 32), (130, 96), (300, 1024)])
def test_tiled_to_logical_round_trip(rows, K):
    rng = np.random.default_rng(rows + K)
    sf = rng.integers(0, 256, size=(rows, K // 32), dtype=np.uint8)
    assert np.array_equal(_mx.tiled_to_logical(oracle.sf_to_tiled(sf, K), rows, K), sf)


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_check_transformed_accepts_the_definition_and_rejects_slips(fmt):
    rng = np.random.default_rng(3)
    rows, K = 40, 256
    x = (rng.standard_normal((rows, K)) * 3).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    ref = oracle.quantize_transformed(bits, _mx.FMT[fmt], 32)
    tiled = oracle.sf_to_tiled(ref["sf"], K)
    codes = ref["codes"].reshape(-1).copy()
    _mx.check_transformed(codes, tiled, rows, K, fmt, ref, "definition", max_uncertain=None)
    # one certain element changed
    bad = codes.copy()
    bad[7] ^= 0x01
    with pytest.raises(AssertionError):
        _mx.check_transformed(bad, tiled, rows, K, fmt, ref, "slip", max_uncertain=None)
    # one certain scale changed
    sf2 = ref["sf"].copy()
    sf2[3, 2] += 1
    with pytest.raises(AssertionError):
        _mx.check_transformed(codes, oracle.sf_to_tiled(sf2, K), rows, K, fmt, ref, "slip", max_uncertain=None)
