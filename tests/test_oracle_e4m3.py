"""Pins of the oracle's e4m3 codec (OCP FP8 E4M3) and of its per-token
fp8 quantisation of cache rows."""
import numpy as np
import pytest
import torch

import oracle
from oracle import mla as om


def _spec_value(code: int) -> float:
    """Value of one code straight from the format definition (scalar, by hand)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def test_decode_all_codes_match_definition():
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_decode(codes)
    for c in range(256):
        ref = _spec_value(c)
        if np.isnan(ref):
            assert np.isnan(v[c])
        else:
            assert v[c] == ref
    assert np.nanmax(v) == 448.0 and np.nanmin(v) == -448.0
    assert v[1] == 2.0 ** -9          # smallest subnormal


def test_encode_roundtrip_every_finite_code():
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_decode(codes)
    fin = ~np.isnan(v)
    back = oracle.e4m3_encode(v[fin].astype(np.float32))
    # +0 and -0 both encode to their own sign
    np.testing.assert_array_equal(back, codes[fin])


def test_encode_ties_to_even_and_saturation():
    enc = lambda x: int(oracle.e4m3_encode(np.array([x], np.float32))[0])
    # between 1.0 (0x38) and 1.125 (0x39): midpoint 1.0625 -> even mantissa 0x38
    assert enc(1.0625) == 0x38
    # between 1.125 (0x39) and 1.25 (0x3A): midpoint 1.1875 -> 0x3A (even)
    assert enc(1.1875) == 0x3A
    assert enc(1.0626) == 0x39
    # subnormal midpoint: 1.5 * 2^-9 between codes 1 and 2 -> 2
    assert enc(1.5 * 2.0 ** -9) == 0x02
    assert enc(0.5 * 2.0 ** -9) == 0x00          # ties to even -> zero
    # saturation: anything at or above 448 in magnitude becomes +-448
    for x in (448.0, 460.0, 470.0, 1e6, np.inf):
        assert enc(x) == 0x7E
        assert enc(-x) == 0xFE
    assert enc(np.nan) == 0x7F


def test_encode_matches_torch_float8_in_range():
    """torch's CPU float8_e4m3fn conversion (round to nearest even) is a library
    reference for every input whose magnitude stays below the saturation point."""
    rng = np.random.default_rng(0)
    x = rng.standard_normal(400000).astype(np.float32) * np.exp2(rng.uniform(-12, 9, 400000)).astype(np.float32)
    x = x[np.abs(x) < 448.0]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(x), ref)


def test_fp8_quantize_row_error_bound_and_scale():
    rng = np.random.default_rng(1)
    rows = rng.standard_normal((500, 576)).astype(np.float32)
    rows[3] = 0.0
    codes, scale = om.fp8_quantize_row(rows)
    assert codes.dtype == np.uint8 and scale.dtype == np.float32
    assert scale[3] == 1.0 and np.all(codes[3] == 0)
    amax = np.abs(rows).max(1)
    nz = amax > 0
    np.testing.assert_array_equal(scale[nz], (amax[nz] / np.float32(448.0)).astype(np.float32))
    deq = oracle.e4m3_decode(codes) * scale[:, None].astype(np.float64)
    # round-trip error of each element <= half an e4m3 step at its magnitude, times scale
    scaled = rows.astype(np.float64) / scale[:, None]
    _, k = np.frexp(np.where(scaled != 0, np.abs(scaled), 1.0))
    step = np.ldexp(1.0, np.maximum(k - 1, -6) - 3)
    bound = 0.5 * step * scale[:, None] * (1 + 1e-6) + 1e-30
    assert np.all(np.abs(deq - rows) <= bound)
    # the row maximum maps to +-448 exactly
    imax = np.abs(rows[nz]).argmax(1)
    assert np.all(np.abs(oracle.e4m3_decode(codes[nz][np.arange(nz.sum()), imax])) == 448.0)
