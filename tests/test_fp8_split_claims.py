"""The number-format facts the FP8 decode kernel relies on, checked
exhaustively on the CPU with the oracle's e4m3 encoder and decoder (OCP E4M3
as the pages' knob 4 names it):

- a bf16 query element scaled by a power of two into [2^-2, 256) is exactly
  hi + lo with hi = e4m3(x) and lo = e4m3(x - hi);
- smaller elements (below 2^-10 of a head maximum in [128, 256)) lose at
  most 2^-10 absolute, i.e. under 2^-17 of that maximum;
- an f16 probability in [0, 256] split the same way keeps 8 significant
  bits: |p - hi - lo| <= 2^-8 |p| + 2^-10;
- every e4m3 value is exact in f16, so the f16 residual p - hi is exact."""
import numpy as np

import oracle
import synth


def _split(x32):
    hi = oracle.e4m3_from_float32(x32)
    hv = oracle.e4m3_to_float64(hi)
    r = (x32.astype(np.float64) - hv).astype(np.float32)
    lo = oracle.e4m3_from_float32(r)
    return hv, oracle.e4m3_to_float64(lo)


def _all_bf16_in(lo, hi):
    bits = np.arange(0, 0x8000, dtype=np.uint32)  # non-negative bf16 patterns
    vals = synth.bf16_bits_to_f32(bits.astype(np.uint16))
    sel = np.isfinite(vals) & (vals >= lo) & (vals < hi)
    v = vals[sel]
    return np.concatenate([v, -v]).astype(np.float32)


def test_bf16_query_split_is_exact_in_range():
    x = _all_bf16_in(2.0 ** -2, 256.0)
    hv, lv = _split(x)
    assert np.array_equal(hv + lv, x.astype(np.float64))


def test_small_query_elements_lose_under_2_to_minus_10():
    x = _all_bf16_in(2.0 ** -40, 2.0 ** -2)
    hv, lv = _split(x)
    assert np.max(np.abs(hv + lv - x.astype(np.float64))) <= 2.0 ** -10


def test_probability_split_keeps_8_bits():
    # every positive f16 value up to 256 (the kernel forms p = 256 * 2^(x - m))
    bits = np.arange(1, 0x5C01, dtype=np.uint16)
    p = bits.view(np.float16).astype(np.float32)
    p = p[np.isfinite(p) & (p <= 256.0)]
    hv, lv = _split(p)
    err = np.abs(hv + lv - p.astype(np.float64))
    assert np.all(err <= 2.0 ** -8 * p + 2.0 ** -10)


def test_e4m3_values_and_residuals_are_exact_in_f16():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    v = oracle.e4m3_to_float64(codes)
    assert np.array_equal(v.astype(np.float16).astype(np.float64), v)
    # residual of rounding an f16 to e4m3 is representable in f16
    bits = np.arange(1, 0x5C01, dtype=np.uint16)
    p = bits.view(np.float16).astype(np.float64)
    p = p[np.isfinite(p) & (p <= 256.0)]
    hi = oracle.e4m3_to_float64(oracle.e4m3_from_float32(p.astype(np.float32)))
    r = p - hi
    assert np.array_equal(r.astype(np.float16).astype(np.float64), r)
