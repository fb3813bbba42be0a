"""Property-based pins of the oracle (hypothesis): random and adversarial groups
(ties, extreme magnitudes, zeros, constant runs) checked against properties that
the definitions fix, independently of how the oracle computes them.

- affine: codes within [0, 2^bits - 1], code 0 at the group minimum and the top
  code at the maximum (non-degenerate groups), and |w - w'| <= scale16 *
  (1/2 + 2^(bits-23)) (round to nearest on the stored grid);
- mxfp4 / mxfp8: every code is the nearest of all representable signed values at
  the group's scale (brute force), and max|w| / X lies in the format's window;
- nvfp4: every block scale is the E4M3 value nearest to amax / (6 g), every code
  the nearest E2M1 value at that scale;
- range search: the chosen grid's squared error is never above round-to-nearest's.
"""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from pins import E2M1_VALUES, affine_values_f64, bitwise_unpack, e4m3_all_values, group_sq_error_f64

SETTINGS = settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])


def _f32(x):
    return float(np.float32(x))


def group_values(n, max_mag):
    """n float32 values: a mix of normal draws, exact grid points, repeats, zeros and signs."""
    m = _f32(max_mag)
    finite = st.floats(min_value=-m, max_value=m, allow_nan=False, allow_infinity=False, width=32)
    special = st.sampled_from([0.0, -0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, 448.0, 464.0, 1e-30, -1e-30])
    return st.lists(st.one_of(finite, special), min_size=n, max_size=n).map(
        lambda v: np.array(v, dtype=np.float32))


@SETTINGS
@given(st.sampled_from([2, 3, 4, 8]), st.sampled_from([32, 64]), st.data())
def test_affine_codes_range_extremes_and_error_bound(bits, G, data):
    w = data.draw(group_values(G, 3.0e4))[None, :]
    p, s, b = oracle.quantize(w, G, bits)
    q = oracle.unpack_codes(p, G, bits)[0].astype(np.int64)
    qmax = (1 << bits) - 1
    assert q.min() >= 0 and q.max() <= qmax
    s16 = float(s.view(np.float16)[0, 0])
    if s16 > 0:
        assert q[int(np.argmin(w[0]))] == 0
        # the maximum lands on the top code unless fp16 rounding of the scale pulled it below
        wq = affine_values_f64(q[None, :], s, b, G)[0]
        err = np.abs(w[0].astype(np.float64) - wq)
        inside = w[0].astype(np.float64) <= float(b.view(np.float16)[0, 0]) + qmax * s16
        assert (err[inside] <= s16 * (0.5 + 2.0 ** (bits - 23)) + 1e-300).all()
    else:
        assert (q == 0).all()


@SETTINGS
@given(st.data())
def test_mxfp4_codes_are_nearest(data):
    w = data.draw(group_values(32, 1.0e30))[None, :]
    p, s = oracle.mxfp4_quantize(w)
    codes = oracle.unpack_codes(p, 32, 4)[0].astype(np.int64)
    X = np.ldexp(1.0, int(s[0, 0]) - 127)
    v = w[0].astype(np.float64)
    chosen = np.abs(v - E2M1_VALUES[codes] * X)
    assert (chosen <= np.abs(v[:, None] - E2M1_VALUES[None, :] * X).min(axis=1)).all()
    amax = np.abs(v).max()
    if amax > 0 and s[0, 0] > 0:
        assert 4.0 <= amax / X < 8.0


@SETTINGS
@given(st.data())
def test_mxfp8_codes_are_nearest(data):
    w = data.draw(group_values(32, 1.0e30))[None, :]
    p, s = oracle.mxfp8_quantize(w)
    codes = oracle.unpack_codes(p, 32, 8)[0].astype(np.int64)
    X = np.ldexp(1.0, int(s[0, 0]) - 127)
    mags = e4m3_all_values()
    allv = np.concatenate([mags, -mags])
    v = w[0].astype(np.float64)
    val = np.where(codes & 0x80, -mags[codes & 0x7F], mags[codes & 0x7F]) * X
    assert (np.abs(v - val) <= np.abs(v[:, None] - allv[None, :] * X).min(axis=1)).all()
    assert not (codes == 0x80).any()


@SETTINGS
@given(st.data())
def test_nvfp4_scales_and_codes_are_nearest(data):
    w = data.draw(group_values(64, 1.0e4))[None, :]
    p, s, g = oracle.nvfp4_quantize(w)
    mags = e4m3_all_values()
    amax_b = np.abs(w[0].reshape(4, 16)).max(axis=1)
    six_g = np.float32(6.0) * np.float32(g)
    for blk in range(4):
        target = float(np.float32(amax_b[blk]) / six_g)
        sv = mags[int(s[0, blk])]
        assert abs(target - sv) <= np.abs(target - mags).min()
    codes = oracle.unpack_codes(p, 64, 4)[0].astype(np.int64)
    for blk in range(4):
        sv = mags[int(s[0, blk])]
        if sv == 0:
            assert (codes[16 * blk:16 * blk + 16] == 0).all()
            continue
        denom = float(np.float32(np.float32(sv) * np.float32(g)))
        t = np.abs(w[0, 16 * blk:16 * blk + 16].astype(np.float32)) / np.float32(denom)
        mag = E2M1_VALUES[codes[16 * blk:16 * blk + 16] & 7]
        assert (np.abs(t.astype(np.float64) - mag) <= np.abs(t[:, None].astype(np.float64) - E2M1_VALUES[None, :8]).min(axis=1)).all()


@SETTINGS
@given(st.sampled_from([2, 3, 4]), st.data())
def test_range_search_never_worse_than_round_to_nearest(bits, data):
    w = data.draw(group_values(64, 100.0))[None, :]
    pm, sm, bm = oracle.quantize_mse(w, 64, bits)
    p0, s0, b0 = oracle.quantize(w, 64, bits)
    em = group_sq_error_f64(w, bitwise_unpack(pm, 64, bits), sm, bm, 64)
    e0 = group_sq_error_f64(w, bitwise_unpack(p0, 64, bits), s0, b0, 64)
    assert (em <= e0 * (1 + 2e-5) + 1e-30).all()
