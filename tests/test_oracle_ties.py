"""Pins of the oracle's rounding-tie bands.

A code mismatch between the kernels and the oracle is excused only where the
oracle flags a tie: the exact value lies within a relative 2^-15 of a rounding
midpoint (k + 1/2 for the integer codes, the midpoint between two adjacent
fp16 values for the KV4 scale and zero).  A band that is too wide would hide
real mismatches, one that is too narrow or off-centre would fail honest fp32
results, so both edges are pinned here from the definitions, on hand-picked
values.
"""

import numpy as np

from oracle import quant

EPS = 2.0 ** -15


def test_tie_band_width_is_2_to_minus_15():
    assert quant.TIE_EPS == EPS


def test_near_half_at_and_around_midpoints():
    mids = np.array([0.5, 1.5, 2.5, -0.5, -3.5, 6.5, 14.5])
    assert quant._near_half(mids).all()
    # inside the band (relative to max(1, |v|)), on both sides
    inside = np.concatenate([mids + 0.9 * EPS * np.maximum(1, np.abs(mids)),
                             mids - 0.9 * EPS * np.maximum(1, np.abs(mids))])
    assert quant._near_half(inside).all()
    # just outside it
    outside = np.concatenate([mids + 1.1 * EPS * np.maximum(1, np.abs(mids)),
                              mids - 1.1 * EPS * np.maximum(1, np.abs(mids))])
    assert not quant._near_half(outside).any()


def test_near_half_not_at_integers_or_quarters():
    v = np.array([0.0, 1.0, -2.0, 7.0, 0.25, 0.75, -1.25, 3.3])
    assert not quant._near_half(v).any()


def test_near_half_band_is_absolute_below_one():
    # below |v| = 1 the band is eps wide in absolute terms, not eps * |v|
    assert quant._near_half(np.array([0.5 + 0.9 * EPS]))[0]
    assert not quant._near_half(np.array([0.5 + 1.1 * EPS]))[0]


def _fp16_mid(a):
    """Midpoint between fp16 value a and the next fp16 value above it."""
    h = np.float16(a)
    up = np.nextafter(h, np.float16(np.inf))
    return 0.5 * (float(h) + float(up))


def test_fp16_tie_at_midpoints():
    for a in (1.0, 0.1, 3.0, 1000.0, 2.0 ** -10, -5.5):
        m = _fp16_mid(a)
        assert quant._fp16_tie(np.array([m]))[0], a
        assert quant._fp16_tie(np.array([m * (1 + 0.5 * EPS)]))[0], a
        assert not quant._fp16_tie(np.array([m * (1 + 4 * EPS)]))[0], a


def test_fp16_tie_not_at_representable_values():
    v = np.array([1.0, 0.5, 2.0 ** -14, 1000.0, -3.0, float(np.float16(0.1))])
    assert not quant._fp16_tie(v).any()


def test_fp16_tie_floor_below_the_subnormals():
    # the band never shrinks below 2^-24 * eps in absolute terms, so a value
    # next to zero is only a tie near the first subnormal midpoint
    assert quant._fp16_tie(np.array([2.0 ** -25]))[0]          # midpoint of 0 and 2^-24
    assert not quant._fp16_tie(np.array([2.0 ** -26]))[0]
