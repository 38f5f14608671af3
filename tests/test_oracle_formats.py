"""Pins for the oracle's E2M1 / E4M3 / fp16 handling (CPU only).

Against hand-written tables from the format definitions (tests/golden) and
against PyTorch's float8_e4m3fn and float16 conversions (library routines).
"""

import numpy as np
import torch

from oracle import formats


def test_e2m1_grid_golden(golden):
    for line in golden("e2m1_grid.txt"):
        code, val = line.split()
        assert formats.e2m1_decode(int(code)) == float(val)
    mags = sorted({abs(formats.e2m1_decode(c)) for c in range(16)})
    assert mags == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e2m1_rounding_golden(golden):
    for line in golden("e2m1_rounding.txt"):
        v, code = line.split()
        got, _ = formats.e2m1_round(np.array([float(v)]))
        assert int(got[0]) == int(code), (v, code, got)


def test_e4m3_points_golden(golden):
    for line in golden("e4m3_points.txt"):
        code, val = line.split()
        got = formats.e4m3_decode(int(code, 16))
        if val == "nan":
            assert np.isnan(got)
        else:
            assert got == float(val)


def test_e4m3_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([formats.e4m3_decode(c) for c in range(256)])
    both_nan = np.isnan(ref) & np.isnan(mine)
    assert np.all(both_nan | (ref == mine))


def test_e4m3_rounding_matches_torch_in_range():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 20000)),
        formats.E4M3_POS_VALUES,
        0.5 * (formats.E4M3_POS_VALUES[1:] + formats.E4M3_POS_VALUES[:-1]),   # exact midpoints
    ])
    vals = vals[vals <= 448.0]
    mine, _ = formats.e4m3_round_unsigned(vals)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int64)
    assert np.array_equal(mine, ref)


def test_e4m3_saturates():
    codes, _ = formats.e4m3_round_unsigned(np.array([448.0, 465.0, 1e6]))
    assert list(codes) == [0x7E, 0x7E, 0x7E]


def test_fp16_matches_torch():
    """On fp32-representable inputs torch's float16 cast is a single RNE rounding."""
    rng = np.random.default_rng(2)
    v = (rng.standard_normal(10000) * 10.0 ** rng.integers(-6, 4, 10000)).astype(np.float32).astype(np.float64)
    v = np.concatenate([v, [1 + 2 ** -11, 1 + 3 * 2 ** -11, 2049.0, 2051.0, 65504.0]])
    ref = torch.from_numpy(v).to(torch.float16).to(torch.float64).numpy()
    assert np.array_equal(formats.to_fp16(v), ref)


def test_fp16_rounds_fp64_directly():
    """fp64 -> fp16 in one rounding: just above a midpoint goes up (no double rounding)."""
    assert formats.to_fp16(np.array([1 + 2 ** -11 + 2 ** -40]))[0] == 1 + 2 ** -10
    assert formats.to_fp16(np.array([1 + 2 ** -11]))[0] == 1.0


def test_e8m0_decode_closed_form():
    # E8M0 (OCP Microscaling shared scale): value 2^(code - 127), code 255 = NaN
    import math
    for c in range(255):
        assert formats.e8m0_decode(c) == math.ldexp(1.0, c - 127)
    assert math.isnan(formats.e8m0_decode(255))
    assert formats.e8m0_decode(127) == 1.0
    v = formats.e8m0_values(np.arange(255))
    assert np.all(v[1:] == 2.0 * v[:-1])
