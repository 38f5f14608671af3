"""Oracle: the number formats the pages name, decoded from their definitions.

Test infrastructure only (see ``oracle/__init__.py``).

"Rotations for 4-Bit Activations: QuaRot, SpinQuant, and Friends", section
"What it buys in 4 bits, and what it doesn't": NVFP4 stores E2M1 values ("E2M1's
eight magnitudes") with an FP8 scale for every block of 16 values.  The FP8
scale is E4M3.  The pages give only the format names; the bit layouts below
are the standard ones (OCP Microscaling formats / NVIDIA FP8):

* E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit, no inf/NaN.
  Magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
* E4M3 (fn): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; S.1111.111 is
  NaN; no inf; max finite 448; min subnormal 2^-9.

Rounding, as the reading of the pages' silence: round to nearest, ties to the
even code (the one whose least significant bit is 0), saturating to the largest
finite magnitude (the behaviour of a hardware "rn.satfinite" conversion).
Each rounding is done by an exhaustive nearest search over the decoded grid,
so it does not depend on any bit trick.
"""

import numpy as np


def e2m1_decode(code):
    """Value of a 4-bit E2M1 code (int 0..15)."""
    code = int(code)
    sign = -1.0 if (code >> 3) & 1 else 1.0
    exp = (code >> 1) & 0x3
    man = code & 0x1
    if exp == 0:
        mag = man * 0.5                      # subnormal: 0.m x 2^(1-bias) = m/2
    else:
        mag = (1.0 + man / 2.0) * 2.0 ** (exp - 1)
    return sign * mag


def e4m3_decode(code):
    """Value of an 8-bit E4M3 (fn) code (int 0..255); NaN for S.1111.111."""
    code = int(code)
    sign = -1.0 if (code >> 7) & 1 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return float("nan")
    if exp == 0:
        mag = (man / 8.0) * 2.0 ** (1 - 7)
    else:
        mag = (1.0 + man / 8.0) * 2.0 ** (exp - 7)
    return sign * mag


E2M1_POS_CODES = np.arange(8)
E2M1_POS_VALUES = np.array([e2m1_decode(c) for c in E2M1_POS_CODES])
E2M1_MAX = 6.0

# Finite non-negative E4M3 codes 0x00..0x7E (0x7F is NaN).
E4M3_POS_CODES = np.arange(0x7F)
E4M3_POS_VALUES = np.array([e4m3_decode(c) for c in E4M3_POS_CODES])
E4M3_MAX = 448.0


def _round_to_grid(mag, grid_vals, grid_codes, chunk=1 << 15):
    """Nearest grid point to each non-negative magnitude; ties -> even code;
    beyond the largest grid value -> the largest (saturation).

    Returns (codes, tie_distance) where tie_distance is the distance of the
    input to the nearest midpoint between adjacent grid values (used to flag
    rounding-boundary ties).  Exhaustive search, in chunks to bound memory.
    """
    mag = np.asarray(mag, dtype=np.float64)
    flat = mag.reshape(-1)
    codes = np.empty(flat.shape, dtype=np.int64)
    tie_dist = np.empty(flat.shape, dtype=np.float64)
    mids = 0.5 * (grid_vals[1:] + grid_vals[:-1])
    even = (grid_codes[None, :] & 1) == 0
    for s in range(0, flat.size, chunk):
        f = flat[s:s + chunk]
        d = np.abs(f[:, None] - grid_vals[None, :])          # [n, G]
        best = d.min(axis=1)
        cand = d == best[:, None]
        pick_even = cand & even          # among equally near codes keep the even one
        has_even = pick_even.any(axis=1)
        idx = np.where(has_even, np.argmax(pick_even, axis=1), np.argmax(cand, axis=1))
        c = grid_codes[idx]
        codes[s:s + chunk] = np.where(f >= grid_vals[-1], grid_codes[-1], c)
        tie_dist[s:s + chunk] = np.abs(f[:, None] - mids[None, :]).min(axis=1)
    return codes.reshape(mag.shape), tie_dist.reshape(mag.shape)


def e2m1_round(v):
    """E2M1 RNE-satfinite codes (int 0..15, sign in bit 3) of real values v.

    Also returns the distance of |v| to the nearest rounding midpoint.
    """
    v = np.asarray(v, dtype=np.float64)
    codes, tie_dist = _round_to_grid(np.abs(v), E2M1_POS_VALUES, E2M1_POS_CODES)
    neg = (v < 0) & (codes != 0)      # -0 is encoded as +0
    return np.where(neg, codes | 0x8, codes).astype(np.int64), tie_dist


def e4m3_round_unsigned(v):
    """E4M3 RNE-satfinite codes (0..0x7E) of non-negative values v.

    Also returns the distance of v to the nearest rounding midpoint.
    """
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0):
        raise ValueError("block scales are non-negative")
    codes, tie_dist = _round_to_grid(v, E4M3_POS_VALUES, E4M3_POS_CODES)
    return codes.astype(np.int64), tie_dist


def e8m0_decode(code):
    """Value of an 8-bit E8M0 scale code: 2^(code - 127); code 255 is NaN.

    E8M0 is the OCP Microscaling shared-scale format: an 8-bit unsigned
    biased exponent, no sign, no mantissa ("powers of two", as the pages
    describe MXFP4's scales).
    """
    code = int(code)
    if code == 255:
        return float("nan")
    return 2.0 ** (code - 127)


def e8m0_values(codes):
    table = np.array([e8m0_decode(c) for c in range(256)])
    return table[np.asarray(codes, dtype=np.int64)]


def e2m1_values(codes):
    table = np.array([e2m1_decode(c) for c in range(16)])
    return table[np.asarray(codes, dtype=np.int64)]


def e4m3_values(codes):
    table = np.array([e4m3_decode(c) for c in range(256)])
    return table[np.asarray(codes, dtype=np.int64)]


def to_fp16(v):
    """Round fp64 values to IEEE half (round to nearest even), returned as fp64."""
    return np.asarray(v, dtype=np.float64).astype(np.float16).astype(np.float64)


def to_fp32(v):
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)
