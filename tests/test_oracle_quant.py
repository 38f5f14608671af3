"""Pins for the oracle's quantizers and packing (CPU only).

Brute force (argmin over all 16 codes), round-trip bounds, the packing golden
examples and the special cases (zero rows, one-hot rows, constant KV vectors).
"""

import numpy as np
import pytest

from oracle import formats, hadamard, quant


def _int4_bruteforce(x, s):
    codes = np.arange(-8, 8)
    d = np.abs(x[..., None] - codes * s)
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    # ties: choose the even integer (round half to even)
    even = (codes % 2) == 0
    pick = np.where((cand & even).any(axis=-1), np.argmax(cand & even, axis=-1), np.argmax(cand, axis=-1))
    return codes[pick]


def test_int4_bruteforce_and_bound():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 256))
    x[:, 3] *= 40
    q, s, tie = quant.int4_sym_rows(x)
    assert q.min() >= -7 and q.max() <= 7         # -8 never produced (s = amax / 7)
    for r in range(x.shape[0]):
        bf = _int4_bruteforce(x[r], float(s[r]))
        ok = (bf == q[r]) | tie[r]
        assert ok.all()
    err = np.abs(x - quant.int4_dequant(q, s))
    assert np.all(err <= s.astype(np.float64)[:, None] * (0.5 + 1e-6))
    # the extreme element of every row maps to +-7
    arg = np.abs(x).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(64), arg]) == 7)


def test_int4_scale_is_fp32_amax_over_7():
    x = np.array([[0.0, -3.5, 1.0, 7.0 / 3.0]])
    q, s, _ = quant.int4_sym_rows(x)
    assert s.dtype == np.float32
    assert s[0] == np.float32(3.5) / np.float32(7.0)
    assert list(q[0]) == [0, -7, 2, 5]          # 1/0.5 = 2 ; (7/3)/0.5 = 4.67 -> 5


def test_int4_zero_row():
    q, s, tie = quant.int4_sym_rows(np.zeros((2, 16)))
    assert np.all(q == 0) and np.all(s == 0) and not tie.any()


def test_int4_half_even_ties():
    # scale = 1: values k + 0.5 round to the even neighbour
    x = np.array([[7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5]])
    q, s, tie = quant.int4_sym_rows(x)
    assert s[0] == 1.0
    assert list(q[0]) == [7, 0, 2, 2, 0, -2, -2, 4]
    assert list(tie[0]) == [False] + [True] * 7


def test_packing_golden(golden):
    for line in golden("int4_packing.txt"):
        codes, packed = line.split(";")
        c = np.array([int(t) for t in codes.split()])
        p = np.array([int(t, 16) for t in packed.split()], dtype=np.uint8)
        assert np.array_equal(quant.pack_nibbles(c), p)
        assert np.array_equal(quant.unpack_nibbles(p, signed=True), c)


def _nvfp4_bruteforce(x, sdec, g):
    vals = np.array([formats.e2m1_decode(c) for c in range(16)]) * sdec * g
    d = np.abs(x[:, None] - vals[None, :])
    return vals[np.argmin(d, axis=1)]


def test_nvfp4_bruteforce_and_structure():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((16, 256))
    x[:, 7] *= 30
    g = quant.nvfp4_global_scale(x)
    assert g == np.float32(np.float32(np.abs(x).max()) / np.float32(2688.0))
    e, sc, tie_e, tie_s = quant.nvfp4_rows(x, g)
    assert sc.shape == (16, 16) and sc.max() <= 0x7E
    xh = quant.nvfp4_dequant(e, sc, g)
    sdec = formats.e4m3_values(sc)
    for r in range(16):
        for b in range(16):
            sl = slice(16 * b, 16 * b + 16)
            if sdec[r, b] == 0:
                assert np.all(e[r, sl] == 0)
                continue
            bf = _nvfp4_bruteforce(x[r, sl], sdec[r, b], np.float64(g))
            ok = (np.abs(bf - xh[r, sl]) == 0) | tie_e[r, sl]
            assert ok.all()
    # the global amax element lands on +-6 * S * g with S = 448 (up to E4M3 rounding)
    r, c = np.unravel_index(np.abs(x).argmax(), x.shape)
    assert sc[r, c // 16] == 0x7E
    assert abs(formats.e2m1_decode(e[r, c])) == 6.0


def test_nvfp4_static_scale_saturates():
    x = np.full((1, 16), 100.0)
    e, sc, _, _ = quant.nvfp4_rows(x, np.float32(0.001))     # far too small a g
    assert sc[0, 0] == 0x7E and np.all(e == 7)


def test_nvfp4_zero_block():
    x = np.zeros((2, 32))
    x[0, 20] = 1.0
    g = quant.nvfp4_global_scale(x)
    e, sc, _, _ = quant.nvfp4_rows(x, g)
    assert sc[0, 0] == 0 and np.all(e[0, :16] == 0) and np.all(sc[1] == 0)


def test_kv4_bruteforce_and_bound():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((3, 5, 128))
    xr = hadamard.rotate(x.reshape(-1, 128), rng.choice([-1, 1], size=128), 128).reshape(x.shape)
    q, s_h, z_h, tie, _ = quant.kv4_vectors(xr)
    assert q.min() >= 0 and q.max() <= 15
    codes = np.arange(16)
    recon = codes[None, None, None, :] * s_h[..., None, None] + z_h[..., None, None]
    bf = np.argmin(np.abs(xr[..., None] - recon), axis=-1)
    assert np.all((bf == q) | tie)
    lo, hi = xr.min(-1), xr.max(-1)
    s = (hi - lo) / 15
    bound = s_h / 2 + np.abs(lo - z_h) + 15 * np.abs(s - s_h)
    assert np.all(np.abs(xr - quant.kv4_dequant(q, s_h, z_h)) <= bound[..., None] * (1 + 1e-9))
    # scale and zero are fp16 values
    assert np.array_equal(formats.to_fp16(s_h), s_h) and np.array_equal(formats.to_fp16(z_h), z_h)


def test_kv4_constant_vector():
    x = np.full((1, 128), 3.0)
    q, s_h, z_h, _, _ = quant.kv4_vectors(x)
    assert np.all(q == 0) and s_h[0] == 0 and z_h[0] == 3.0


@pytest.mark.parametrize("k", [16, 512])
def test_unpack_roundtrip_unsigned(k):
    rng = np.random.default_rng(k)
    c = rng.integers(0, 16, size=(3, k))
    assert np.array_equal(quant.unpack_nibbles(quant.pack_nibbles(c), signed=False), c)


# ---------------------------------------------------------------- MXFP4
def _mx_block(vals):
    x = np.zeros((1, 32))
    x[0, :len(vals)] = vals
    return x


def test_mxfp4_hand_block():
    # amax = 6: floor(log2 6) - 2 = 0, scale 1; codes are E2M1 of the values
    # themselves, nearest with ties to the even code, saturating at 6.
    vals = [6.0, -3.0, 1.5, 0.75, 0.25, 0.3, -0.26, 5.0, 2.5, -1.25, 3.5]
    want = [7, 8 | 5, 3, 2, 0, 1, 8 | 1, 6, 4, 8 | 2, 6]
    #       6  -3     1.5 1(tie 0.5|1 -> even 1.0) 0(tie 0|0.5 -> even 0) 0.5 -0.5
    #       4(tie 4|6 -> even 4) 2(tie 2|3 -> even 2) -1(tie 1|1.5 -> even 1) 4(tie 3|4 -> even 4)
    e, s, tie_e, tie_s = quant.mxfp4_rows(_mx_block(vals))
    assert s[0, 0] == 127
    assert list(e[0, :len(vals)]) == want
    assert np.all(e[0, len(vals):] == 0)
    assert tie_e[0, 3] and tie_e[0, 4] and tie_e[0, 7] and not tie_e[0, 0]


def test_mxfp4_saturates_and_scales():
    # amax = 7.9 * 2^5: exponent floor(log2 7.9) + 5 - 2 = 5; 7.9 -> 6 (saturation)
    x = _mx_block([7.9 * 32, 1.0 * 32, -0.5 * 32])
    e, s, _, _ = quant.mxfp4_rows(x)
    assert s[0, 0] == 127 + 5
    assert list(e[0, :3]) == [7, 2, 8 | 1]
    # amax = 1: exponent -2, scale 1/4, so 1 -> 4 and 0.3 -> 1.2 -> 1
    e, s, _, _ = quant.mxfp4_rows(_mx_block([1.0, 0.3]))
    assert s[0, 0] == 125 and list(e[0, :2]) == [6, 2]


def test_mxfp4_scale_rule_by_search():
    # the shared exponent is the unique integer e with 2^(e+2) <= amax < 2^(e+3)
    rng = np.random.default_rng(11)
    for _ in range(400):
        mag = np.ldexp(rng.uniform(1.0, 2.0), int(rng.integers(-60, 60)))
        x = _mx_block(rng.uniform(-1, 1, 32) * mag)
        amax = np.abs(x).max()
        e_search = next(c for c in range(-200, 200) if 2.0 ** (c + 2) <= amax < 2.0 ** (c + 3))
        _, s, _, _ = quant.mxfp4_rows(x)
        assert s[0, 0] - 127 == min(max(e_search, -127), 127)


def test_mxfp4_power_of_two_equivariance():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((4, 64)) * 3
    e0, s0, _, _ = quant.mxfp4_rows(x)
    for j in (-9, -1, 1, 13):
        e1, s1, _, _ = quant.mxfp4_rows(x * 2.0 ** j)
        assert np.array_equal(e0, e1) and np.array_equal(s1, s0 + j)


def test_mxfp4_roundtrip_bound_and_zero_block():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((8, 128)) * rng.uniform(0.01, 100, size=(8, 1))
    x[3, 32:64] = 0.0
    e, s, _, _ = quant.mxfp4_rows(x)
    xh = quant.mxfp4_dequant(e, s)
    sc = np.repeat(formats.e8m0_values(s), 32, axis=1)
    v = np.abs(x) / sc
    grid = formats.E2M1_POS_VALUES
    # half the local grid spacing below 6; saturated values sit at 6 * scale
    idx = np.clip(np.searchsorted(grid, np.minimum(v, 6.0)), 1, len(grid) - 1)
    half_gap = 0.5 * (grid[idx] - grid[idx - 1])
    ok = np.where(v <= 6.0, np.abs(x - xh) <= half_gap * sc + 1e-300, np.abs(xh) == 6.0 * sc)
    assert ok.all()
    assert s[3, 1] == 0 and np.all(e[3, 32:64] == 0)


def test_mxfp4_power_of_two_amax_is_a_scale_tie():
    x = _mx_block([4.0, 1.0])
    _, s, _, tie_s = quant.mxfp4_rows(x)
    assert s[0, 0] == 127 and tie_s[0, 0]
    _, _, _, tie_s = quant.mxfp4_rows(_mx_block([5.0, 1.0]))
    assert not tie_s[0, 0]


# ---------------------------------------------------------------- 6- and 8-bit RTN
def _int_bruteforce(x, s, bits):
    qmax = 2 ** (bits - 1) - 1
    codes = np.arange(-qmax - 1, qmax + 1)
    d = np.abs(x[..., None] - codes * s)
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    even = (codes % 2) == 0
    pick = np.where((cand & even).any(axis=-1), np.argmax(cand & even, axis=-1), np.argmax(cand, axis=-1))
    return codes[pick]


@pytest.mark.parametrize("bits", [6, 8])
def test_int_sym_bruteforce_and_bound(bits):
    """Each code is the nearest of all 2^b codes to x / s (argmin search, half to even)."""
    qmax = 2 ** (bits - 1) - 1
    rng = np.random.default_rng(40 + bits)
    x = rng.standard_normal((24, 128))
    x[:, 5] *= 30
    q, s, tie = quant.int_sym_rows(x, bits)
    assert q.min() >= -qmax and q.max() <= qmax   # -qmax-1 never produced (s = amax / qmax)
    for r in range(x.shape[0]):
        bf = _int_bruteforce(x[r], float(s[r]), bits)
        assert ((bf == q[r]) | tie[r]).all()
    err = np.abs(x - quant.int4_dequant(q, s))
    assert np.all(err <= s.astype(np.float64)[:, None] * (0.5 + 1e-6))
    arg = np.abs(x).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(24), arg]) == qmax)


def test_int8_and_int6_hand_worked_row():
    """x = [2.54, -1, 0.5, 0.071]: s = 2.54/127 = 0.02 -> codes 127, -50, 25, 3.55 -> 4;
    s = 2.54/31 = 0.08193548 -> 31, -12.20 -> -12, 6.10 -> 6, 0.867 -> 1."""
    x = np.array([[2.54, -1.0, 0.5, 0.071]])
    q8, s8, _ = quant.int_sym_rows(x, 8)
    assert s8[0] == np.float32(np.float32(2.54) / np.float32(127.0))
    assert list(q8[0]) == [127, -50, 25, 4]
    q6, s6, _ = quant.int_sym_rows(x, 6)
    assert s6[0] == np.float32(np.float32(2.54) / np.float32(31.0))
    assert list(q6[0]) == [31, -12, 6, 1]


def test_int_sym_zero_row_and_half_even():
    q, s, tie = quant.int_sym_rows(np.zeros((2, 8)), 8)
    assert np.all(q == 0) and np.all(s == 0) and not tie.any()
    # scale 1 (amax = 127): k + 0.5 rounds to the even neighbour
    x = np.array([[127.0, 0.5, 1.5, 2.5, -0.5, -1.5, -126.5, 3.5]])
    q, s, tie = quant.int_sym_rows(x, 8)
    assert s[0] == 1.0
    assert list(q[0]) == [127, 0, 2, 2, 0, -2, -126, 4]
    assert list(tie[0]) == [False] + [True] * 7


def test_int_sym_at_4_bits_is_the_int4_rule():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((8, 64))
    a = quant.int_sym_rows(x, 4)
    b = quant.int4_sym_rows(x)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_more_bits_lower_error():
    """Round to nearest with b bits: the worst error is s/2 = amax / (2 (2^(b-1) - 1)),
    so each extra bit roughly halves it."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal((32, 256))
    errs = []
    for bits in (4, 6, 8):
        q, s, _ = quant.int_sym_rows(x, bits)
        errs.append(np.linalg.norm(x - quant.int4_dequant(q, s)) / np.linalg.norm(x))
    assert errs[0] > 3.5 * errs[1] > 3.5 * 3.5 * errs[2]


# ---------------------------------------------------------------- per-group asymmetric INT4
def test_asym_int4_groups_bruteforce_and_bound():
    """Each group of 128: codes are the nearest of 0..15 to (x - z_h)/s_h (argmin
    search), the group's min maps to 0 and max to 15, |x - deq| <= s_h/2 (+ the
    fp16 rounding of s and z)."""
    rng = np.random.default_rng(21)
    x = rng.standard_normal((6, 512))
    x[:, 130] *= 25
    q, s_h, z_h, tie, tie_sz = quant.asym_int4_groups(x)
    assert q.shape == x.shape and s_h.shape == (6, 4) and q.min() >= 0 and q.max() <= 15
    for r in range(6):
        for g in range(4):
            sl = slice(128 * g, 128 * (g + 1))
            d = np.abs((x[r, sl, None] - z_h[r, g]) - np.arange(16) * s_h[r, g])
            best = d.min(axis=-1, keepdims=True)
            ok = (d[np.arange(128), q[r, sl]] == best[:, 0]) | tie[r, sl]
            assert ok.all()
            assert q[r, sl][np.argmin(x[r, sl])] in (0, 1) and q[r, sl][np.argmax(x[r, sl])] in (14, 15)
    err = np.abs(x - quant.asym_int4_dequant(q, s_h, z_h))
    bound = np.repeat(s_h, 128, axis=1) * 0.5 + np.repeat(np.abs(z_h) + 15 * s_h, 128, axis=1) * 2.0 ** -10
    assert np.all(err <= bound)


def test_asym_int4_groups_hand_worked():
    """A group holding 0, 0.5, ..., 7.5 (eight times): z = min = 0, s = (7.5 - 0)/15
    = 0.5 exactly, so the codes are x / 0.5 = 0..15 with no rounding."""
    g = np.tile(np.arange(16) * 0.5, 8)            # 128 values in [0, 7.5], step 0.5
    q, s_h, z_h, tie, _ = quant.asym_int4_groups(g[None, :])
    assert s_h[0, 0] == 0.5 and z_h[0, 0] == 0.0
    assert np.array_equal(q[0], np.tile(np.arange(16), 8)) and not tie.any()


def test_asym_int4_groups_equal_kv4_per_group():
    rng = np.random.default_rng(22)
    x = rng.standard_normal((3, 256))
    q, s_h, z_h, _, _ = quant.asym_int4_groups(x)
    for g in range(2):
        qg, sg, zg, _, _ = quant.kv4_vectors(x[:, 128 * g:128 * (g + 1)])
        assert np.array_equal(q[:, 128 * g:128 * (g + 1)], qg)
        assert np.array_equal(s_h[:, g], sg) and np.array_equal(z_h[:, g], zg)


# ---------------------------------------------------------------- NVFP4 worked by hand
def _nvfp4_golden(golden):
    """Parse tests/golden/nvfp4_block.txt: the per-tensor scale cases and a
    2 x 32 tensor with its E4M3 block scales and E2M1 codes."""
    gcases, x, e, s = [], np.zeros((2, 32)), np.zeros((2, 32), dtype=np.int64), np.zeros((2, 2), dtype=np.int64)
    for line in golden("nvfp4_block.txt"):
        t = line.split()
        if t[0] == "g":
            gcases.append((float(t[1]), int(t[2], 16)))
            continue
        r, b = int(t[1]), int(t[2])
        sl = slice(16 * b, 16 * b + 16)
        if t[0] == "x":
            x[r, sl] = [float(v) for v in t[3:]]
        elif t[0] == "e":
            e[r, sl] = [int(v) for v in t[3:]]
        elif t[0] == "s":
            s[r, b] = int(t[3], 16)
    return gcases, x, e, s


def test_nvfp4_global_scale_golden(golden):
    gcases, _, _, _ = _nvfp4_golden(golden)
    assert len(gcases) == 4
    for amax, bits in gcases:
        x = np.array([[0.25 * amax, -amax, 0.0, 0.5 * amax]])     # the max is taken over |x|
        g = quant.nvfp4_global_scale(x)
        assert g.dtype == np.float32
        assert int(np.asarray(g).view(np.uint32)) == bits, (amax, hex(int(np.asarray(g).view(np.uint32))))


def test_nvfp4_block_golden(golden):
    """Every block scale and code of the hand-worked tensor (two saturating,
    one subnormal-scale and two in-between blocks' worth of rounding cases,
    ties resolved to the even code, -0 written as +0)."""
    _, x, e_ref, s_ref = _nvfp4_golden(golden)
    # the fixture's values are exact in bf16, so the same tensor can feed the GPU path
    import torch
    assert np.array_equal(torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy(), x)
    g = quant.nvfp4_global_scale(x)
    assert g == np.float32(0.0625)
    e, sc, tie_e, tie_s = quant.nvfp4_rows(x, g)
    assert np.array_equal(sc, s_ref), (sc, s_ref)
    assert np.array_equal(e, e_ref), np.argwhere(e != e_ref)
    assert not tie_s.any()
    # exact midpoints are flagged as ties (and resolved to the even code above)
    assert tie_e[0, 3] and tie_e[0, 4] and tie_e[0, 5] and tie_e[1, 16 + 2] and not tie_e[0, 0]
    xh = quant.nvfp4_dequant(e, sc, g)
    assert xh[1, 16] == 6 * 2.0 ** -13                               # 8 * 2^-13 saturates to 6 * S g


def test_nvfp4_block_golden_catches_a_wrong_scale_divisor(golden, monkeypatch):
    """A planted mistake in the oracle -- the block scale's divisor 6 g taken
    as 4 g -- changes three of the four golden block scales."""
    _, x, _, s_ref = _nvfp4_golden(golden)
    g = quant.nvfp4_global_scale(x)
    monkeypatch.setattr(quant, "E2M1_MAX", 4.0)
    _, sc, _, _ = quant.nvfp4_rows(x, g)
    assert (sc != s_ref).sum() == 3
