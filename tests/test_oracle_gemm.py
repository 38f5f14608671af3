"""Pins for the oracle's W4A4 product (CPU only): triple loops on tiny inputs."""

import numpy as np
import pytest

from oracle import formats, gemm, quant


def test_int4_acc_matches_triple_loop():
    rng = np.random.default_rng(0)
    m, n, k = 5, 7, 64
    qx = rng.integers(-8, 8, size=(m, k))
    qw = rng.integers(-8, 8, size=(n, k))
    acc = gemm.int4_acc(qx, qw)
    for i in range(m):
        for j in range(n):
            s = 0
            for t in range(k):
                s += int(qx[i, t]) * int(qw[j, t])
            assert acc[i, j] == s


def test_int4_acc_extreme_fits_int32():
    k = 12288
    acc = gemm.int4_acc(np.full((1, k), -8), np.full((1, k), -8))
    assert acc[0, 0] == 64 * k and acc[0, 0] < 2 ** 31


def test_int4_y_is_scaled_acc():
    acc = np.array([[3, -2]])
    y = gemm.int4_y(acc, np.array([0.5], dtype=np.float32), np.array([2.0, 4.0], dtype=np.float32))
    assert np.array_equal(y, np.array([[3.0, -4.0]]))


def test_nvfp4_y_matches_blockwise_sum():
    """Y = g_x g_w sum_b Sx[m,b] Sw[n,b] sum_{k in b} e_x e_w, by explicit loops."""
    rng = np.random.default_rng(1)
    m, n, k = 3, 4, 64
    ex = rng.integers(0, 16, size=(m, k))
    ew = rng.integers(0, 16, size=(n, k))
    sx = rng.integers(0, 0x7F, size=(m, k // 16))
    sw = rng.integers(0, 0x7F, size=(n, k // 16))
    gx, gw = np.float32(0.013), np.float32(0.25)
    y = gemm.nvfp4_y(ex, sx, gx, ew, sw, gw)
    for i in range(m):
        for j in range(n):
            tot = 0.0
            for b in range(k // 16):
                inner = sum(formats.e2m1_decode(ex[i, t]) * formats.e2m1_decode(ew[j, t])
                            for t in range(16 * b, 16 * b + 16))
                tot += formats.e4m3_decode(sx[i, b]) * formats.e4m3_decode(sw[j, b]) * inner
            assert np.isclose(y[i, j], float(gx) * float(gw) * tot, rtol=1e-14, atol=1e-300)


def test_dequant_roundtrip_nvfp4_codes():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, 64))
    g = quant.nvfp4_global_scale(x)
    e, s, _, _ = quant.nvfp4_rows(x, g)
    xh = quant.nvfp4_dequant(e, s, g)
    e2, s2, _, _ = quant.nvfp4_rows(xh, g)
    # re-quantizing a dequantized tensor is idempotent on its codes wherever the block scale is kept
    same_scale = (s2 == s)[:, :, None].repeat(16, axis=2).reshape(4, 64)
    assert np.array_equal(formats.e2m1_values(e2)[same_scale], formats.e2m1_values(e)[same_scale])


def test_mxfp4_y_matches_blockwise_sum():
    """Y = sum_b 2^(sx[m,b]-127) 2^(sw[n,b]-127) sum_{k in b} e_x e_w, by explicit loops."""
    import math
    rng = np.random.default_rng(3)
    m, n, k = 3, 2, 64
    ex = rng.integers(0, 16, size=(m, k))
    ew = rng.integers(0, 16, size=(n, k))
    sx = rng.integers(100, 150, size=(m, k // 32))
    sw = rng.integers(100, 150, size=(n, k // 32))
    y = gemm.mxfp4_y(ex, sx, ew, sw)
    for i in range(m):
        for j in range(n):
            tot = 0.0
            for b in range(k // 32):
                inner = sum(formats.e2m1_decode(ex[i, t]) * formats.e2m1_decode(ew[j, t])
                            for t in range(32 * b, 32 * b + 32))
                tot += math.ldexp(inner, int(sx[i, b]) - 127 + int(sw[j, b]) - 127)
            assert y[i, j] == tot


@pytest.mark.parametrize("bx,bw", [(8, 4), (8, 8), (6, 6)])
def test_int_acc_matches_triple_loop(bx, bw):
    rng = np.random.default_rng(bx * 10 + bw)
    m, n, k = 4, 5, 48
    qx = rng.integers(-(2 ** (bx - 1)), 2 ** (bx - 1), size=(m, k))
    qw = rng.integers(-(2 ** (bw - 1)), 2 ** (bw - 1), size=(n, k))
    acc = gemm.int_acc(qx, qw)
    for i in range(m):
        for j in range(n):
            assert acc[i, j] == sum(int(qx[i, t]) * int(qw[j, t]) for t in range(k))


def test_int_acc_extreme_8bit_fits_int32():
    k = 65536
    acc = gemm.int_acc(np.full((1, k), -128), np.full((1, k), -128))
    assert acc[0, 0] == 16384 * k and acc[0, 0] < 2 ** 31
