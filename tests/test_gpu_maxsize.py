"""GPU parity at the largest sizes the boundary accepts.

include/rq.h: rq_rotate_quantize takes K up to 32768 (blocks of 128); the
GEMMs take K up to 65536 (the int32 accumulator stays below 2^31 there).  The
rows are ragged (M not a multiple of any tile) so that the last tile is
partial at the largest K as well.
"""

import numpy as np
import pytest
import torch

import parity
from oracle import gemm, hadamard, quant
from rotation_w4a4_quantization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

K_ROTATE_MAX = 32768
K_GEMM_MAX = 65536


@pytest.fixture(scope="module")
def rq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rotation_w4a4_quantization_b200 import rq as m
    m.init(0)
    return m


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4", "int8", "int4_asym"])
def test_rotate_quantize_at_max_k(rq, fmt):
    m, k = 37, K_ROTATE_MAX
    g = torch.Generator().manual_seed(321)
    x = torch.randn((m, k), generator=g)
    x[:, 5] *= 40.0
    x[:, k - 3] *= -25.0
    x = x.to(torch.bfloat16)
    s = syn.signs(k, 322)
    codes, sc, gs = rq.rotate_quantize(x.cuda(), s.cuda(), 128, fmt)
    torch.cuda.synchronize()
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128)
    if fmt == "int4":
        parity.check_int4_quant(parity.to_np(codes), parity.to_np(sc), xr)
    elif fmt == "int8":
        parity.check_int_quant(parity.to_np(codes), parity.to_np(sc), xr, 8)
    elif fmt == "nvfp4":
        parity.check_nvfp4_quant(parity.to_np(codes), parity.to_np(sc), parity.to_np(gs)[0], xr)
    elif fmt == "mxfp4":
        parity.check_mxfp4_quant(parity.to_np(codes), parity.to_np(sc), xr)
    else:
        szn = parity.to_np(sc).astype(np.float64)
        parity.check_kv4(parity.to_np(codes).reshape(m, k // 128, 64), szn[..., 0], szn[..., 1],
                         xr.reshape(m, k // 128, 128))
    rq.get_device_error()


def test_int4_gemm_acc_at_max_k(rq):
    """Accumulators bit-exact at K = 65536 with the largest products (-8 x -8)
    in every position of one row / column pair: 64 x 65536 = 2^22 per entry."""
    m, n, k = 130, 264, K_GEMM_MAX
    rng = np.random.default_rng(65)
    qx = rng.integers(-8, 8, size=(m, k))
    qw = rng.integers(-8, 8, size=(n, k))
    qx[7, :] = -8
    qw[11, :] = -8
    sx = np.full(m, 1.0 / 7, dtype=np.float32)
    sw = np.full(n, 0.01, dtype=np.float32)
    dev = lambda q, s: (torch.from_numpy(quant.pack_nibbles(q)).cuda(), torch.from_numpy(s).cuda(), None)
    acc = rq.w4a4_gemm(dev(qx, sx), dev(qw, sw), "int4", "i32")
    torch.cuda.synchronize()
    ref = gemm.int4_acc(qx, qw)
    assert ref[7, 11] == 64 * k
    np.testing.assert_array_equal(parity.to_np(acc).astype(np.int64), ref)


def test_nvfp4_gemm_at_max_k(rq):
    m, n, k = 130, 264, K_GEMM_MAX
    gx, gw = np.float32(0.0071), np.float32(0.00013)
    rng = np.random.default_rng(66)
    ex, sx, _, _ = quant.nvfp4_rows(rng.standard_normal((m, k)), gx)
    ew, sw, _, _ = quant.nvfp4_rows(rng.standard_normal((n, k)), gw)
    dev = lambda e, s, g: (torch.from_numpy(quant.pack_nibbles(e)).cuda(),
                           torch.from_numpy(s.astype(np.uint8)).cuda(),
                           torch.tensor([g], dtype=torch.float32).cuda())
    y = rq.w4a4_gemm(dev(ex, sx, gx), dev(ew, sw, gw), "nvfp4", "f32")
    torch.cuda.synchronize()
    ref = gemm.nvfp4_y(ex, sx, gx, ew, sw, gw)
    assert parity.check_y(parity.to_np(y), ref, tol=1e-5) < 1e-5
