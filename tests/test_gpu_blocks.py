"""GPU parity: format-sized block rotations (blocks of 16 and 32).

Q = blockdiag(diag(s) H_B / sqrt(B)) with B = 16 (one block per NVFP4 scale
group) or 32 (one per MXFP4 group), the rotations the FP4 study cited by
"Rotations for 4-Bit Activations: QuaRot, SpinQuant, and Friends" (section
"Gotchas", "Block size matters") sizes to the format's groups.  The rotation
itself against the fp64 oracle, every quantizer on top of it, the dynamic
NVFP4 scale in one pass and in two, and the whole path to Y.
"""

import numpy as np
import pytest
import torch

import parity
from oracle import gemm, hadamard, quant
from rotation_w4a4_quantization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rotation_w4a4_quantization_b200 import rq as m
    m.init(0)
    return m


def _gauss(m, k, seed, outliers=()):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((m, k), generator=g)
    for c, f in outliers:
        x[:, c] *= f
    return x.to(torch.bfloat16)


SHAPES = [(37, 512), (300, 4096), (5, 12288), (2000, 256)]


@pytest.mark.parametrize("block", [16, 32])
@pytest.mark.parametrize("m,k", SHAPES)
def test_rotate_f32_blocks(rq, block, m, k):
    x = _gauss(m, k, m + k + block, outliers=[(3, 50.0), (k - 2, 20.0)])
    s = syn.signs(k, k + block)
    got = rq.rotate_f32(x.cuda(), s.cuda(), block)
    torch.cuda.synchronize()
    parity.check_rotation(parity.to_np(got), hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), block))


@pytest.mark.parametrize("block", [16, 32])
@pytest.mark.parametrize("fmt", ["int4", "int8", "nvfp4", "mxfp4"])
@pytest.mark.parametrize("m,k", SHAPES[:3])
def test_quantize_blocks(rq, block, fmt, m, k):
    x = _gauss(m, k, 7 * m + k + block, outliers=[(9, 40.0)])
    s = syn.signs(k, 3 * k + block)
    codes, sc, g = rq.rotate_quantize(x.cuda(), s.cuda(), block, fmt)
    torch.cuda.synchronize()
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), block)
    if fmt == "int4":
        parity.check_int4_quant(parity.to_np(codes), parity.to_np(sc), xr)
    elif fmt == "int8":
        parity.check_int_quant(parity.to_np(codes), parity.to_np(sc), xr, 8)
    elif fmt == "nvfp4":
        parity.check_nvfp4_quant(parity.to_np(codes), parity.to_np(sc), parity.to_np(g)[0], xr)
    else:
        parity.check_mxfp4_quant(parity.to_np(codes), parity.to_np(sc), xr)


def test_nvfp4_block16_two_pass(rq):
    """4100 x 4096 does not fit the SMs' shared memory: the max and quantize
    passes each stream X (the one-pass kernel covers the shapes above)."""
    m, k = 4100, 4096
    x = _gauss(m, k, 5, outliers=[(100, 30.0)])
    s = syn.signs(k, 6)
    codes, sc, g = rq.rotate_quantize(x.cuda(), s.cuda(), 16, "nvfp4", "dynamic")
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 16)
    parity.check_nvfp4_quant(parity.to_np(codes), parity.to_np(sc), parity.to_np(g)[0], xr)


@pytest.mark.parametrize("fmt,block", [("nvfp4", 16), ("mxfp4", 32), ("int4", 32)])
def test_end_to_end_blocks(rq, fmt, block):
    name = "tiny_int4"
    x, w, s = syn.activations(name), syn.weights(name), syn.workload_signs(name)
    wq = rq.prepare_weights(w.cuda(), s.cuda(), block, fmt)
    xq = rq.rotate_quantize(x.cuda(), s.cuda(), block, fmt)
    y = rq.w4a4_gemm(xq, wq, fmt, "f32")
    torch.cuda.synchronize()
    xd, wd = parity.bf16_to_f64(x), parity.bf16_to_f64(w)
    xr, wr = hadamard.rotate(xd, s.numpy(), block), hadamard.rotate(wd, s.numpy(), block)
    if fmt == "int4":
        qx, sx, tx = quant.int4_sym_rows(xr)
        qw, sw, tw = quant.int4_sym_rows(wr)
        ref = gemm.int4_y(gemm.int4_acc(qx, qw), sx, sw)
        xh, dx = parity.int4_tie_bounds(qx, sx, tx)
        wh, dw = parity.int4_tie_bounds(qw, sw, tw)
    elif fmt == "nvfp4":
        gx, gw = quant.nvfp4_global_scale(xr), quant.nvfp4_global_scale(wr)
        ex, sfx, tex, tsx = quant.nvfp4_rows(xr, gx)
        ew, sfw, tew, tsw = quant.nvfp4_rows(wr, gw)
        ref = gemm.nvfp4_y(ex, sfx, gx, ew, sfw, gw)
        xh, dx = parity.nvfp4_tie_bounds(ex, sfx, gx, tex, tsx)
        wh, dw = parity.nvfp4_tie_bounds(ew, sfw, gw, tew, tsw)
    else:
        ex, sfx, tex, tsx = quant.mxfp4_rows(xr)
        ew, sfw, tew, tsw = quant.mxfp4_rows(wr)
        ref = gemm.mxfp4_y(ex, sfx, ew, sfw)
        xh, dx = parity.mxfp4_tie_bounds(ex, sfx, tex, tsx)
        wh, dw = parity.mxfp4_tie_bounds(ew, sfw, tew, tsw)
    parity.check_y_with_ties(parity.to_np(y), ref, xh, dx, wh, dw)
    rq.get_device_error()


def test_rejects_other_blocks(rq):
    x = _gauss(4, 256, 1)
    s = syn.signs(256, 2)
    for block in (8, 64, 256):
        with pytest.raises(rq.RQError) as e:
            rq.rotate_quantize(x.cuda(), s.cuda(), block, "int4")
        assert e.value.status == 2
    with pytest.raises(rq.RQError):
        rq.rotate_quantize(x.cuda(), s.cuda(), 0, "nvfp4")   # full width is integer formats only


# ---------------------------------------------------------------- per-group asymmetric INT4
@pytest.mark.parametrize("block", [16, 32, 128])
@pytest.mark.parametrize("m,k", [(37, 512), (300, 4096), (5, 12288), (2000, 256)])
def test_asym_int4_groups(rq, block, m, k):
    """Per-group (128) asymmetric INT4 of X~ against the oracle's rule on every
    group: fp16 scale / zero equal except at flagged ties, codes equal except at
    flagged ties or in a group whose scale legitimately differed."""
    x = _gauss(m, k, 11 * m + k + block, outliers=[(5, 30.0)])
    x[m // 2, :128] = 0                                   # a zero group
    s = syn.signs(k, 5 * k + block)
    codes, sz, _ = rq.rotate_quantize(x.cuda(), s.cuda(), block, "int4_asym")
    torch.cuda.synchronize()
    assert codes.shape == (m, k // 2) and sz.shape == (m, k // 128, 2)
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), block).reshape(m, k // 128, 128)
    szn = parity.to_np(sz).astype(np.float64)
    parity.check_kv4(parity.to_np(codes).reshape(m, k // 128, 64), szn[..., 0], szn[..., 1], xr)
    assert szn[m // 2, 0, 0] == 0 and np.all(parity.to_np(codes)[m // 2, :64] == 0)


def test_asym_int4_strided_rows(rq):
    big = _gauss(64, 1024 + 128, 3, outliers=[(1, 20.0)])
    s = syn.signs(1024, 4)
    codes, sz, _ = rq.rotate_quantize(big.cuda()[:, :1024], s.cuda(), 128, "int4_asym")
    xr = hadamard.rotate(parity.bf16_to_f64(big[:, :1024]), s.numpy(), 128).reshape(64, 8, 128)
    szn = parity.to_np(sz).astype(np.float64)
    parity.check_kv4(parity.to_np(codes).reshape(64, 8, 64), szn[..., 0], szn[..., 1], xr)
