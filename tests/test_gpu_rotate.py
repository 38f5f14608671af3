"""GPU parity: fused rotation + quantization kernels against the fp64 oracle.

All calls go through the C ABI (librq.so) via the thin binding.
"""

import numpy as np
import pytest
import torch

import parity
from oracle import hadamard, quant
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


def _signs(k, seed):
    return syn.signs(k, seed)


# ---------------------------------------------------------------- rotation fp32
@pytest.mark.parametrize("m,k,block", [
    (64, 512, 128), (1000, 512, 128), (37, 12288, 128), (5, 128, 128),
    (300, 4096, 0), (77, 256, 0), (33, 512, 0), (40, 1024, 0), (21, 2048, 0),
])
def test_rotate_f32(rq, m, k, block):
    x = _gauss(m, k, 10 + m + k, outliers=[(3, 50.0)])
    s = _signs(k, 20 + k)
    got = rq.rotate_f32(x.cuda(), s.cuda(), block)
    torch.cuda.synchronize()
    ref = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), block)
    parity.check_rotation(parity.to_np(got), ref)


def test_rotate_f32_strided_rows(rq):
    k = 1024
    big = _gauss(50, k + 64, 5)
    x = big[:, :k]
    s = _signs(k, 6)
    got = rq.rotate_f32(big.cuda()[:, :k], s.cuda(), 128)
    ref = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128)
    parity.check_rotation(parity.to_np(got), ref)


# ---------------------------------------------------------------- INT4
@pytest.mark.parametrize("m,k,block", [
    (64, 512, 128),        # tiny config shape
    (20000, 512, 128),     # many tiles per CTA (pipeline wrap-around) + ragged tail
    (1203, 4096, 128),
    (517, 12288, 128),     # down_proj width, 96 blocks per row
    (3700, 4096, 0),       # q_proj full-width, several tiles per CTA, ragged
    (129, 256, 0), (50, 1024, 0), (31, 2048, 0), (64, 512, 0),
])
def test_int4_rotate_quantize(rq, m, k, block):
    x = _gauss(m, k, 100 + m, outliers=[(7, 40.0), (k - 1, 25.0)])
    s = _signs(k, 200 + k)
    codes, scales, _ = rq.rotate_quantize(x.cuda(), s.cuda(), block, "int4")
    torch.cuda.synchronize()
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), block)
    parity.check_int4_quant(parity.to_np(codes), parity.to_np(scales), xr)


def test_int4_tiny_workload(rq):
    x = syn.activations("tiny_int4")
    s = syn.workload_signs("tiny_int4")
    codes, scales, _ = rq.rotate_quantize(x.cuda(), s.cuda(), 128, "int4")
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128)
    parity.check_int4_quant(parity.to_np(codes), parity.to_np(scales), xr)


def test_int4_edge_rows(rq):
    """Zero rows, one-hot rows (exactly +-1/sqrt(B) times the value), constant rows, all-plus signs."""
    k = 512
    x = torch.zeros((8, k), dtype=torch.float32)
    x[1, 5] = 3.0
    x[2, :] = 1.0
    x[3, 100] = -1e-3
    x[4] = torch.linspace(-2, 2, k)
    x[6, 511] = 7.5
    x = x.to(torch.bfloat16)
    s = torch.ones(k, dtype=torch.int8)
    codes, scales, _ = rq.rotate_quantize(x.cuda(), s.cuda(), 128, "int4")
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128)
    parity.check_int4_quant(parity.to_np(codes), parity.to_np(scales), xr)
    sc = parity.to_np(scales)
    assert sc[0] == 0 and sc[5] == 0 and np.all(parity.to_np(codes)[0] == 0)
    # one-hot: the 128-block holds +-3/sqrt(128) -> all codes +-7 in that block, 0 elsewhere
    q1 = quant.unpack_nibbles(parity.to_np(codes)[1], signed=True)
    assert np.all(np.abs(q1[:128]) == 7) and np.all(q1[128:] == 0)


def test_int4_strided_and_empty(rq):
    k = 512
    big = _gauss(40, k + 128, 9)
    s = _signs(k, 8)
    codes, scales, _ = rq.rotate_quantize(big.cuda()[:, :k], s.cuda(), 128, "int4")
    xr = hadamard.rotate(parity.bf16_to_f64(big[:, :k]), s.numpy(), 128)
    parity.check_int4_quant(parity.to_np(codes), parity.to_np(scales), xr)
    e = torch.empty((0, k), dtype=torch.bfloat16, device="cuda")
    c0, s0, _ = rq.rotate_quantize(e, s.cuda(), 128, "int4")
    assert c0.shape == (0, k // 2) and s0.shape == (0,)


def test_prepare_weights_int4(rq):
    w = syn.weights("tiny_int4")
    s = syn.workload_signs("tiny_int4")
    codes, scales, _ = rq.prepare_weights(w.cuda(), s.cuda(), 128, "int4")
    wr = hadamard.rotate(parity.bf16_to_f64(w), s.numpy(), 128)
    parity.check_int4_quant(parity.to_np(codes), parity.to_np(scales), wr)


# ---------------------------------------------------------------- NVFP4
@pytest.mark.parametrize("m,k", [(64, 512), (2048, 4096), (333, 4096), (9000, 512), (77, 12288)])
def test_nvfp4_rotate_quantize_dynamic(rq, m, k):
    x = _gauss(m, k, 300 + m, outliers=[(11, 30.0)])
    s = _signs(k, 400 + k)
    codes, sc, g = rq.rotate_quantize(x.cuda(), s.cuda(), 128, "nvfp4", "dynamic")
    torch.cuda.synchronize()
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128)
    parity.check_nvfp4_quant(parity.to_np(codes), parity.to_np(sc), parity.to_np(g)[0], xr)


def test_nvfp4_dynamic_strided_rows(rq):
    # rows ldx = K + 256 apart: the one-pass kernel copies them row by row
    m, k = 300, 4096
    big = _gauss(m, k + 256, 91, outliers=[(7, 25.0)])
    x = big.cuda()[:, :k]
    s = _signs(k, 92)
    codes, sc, g = rq.rotate_quantize(x, s.cuda(), 128, "nvfp4", "dynamic")
    xr = hadamard.rotate(parity.bf16_to_f64(big[:, :k]), s.numpy(), 128)
    parity.check_nvfp4_quant(parity.to_np(codes), parity.to_np(sc), parity.to_np(g)[0], xr)


def test_nvfp4_dynamic_larger_than_shared_memory(rq):
    # 4100 x 4096 bf16 (33.6 MB) exceeds what the SMs' shared memory holds at
    # once, so the max pass and the quantize pass stream X from HBM twice;
    # the scale is checked against the whole tensor, the codes on sampled rows
    m, k = 4100, 4096
    x = _gauss(m, k, 93, outliers=[(100, 40.0)])
    s = _signs(k, 94)
    codes, sc, g = rq.rotate_quantize(x.cuda(), s.cuda(), 128, "nvfp4", "dynamic")
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128)
    g_o = quant.nvfp4_global_scale(xr)
    assert abs(float(parity.to_np(g)[0]) - float(g_o)) <= parity.SCALE_RTOL * float(g_o)
    rows = np.unique(np.concatenate([np.arange(0, m, 67), [m - 1]]))
    parity.check_nvfp4_quant(parity.to_np(codes)[rows], parity.to_np(sc)[rows], None, xr[rows], g_ref=g_o)


def test_nvfp4_static_scale(rq):
    m, k = 300, 1024
    x = _gauss(m, k, 55)
    s = _signs(k, 56)
    g = torch.tensor([0.0013], dtype=torch.float32, device="cuda")
    codes, sc, g2 = rq.rotate_quantize(x.cuda(), s.cuda(), 128, "nvfp4", "static", gscale=g)
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128)
    parity.check_nvfp4_quant(parity.to_np(codes), parity.to_np(sc), None, xr, g_ref=np.float32(0.0013))


def test_nvfp4_zero_and_onehot(rq):
    k = 256
    x = torch.zeros((4, k))
    x[1, 3] = 2.0
    x[2, 200] = -0.25
    x = x.to(torch.bfloat16)
    s = _signs(k, 77)
    codes, sc, g = rq.rotate_quantize(x.cuda(), s.cuda(), 128, "nvfp4", "dynamic")
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128)
    parity.check_nvfp4_quant(parity.to_np(codes), parity.to_np(sc), parity.to_np(g)[0], xr)
    assert np.all(parity.to_np(codes)[0] == 0) and np.all(parity.to_np(sc)[0] == 0)


# ---------------------------------------------------------------- argument errors reach the caller
def test_rejects_bad_arguments(rq):
    x = torch.zeros((4, 384), dtype=torch.bfloat16, device="cuda")
    s = torch.ones(384, dtype=torch.int8, device="cuda")
    with pytest.raises(rq.RQError) as e:
        rq.rotate_quantize(x, s, 0, "int4")      # full width needs a power of two
    assert e.value.status == 2
    with pytest.raises(rq.RQError):
        rq.rotate_quantize(x, s, 64, "int4")     # block must be 128 or 0
    with pytest.raises(rq.RQError):
        rq.rotate_quantize(x[:, 1:], s[1:], 128, "int4")
    rq.get_device_error()


# ---------------------------------------------------------------- K = 4096 full width: team edge cases
@pytest.mark.parametrize("m", [1, 3, 5, 1185, 4097])
@pytest.mark.parametrize("fmt", ["int4", "int8", "f32"])
def test_full_width_4096_row_counts(rq, m, fmt):
    """Fewer rows than a CTA's four row teams, a ragged last team, several rows
    per team; a zero row; rows of a wider tensor (row stride 4160)."""
    k = 4096
    big = _gauss(m, k + 64, 300 + m, outliers=[(11, 60.0)])
    big[m // 2] = 0
    x = big[:, :k]
    s = _signs(k, 77)
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 0)
    view = big.cuda()[:, :k]
    if fmt == "f32":
        got = rq.rotate_f32(view, s.cuda(), 0)
        parity.check_rotation(parity.to_np(got), xr)
        return
    codes, scales, _ = rq.rotate_quantize(view, s.cuda(), 0, fmt)
    torch.cuda.synchronize()
    if fmt == "int4":
        parity.check_int4_quant(parity.to_np(codes), parity.to_np(scales), xr)
    else:
        parity.check_int_quant(parity.to_np(codes), parity.to_np(scales), xr, 8)
    assert parity.to_np(scales)[m // 2] == 0


@pytest.mark.parametrize("block,k", [(128, 512), (32, 256), (16, 256), (0, 4096), (0, 1024)])
def test_rotate_f32_onehot_is_exact(rq, block, k):
    """A one-hot row rotates to +-v/sqrt(B) on its block and exact zeros elsewhere
    (one nonzero term per output: no rounding but the fp32 1/sqrt(B) itself)."""
    b = k if block == 0 else block
    rows = [(0, 1.0), (k - 1, -2.0), (k // 2 + 5, 0.5)]
    x = torch.zeros((len(rows), k), dtype=torch.float32)
    for r, (ch, val) in enumerate(rows):
        x[r, ch] = val
    s = _signs(k, 31)
    got = parity.to_np(rq.rotate_f32(x.to(torch.bfloat16).cuda(), s.cuda(), block)).astype(np.float64)
    inv = float(np.float32(1.0 / np.sqrt(b)))
    for r, (ch, val) in enumerate(rows):
        blk = ch // b
        inside = got[r, blk * b:(blk + 1) * b]
        assert np.all(np.abs(inside) == abs(val) * inv)
        assert np.all(np.delete(got[r], np.s_[blk * b:(blk + 1) * b]) == 0)
