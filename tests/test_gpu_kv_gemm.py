"""GPU parity: KV4 kernel and the W4A4 GEMMs (INT4 kind::i8, NVFP4 kind::mxf4nvf4)."""

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


# ---------------------------------------------------------------- KV4
@pytest.mark.parametrize("b,h,s", [(2, 4, 300), (1, 32, 64), (3, 5, 1001)])
def test_kv4(rq, b, h, s):
    kv = syn.kv(batch=b, heads=h, seq=s)
    sg = syn.workload_signs("kv4")
    codes, scale, zero = rq.kv_rotate_quantize(kv.cuda(), sg.cuda())
    torch.cuda.synchronize()
    x = parity.bf16_to_f64(kv)
    xr = hadamard.rotate(x.reshape(-1, 128), sg.numpy(), 128).reshape(x.shape)
    parity.check_kv4(parity.to_np(codes), parity.to_np(scale).astype(np.float64),
                     parity.to_np(zero).astype(np.float64), xr)


def test_kv4_strided_view(rq):
    """A slice of a larger cache along the sequence axis (non-contiguous rows)."""
    full = syn.kv(batch=2, heads=3, seq=200, which=1)
    view = full.cuda()[:, :, 17:150, :]
    sg = syn.workload_signs("kv4")
    codes, scale, zero = rq.kv_rotate_quantize(view, sg.cuda())
    x = parity.bf16_to_f64(full[:, :, 17:150, :])
    xr = hadamard.rotate(x.reshape(-1, 128), sg.numpy(), 128).reshape(x.shape)
    parity.check_kv4(parity.to_np(codes), parity.to_np(scale).astype(np.float64),
                     parity.to_np(zero).astype(np.float64), xr)


def test_kv4_constant_and_zero_vectors(rq):
    kv = torch.zeros((1, 1, 4, 128))
    kv[0, 0, 1] = 3.0        # constant -> rotated one-hot on dim 0 -> max != min
    kv[0, 0, 2, 7] = -1.5
    kv = kv.to(torch.bfloat16)
    sg = torch.ones(128, dtype=torch.int8)
    codes, scale, zero = rq.kv_rotate_quantize(kv.cuda(), sg.cuda())
    x = parity.bf16_to_f64(kv)
    xr = hadamard.rotate(x.reshape(-1, 128), sg.numpy(), 128).reshape(x.shape)
    parity.check_kv4(parity.to_np(codes), parity.to_np(scale).astype(np.float64),
                     parity.to_np(zero).astype(np.float64), xr)
    assert parity.to_np(scale)[0, 0, 0] == 0 and np.all(parity.to_np(codes)[0, 0, 0] == 0)


def _near_fp16_midpoint_vectors(signs, n, seed):
    """n head vectors whose exact rotated min (even rows) or (max - min)/15 (odd
    rows) lies within 2^-22 of its size from an fp16 rounding midpoint, where an
    fp32 rotation may round z or s to the wrong side: the kernels must take
    those decisions from the exact values (their fp64 second look).

    Each vector has three nonzero channels, 1, 2 and 4, holding a, b, c (times
    the channel's sign): after diag(s) and H_128 / sqrt(128) its values are
    (+-a +-b +-c) / sqrt(128), the min -(a + b + c) / sqrt(128) at channel 7
    and the max at channel 0.  a + b + c, three bf16 values of falling size,
    is chosen to put the target within 2^-22 of a midpoint; rows that miss are
    redrawn.  Plain numpy on the pages' definitions; the expected values come
    from the oracle."""
    rng = np.random.default_rng(seed)
    c = 2.0 ** -3.5

    def bf16(v):
        return float(torch.tensor(v, dtype=torch.float64).to(torch.bfloat16).to(torch.float64))

    def midpoint(t):
        ulp = np.ldexp(1.0, int(np.floor(np.log2(t))) - 10)
        return (np.floor(t / ulp) + 0.5) * ulp

    rows = []
    while len(rows) < n:
        scale_row = len(rows) % 2 == 1
        m = midpoint(2.0 ** rng.uniform(-6, 6))
        t = m * (1.0 + rng.uniform(-2.0 ** -24, 2.0 ** -24))
        total = t * 15.0 / (2.0 * c) if scale_row else t / c
        a = bf16(total * 0.99)
        b = bf16(total - a)
        cc = bf16(total - a - b)
        got = (a + b + cc) * c * (2.0 / 15.0 if scale_row else 1.0)
        if not (a > 0 and b > 0 and cc > 0) or abs(got - midpoint(got)) > 2.0 ** -22 * got:
            continue
        x = np.zeros(128)
        x[1], x[2], x[4] = a * signs[1], b * signs[2], cc * signs[4]
        rows.append(x)
    return np.array(rows)


def _check_exact_scale_zero(codes, scale, zero, xr):
    q, s_h, z_h, tie, _ = quant.kv4_vectors(xr)
    # no tie excuse for the fp16 decisions: they must be the exact ones
    np.testing.assert_array_equal(np.asarray(scale, dtype=np.float64).reshape(s_h.shape), s_h)
    np.testing.assert_array_equal(np.asarray(zero, dtype=np.float64).reshape(z_h.shape), z_h)
    parity.check_codes(quant.unpack_nibbles(codes, signed=False).reshape(q.shape), q, tie, what="codes")


def test_kv4_scale_zero_near_fp16_midpoints(rq):
    sg = syn.workload_signs("kv4")
    x = _near_fp16_midpoint_vectors(sg.numpy(), 512, 77)
    kv = torch.from_numpy(x).to(torch.bfloat16).reshape(1, 1, -1, 128)
    assert np.array_equal(parity.bf16_to_f64(kv).reshape(x.shape), x)   # the inputs are exactly these
    codes, scale, zero = rq.kv_rotate_quantize(kv.cuda(), sg.cuda())
    xr = hadamard.rotate(x, sg.numpy(), 128)
    _check_exact_scale_zero(parity.to_np(codes).reshape(-1, 64), parity.to_np(scale), parity.to_np(zero), xr)


def test_int4_asym_scale_zero_near_fp16_midpoints(rq):
    sg = syn.workload_signs("kv4")
    x = _near_fp16_midpoint_vectors(sg.numpy(), 384, 78)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    codes, sz, _ = rq.rotate_quantize(xb.cuda(), sg.cuda(), 128, "int4_asym")
    sz = parity.to_np(sz).astype(np.float64).reshape(-1, 2)
    xr = hadamard.rotate(x, sg.numpy(), 128)
    _check_exact_scale_zero(parity.to_np(codes), sz[:, 0], sz[:, 1], xr)


# ---------------------------------------------------------------- INT4 GEMM on identical codes
def _rand_int4_operands(m, n, k, seed):
    rng = np.random.default_rng(seed)
    qx = rng.integers(-8, 8, size=(m, k))
    qw = rng.integers(-8, 8, size=(n, k))
    sx = (rng.random(m) + 0.5).astype(np.float32) / 7
    sw = (rng.random(n) * 0.01 + 0.001).astype(np.float32)
    return qx, qw, sx, sw


def _dev_int4(q, s):
    return (torch.from_numpy(quant.pack_nibbles(q)).cuda(), torch.from_numpy(s).cuda(), None)


@pytest.mark.parametrize("m,n,k", [(64, 256, 512), (1100, 4200, 512), (300, 600, 4096), (128, 256, 128),
                                   (5, 40, 256), (257, 513, 1152)])
def test_int4_gemm_acc_bit_exact(rq, m, n, k):
    qx, qw, sx, sw = _rand_int4_operands(m, n, k, m + n + k)
    acc = rq.w4a4_gemm(_dev_int4(qx, sx), _dev_int4(qw, sw), "int4", "i32")
    torch.cuda.synchronize()
    ref = gemm.int4_acc(qx, qw)
    got = parity.to_np(acc).astype(np.int64)
    assert np.array_equal(got, ref), np.argwhere(got != ref)[:5]


@pytest.mark.parametrize("m,n,k", [(1100, 4200, 512), (96, 300, 1024)])
def test_int4_gemm_y(rq, m, n, k):
    qx, qw, sx, sw = _rand_int4_operands(m, n, k, 7 * m + n)
    xq, wq = _dev_int4(qx, sx), _dev_int4(qw, sw)
    y = rq.w4a4_gemm(xq, wq, "int4", "f32")
    yb = rq.w4a4_gemm(xq, wq, "int4", "bf16")
    torch.cuda.synchronize()
    ref = gemm.int4_y(gemm.int4_acc(qx, qw), sx, sw)
    err = parity.check_y(parity.to_np(y), ref, tol=1e-6)
    assert err < 1e-6
    ybf = yb.float().cpu().numpy().astype(np.float64)
    rb = parity.bf16_round(ref)
    ulp = np.abs(rb) * 2.0 ** -7
    assert np.all(np.abs(ybf - rb) <= ulp + 1e-30)


def test_int4_gemm_extremes(rq):
    """All codes -8 (never produced by the quantizer, but valid INT4): |acc| = 64 K."""
    m, n, k = 128, 256, 4096
    qx = np.full((m, k), -8)
    qw = np.full((n, k), -8)
    qw[1] = 7
    acc = rq.w4a4_gemm(_dev_int4(qx, np.ones(m, np.float32)), _dev_int4(qw, np.ones(n, np.float32)), "int4", "i32")
    got = parity.to_np(acc)
    assert np.all(got[:, 0] == 64 * k) and np.all(got[:, 1] == -56 * k)


# ---------------------------------------------------------------- NVFP4 GEMM on identical codes
def _rand_nvfp4_operands(m, k, seed, g):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((m, k))
    x[:, 3] *= 20
    e, s, _, _ = quant.nvfp4_rows(x, g)
    return e, s


def _dev_nvfp4(e, s, g):
    return (torch.from_numpy(quant.pack_nibbles(e)).cuda(), torch.from_numpy(s.astype(np.uint8)).cuda(),
            torch.tensor([g], dtype=torch.float32).cuda())


@pytest.mark.parametrize("m,n,k", [(64, 256, 512), (1100, 4200, 512), (300, 600, 4096), (5, 40, 256)])
def test_nvfp4_gemm_y(rq, m, n, k):
    gx, gw = np.float32(0.0071), np.float32(0.00013)
    ex, sx = _rand_nvfp4_operands(m, k, m + k, gx)
    ew, sw = _rand_nvfp4_operands(n, k, n + 3 * k, gw)
    y = rq.w4a4_gemm(_dev_nvfp4(ex, sx, gx), _dev_nvfp4(ew, sw, gw), "nvfp4", "f32")
    torch.cuda.synchronize()
    ref = gemm.nvfp4_y(ex, sx, gx, ew, sw, gw)
    err = parity.check_y(parity.to_np(y), ref, tol=1e-5)
    assert err < 1e-5


@pytest.mark.parametrize("m,n,k", [(1100, 4200, 512), (5, 40, 256), (300, 300, 1024), (2048, 4096, 4096)])
def test_nvfp4_gemm_bf16(rq, m, n, k):
    """bf16 Y: each element within one bf16 step of the rounded oracle value
    (rows of 16-byte multiples go through the TMA-store epilogue, others not)."""
    gx, gw = np.float32(0.0071), np.float32(0.00013)
    ex, sx = _rand_nvfp4_operands(m, k, 5 * m + k, gx)
    ew, sw = _rand_nvfp4_operands(n, k, n + 7 * k, gw)
    y = rq.w4a4_gemm(_dev_nvfp4(ex, sx, gx), _dev_nvfp4(ew, sw, gw), "nvfp4", "bf16")
    torch.cuda.synchronize()
    ref = gemm.nvfp4_y(ex, sx, gx, ew, sw, gw)
    absterms = np.abs(quant.nvfp4_dequant(ex, sx, gx)) @ np.abs(quant.nvfp4_dequant(ew, sw, gw)).T
    parity.check_bf16_y(y.float().cpu().numpy(), ref, absterms, k)


# ---------------------------------------------------------------- end to end: X, W -> Y
@pytest.mark.parametrize("fmt,block", [("int4", 128), ("int4", 0), ("nvfp4", 128)])
def test_end_to_end(rq, fmt, block):
    name = "tiny_int4"
    x = syn.activations(name)
    w = syn.weights(name)
    s = syn.workload_signs(name)
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
    else:
        gx, gw = quant.nvfp4_global_scale(xr), quant.nvfp4_global_scale(wr)
        ex, sx, tex, tsx = quant.nvfp4_rows(xr, gx)
        ew, sw, tew, tsw = quant.nvfp4_rows(wr, gw)
        ref = gemm.nvfp4_y(ex, sx, gx, ew, sw, gw)
        xh, dx = parity.nvfp4_tie_bounds(ex, sx, gx, tex, tsx)
        wh, dw = parity.nvfp4_tie_bounds(ew, sw, gw, tew, tsw)
    parity.check_y_with_ties(parity.to_np(y), ref, xh, dx, wh, dw)
    rq.get_device_error()
