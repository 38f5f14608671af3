"""GPU parity: 6- and 8-bit round to nearest (W8A8, W6A6) and W4A8.

The rotate kernel's INT6 / INT8 modes against the oracle's per-row symmetric
quantizer on the same rotated inputs (codes equal except at flagged rounding
ties), the integer GEMM with 8-bit activation codes against exact integer
sums (bit-exact int32 accumulators, Y within 1e-6), and the whole path from
bf16 X and W to Y ("QuaRot (rotation-based outlier removal, W4A4KV4)", field
"Bits"; "SpinQuant (learned rotations + W4A4KV4)", field "Activation scheme").
"""

import numpy as np
import pytest
import torch

import parity
from oracle import gemm, hadamard, quant
from rotation_w4a4_quantization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

BITS = {"int8": 8, "int6": 6, "int4": 4}


@pytest.fixture(scope="module")
def rq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rotation_w4a4_quantization_b200 import rq as m
    m.init(0)
    return m


def _planted(m, k, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((m, k), generator=g)
    x[:, (7 * seed) % k] *= 40.0
    return x.to(torch.bfloat16)


# ---------------------------------------------------------------- rotate + 6/8-bit quantize
@pytest.mark.parametrize("fmt", ["int8", "int6"])
@pytest.mark.parametrize("m,k,block", [(37, 512, 128), (300, 4096, 128), (129, 256, 0), (70, 4096, 0),
                                       (5, 1024, 0), (1, 12288, 128)])
def test_rotate_quantize_int(rq, fmt, m, k, block):
    x = _planted(m, k, m + k)
    s = syn.signs(k, seed=k + 1)
    codes, scales, _ = rq.rotate_quantize(x.cuda(), s.cuda(), block, fmt)
    torch.cuda.synchronize()
    assert codes.dtype == torch.int8 and codes.shape == (m, k)
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), block)
    parity.check_int_quant(parity.to_np(codes), parity.to_np(scales), xr, BITS[fmt])


@pytest.mark.parametrize("fmt", ["int8", "int6"])
def test_rotate_quantize_int_zero_and_strided_rows(rq, fmt):
    big = _planted(40, 768, 3)
    big[5] = 0
    view = big.cuda()[:, :640]                   # row stride 768 > K
    s = syn.signs(640, seed=11)
    codes, scales, _ = rq.rotate_quantize(view, s.cuda(), 128, fmt)
    torch.cuda.synchronize()
    xr = hadamard.rotate(parity.bf16_to_f64(big[:, :640]), s.numpy(), 128)
    parity.check_int_quant(parity.to_np(codes), parity.to_np(scales), xr, BITS[fmt])
    assert parity.to_np(scales)[5] == 0 and np.all(parity.to_np(codes)[5] == 0)


# ---------------------------------------------------------------- integer GEMM on identical codes
def _operands(m, n, k, bx, bw, seed):
    rng = np.random.default_rng(seed)
    qx = rng.integers(-(2 ** (bx - 1)) + 1, 2 ** (bx - 1), size=(m, k))
    qw = rng.integers(-(2 ** (bw - 1)) + 1, 2 ** (bw - 1), size=(n, k))
    sx = (rng.random(m) + 0.5).astype(np.float32) / (2 ** (bx - 1) - 1)
    sw = (rng.random(n) * 0.01 + 0.001).astype(np.float32)
    return qx, qw, sx, sw


def _dev(q, s, bits):
    if bits == 4:
        codes = torch.from_numpy(quant.pack_nibbles(q)).cuda()
    else:
        codes = torch.from_numpy(q.astype(np.int8)).cuda()
    return codes, torch.from_numpy(s).cuda(), None


PAIRS = [("int8", "int4"), ("int8", "int8"), ("int6", "int6"), ("int6", "int4"), ("int8", "int6")]


@pytest.mark.parametrize("xf,wf", PAIRS)
@pytest.mark.parametrize("m,n,k", [(300, 600, 512), (64, 256, 128), (257, 513, 1152), (5, 40, 256)])
def test_int_gemm_acc_bit_exact(rq, xf, wf, m, n, k):
    bx, bw = BITS[xf], BITS[wf]
    qx, qw, sx, sw = _operands(m, n, k, bx, bw, m + n + k + bx * bw)
    acc = rq.int_gemm(_dev(qx, sx, bx), xf, _dev(qw, sw, bw), wf, "i32")
    torch.cuda.synchronize()
    ref = gemm.int_acc(qx, qw)
    got = parity.to_np(acc).astype(np.int64)
    assert np.array_equal(got, ref), np.argwhere(got != ref)[:5]


@pytest.mark.parametrize("xf,wf", [("int8", "int4"), ("int8", "int8"), ("int6", "int6")])
def test_int_gemm_y_f32_and_bf16(rq, xf, wf):
    m, n, k = 1100, 2100, 1024
    bx, bw = BITS[xf], BITS[wf]
    qx, qw, sx, sw = _operands(m, n, k, bx, bw, 99 + bx + bw)
    xq, wq = _dev(qx, sx, bx), _dev(qw, sw, bw)
    y = rq.int_gemm(xq, xf, wq, wf, "f32")
    yb = rq.int_gemm(xq, xf, wq, wf, "bf16")
    torch.cuda.synchronize()
    ref = gemm.int4_y(gemm.int_acc(qx, qw), sx, sw)
    assert parity.check_y(parity.to_np(y), ref, tol=1e-6) < 1e-6
    ybf = yb.float().cpu().numpy().astype(np.float64)
    rb = parity.bf16_round(ref)
    assert np.all(np.abs(ybf - rb) <= np.abs(rb) * 2.0 ** -7 + 1e-30)


def test_int_gemm_extremes(rq):
    """-128 everywhere (valid int8, never produced by the quantizer): |acc| = 2^14 K,
    and 127 x -8 rows for W4A8."""
    m, n, k = 128, 256, 8192
    one_m, one_n = np.ones(m, np.float32), np.ones(n, np.float32)
    acc = rq.int_gemm(_dev(np.full((m, k), -128), one_m, 8), "int8", _dev(np.full((n, k), -128), one_n, 8), "int8",
                      "i32")
    assert np.all(parity.to_np(acc) == 16384 * k)
    qw = np.full((n, k), -8)
    qw[1] = 7
    acc = rq.int_gemm(_dev(np.full((m, k), 127), one_m, 8), "int8", _dev(qw, one_n, 4), "int4", "i32")
    got = parity.to_np(acc)
    assert np.all(got[:, 0] == -1016 * k) and np.all(got[:, 1] == 889 * k)


def test_int_gemm_rejects_unsupported_pair(rq):
    qx, qw, sx, sw = _operands(128, 256, 256, 4, 8, 1)
    with pytest.raises(rq.RQError) as e:
        rq.int_gemm(_dev(qx, sx, 4), "int4", _dev(qw, sw, 8), "int8", "f32")
    assert e.value.status == 2


# ---------------------------------------------------------------- end to end: X, W -> Y
@pytest.mark.parametrize("xf,wf,block", [("int8", "int4", 128), ("int8", "int4", 0), ("int8", "int8", 128),
                                         ("int6", "int6", 0)])
def test_end_to_end(rq, xf, wf, block):
    name = "tiny_int4"
    x = syn.activations(name)
    w = syn.weights(name)
    s = syn.workload_signs(name)
    xq = rq.rotate_quantize(x.cuda(), s.cuda(), block, xf)
    wq = rq.prepare_weights(w.cuda(), s.cuda(), block, wf)
    y = rq.int_gemm(xq, xf, wq, wf, "f32")
    torch.cuda.synchronize()
    xd, wd = parity.bf16_to_f64(x), parity.bf16_to_f64(w)
    xr, wr = hadamard.rotate(xd, s.numpy(), block), hadamard.rotate(wd, s.numpy(), block)
    qx, sx, tx = quant.int_sym_rows(xr, BITS[xf])
    qw, sw, tw = quant.int_sym_rows(wr, BITS[wf])
    ref = gemm.int4_y(gemm.int_acc(qx, qw), sx, sw)
    xh, dx = parity.int4_tie_bounds(qx, sx, tx)
    wh, dw = parity.int4_tie_bounds(qw, sw, tw)
    parity.check_y_with_ties(parity.to_np(y), ref, xh, dx, wh, dw)
    rq.get_device_error()


def test_w4a8_full_size_sampled(rq):
    """q_proj shape (M 2048, N 4096, K 4096), W4A8 in the launch the bench times:
    sampled rows of Y against the oracle on the GPU's own codes."""
    name = "q_proj_int4"
    c = syn.WORKLOADS[name]
    x = syn.activations(name, device="cuda")
    w = syn.weights(name, device="cuda")
    s = syn.workload_signs(name).cuda()
    xq = rq.rotate_quantize(x, s, c["block"], "int8")
    wq = rq.prepare_weights(w, s, c["block"], "int4")
    y = rq.int_gemm(xq, "int8", wq, "int4", "bf16")
    torch.cuda.synchronize()
    rows = np.random.default_rng(5).choice(c["M"], 24, replace=False)
    qx = parity.to_np(xq[0])[rows].astype(np.int64)
    sx = parity.to_np(xq[1])[rows]
    qw = quant.unpack_nibbles(parity.to_np(wq[0]), signed=True)
    ref = gemm.int4_y(gemm.int_acc(qx, qw), sx, parity.to_np(wq[1]))
    got = y.float().cpu().numpy()[rows].astype(np.float64)
    rb = parity.bf16_round(ref)
    assert np.all(np.abs(got - rb) <= np.abs(rb) * 2.0 ** -7 + 1e-30)
