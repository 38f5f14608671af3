"""GPU parity of the MXFP4 path (E2M1 values, E8M0 power-of-two scale per 32):
the fused rotation + quantization and the block-scaled FP4 GEMM
(tcgen05 kind::mxf4), against the fp64 oracle.  All calls go through the C ABI.

"Rotations for 4-Bit Activations: QuaRot, SpinQuant, and Friends", sections
"The full model in NVFP4, on vLLM" and "When to rotate" (MXFP4: scales that
are powers of two shared by 32 values; rotations help it).
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


@pytest.mark.parametrize("m,k", [(64, 512), (333, 4096), (2048, 4096), (77, 12288), (9, 128)])
def test_mxfp4_rotate_quantize(rq, m, k):
    x = _gauss(m, k, 500 + m, outliers=[(11, 30.0), (k - 5, 45.0)])
    s = syn.signs(k, 600 + k)
    codes, sc, g = rq.rotate_quantize(x.cuda(), s.cuda(), 128, "mxfp4")
    torch.cuda.synchronize()
    assert g is None and tuple(sc.shape) == (m, k // 32)
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128)
    parity.check_mxfp4_quant(parity.to_np(codes), parity.to_np(sc), xr)


def test_mxfp4_zero_onehot_and_strided_rows(rq):
    k = 512
    big = torch.zeros((6, k + 128))
    big[1, 3] = 2.0
    big[2, 200] = -0.25
    big[3, :] = torch.linspace(-1e-3, 1e-3, k + 128)
    big[4, 64] = 3.0e4
    big = big.to(torch.bfloat16)
    s = syn.signs(k, 78)
    codes, sc, _ = rq.rotate_quantize(big.cuda()[:, :k], s.cuda(), 128, "mxfp4")
    xr = hadamard.rotate(parity.bf16_to_f64(big[:, :k]), s.numpy(), 128)
    parity.check_mxfp4_quant(parity.to_np(codes), parity.to_np(sc), xr)
    assert np.all(parity.to_np(codes)[0] == 0) and np.all(parity.to_np(sc)[0] == 0)


def test_prepare_weights_mxfp4(rq):
    name = "q_proj_int4"
    w = syn.weights(name, rows=384)
    s = syn.workload_signs(name)
    codes, sc, g = rq.prepare_weights(w.cuda(), s.cuda(), 128, "mxfp4")
    torch.cuda.synchronize()
    assert g is None
    wr = hadamard.rotate(parity.bf16_to_f64(w), s.numpy(), 128)
    parity.check_mxfp4_quant(parity.to_np(codes), parity.to_np(sc), wr)


# ---------------------------------------------------------------- GEMM on identical codes
def _rand_mx_operands(m, k, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((m, k)) * np.exp(rng.uniform(-3, 3, size=(m, 1)))
    x[:, 7] *= 25
    e, s, _, _ = quant.mxfp4_rows(x)
    return e, s


def _dev_mx(e, s):
    return (torch.from_numpy(quant.pack_nibbles(e)).cuda(), torch.from_numpy(s.astype(np.uint8)).cuda(), None)


@pytest.mark.parametrize("m,n,k", [(64, 256, 512), (1100, 4200, 512), (300, 600, 4096), (5, 40, 1024),
                                   (256, 256, 1536)])
def test_mxfp4_gemm_y(rq, m, n, k):
    ex, sx = _rand_mx_operands(m, k, m + k)
    ew, sw = _rand_mx_operands(n, k, n + 3 * k)
    y = rq.w4a4_gemm(_dev_mx(ex, sx), _dev_mx(ew, sw), "mxfp4", "f32")
    torch.cuda.synchronize()
    ref = gemm.mxfp4_y(ex, sx, ew, sw)
    # fp32 accumulation of exact products: gamma_K * sum |x w| per element
    absterms = np.abs(quant.mxfp4_dequant(ex, sx)) @ np.abs(quant.mxfp4_dequant(ew, sw)).T
    gamma = k * 2.0 ** -24 / (1 - k * 2.0 ** -24)
    got = parity.to_np(y).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2 * gamma * absterms + 1e-30)
    assert parity.check_y(got, ref, tol=1e-5) < 1e-5


@pytest.mark.parametrize("m,n,k", [(1100, 4200, 512), (2048, 4096, 4096), (5, 40, 512)])
def test_mxfp4_gemm_bf16(rq, m, n, k):
    ex, sx = _rand_mx_operands(m, k, 5 * m + k)
    ew, sw = _rand_mx_operands(n, k, n + 7 * k)
    y = rq.w4a4_gemm(_dev_mx(ex, sx), _dev_mx(ew, sw), "mxfp4", "bf16")
    torch.cuda.synchronize()
    ref = gemm.mxfp4_y(ex, sx, ew, sw)
    absterms = np.abs(quant.mxfp4_dequant(ex, sx)) @ np.abs(quant.mxfp4_dequant(ew, sw)).T
    parity.check_bf16_y(y.float().cpu().numpy(), ref, absterms, k)


def test_mxfp4_gemm_rejects_k_not_multiple_of_512(rq):
    ex, sx = _rand_mx_operands(8, 256, 1)
    with pytest.raises(rq.RQError) as e:
        rq.w4a4_gemm(_dev_mx(ex, sx), _dev_mx(ex, sx), "mxfp4", "f32")
    assert e.value.status == 2


def test_mxfp4_end_to_end(rq):
    name = "tiny_int4"
    x, w, s = syn.activations(name), syn.weights(name), syn.workload_signs(name)
    wq = rq.prepare_weights(w.cuda(), s.cuda(), 128, "mxfp4")
    xq = rq.rotate_quantize(x.cuda(), s.cuda(), 128, "mxfp4")
    y = rq.w4a4_gemm(xq, wq, "mxfp4", "f32")
    torch.cuda.synchronize()
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), 128)
    wr = hadamard.rotate(parity.bf16_to_f64(w), s.numpy(), 128)
    ex, sx, tex, tsx = quant.mxfp4_rows(xr)
    ew, sw, tew, tsw = quant.mxfp4_rows(wr)
    ref = gemm.mxfp4_y(ex, sx, ew, sw)
    xh, dx = parity.mxfp4_tie_bounds(ex, sx, tex, tsx)
    wh, dw = parity.mxfp4_tie_bounds(ew, sw, tew, tsw)
    parity.check_y_with_ties(parity.to_np(y), ref, xh, dx, wh, dw)
    rq.get_device_error()
