"""GPU parity: INT4 weights stored one code per byte (RQ_INT4_BYTES).

The W4A4 product of "Rotations for 4-Bit Activations: QuaRot, SpinQuant, and
Friends", section "What it buys in 4 bits, and what it doesn't", with the
weights' INT4 codes kept one per byte: the same codes and per-output-channel
scales as the packed layout (so the same oracle), which the two-SM integer
GEMM feeds to the tensor cores without widening.  Checked: the codes and
scales equal the packed path's and the oracle's, the int32 accumulators are
bit-exact against the integer triple loop, and Y equals the packed-weight
W4A4 GEMM's Y bit for bit (the same integer sums and the same epilogue
arithmetic).
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


@pytest.mark.parametrize("block", [0, 128, 16, 1])
@pytest.mark.parametrize("m,k", [(37, 512), (300, 4096), (5, 12288)])
def test_byte_codes_equal_packed_codes(rq, block, m, k):
    if block == 0 and k == 12288:
        pytest.skip("full width needs a power of two")
    w = _gauss(m, k, m + k + block, outliers=[(3, 30.0)])
    s = syn.signs(k, k + 3)
    cb, sb, _ = rq.prepare_weights(w.cuda(), s.cuda(), block, "int4_bytes")
    cp, sp, _ = rq.prepare_weights(w.cuda(), s.cuda(), block, "int4")
    torch.cuda.synchronize()
    unpacked = quant.unpack_nibbles(parity.to_np(cp), signed=True)
    assert np.array_equal(parity.to_np(cb).astype(np.int64), unpacked)
    assert torch.equal(sb, sp)
    wr = hadamard.rotate(parity.bf16_to_f64(w), s.numpy(), block)
    parity.check_int4_quant(parity.to_np(cp), parity.to_np(sp), wr)


@pytest.mark.parametrize("m,n,k", [(300, 600, 512), (1100, 4200, 512), (257, 513, 1152), (5, 40, 256),
                                   (2048, 512, 4096)])
def test_byte_weight_gemm_acc_bit_exact(rq, m, n, k):
    rng = np.random.default_rng(m + n + k)
    qx = rng.integers(-7, 8, size=(m, k))
    qw = rng.integers(-7, 8, size=(n, k))
    sx = (rng.random(m) + 0.5).astype(np.float32) / 7
    sw = (rng.random(n) * 0.01 + 0.001).astype(np.float32)
    xq = (torch.from_numpy(quant.pack_nibbles(qx)).cuda(), torch.from_numpy(sx).cuda(), None)
    wq = (torch.from_numpy(qw.astype(np.int8)).cuda(), torch.from_numpy(sw).cuda(), None)
    acc = rq.int_gemm(xq, "int4", wq, "int4_bytes", "i32")
    torch.cuda.synchronize()
    ref = gemm.int4_acc(qx, qw)
    got = parity.to_np(acc).astype(np.int64)
    assert np.array_equal(got, ref), np.argwhere(got != ref)[:5]


@pytest.mark.parametrize("name", ["tiny_int4", "q_proj_int4"])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_byte_weight_gemm_equals_packed_gemm(rq, name, out):
    c = syn.WORKLOADS[name]
    rows = min(c["M"], 512)
    x = syn.activations(name, rows=rows)
    w = syn.weights(name, rows=min(c["N"], 768))
    s = syn.workload_signs(name)
    block = c["block"]
    xq = rq.rotate_quantize(x.cuda(), s.cuda(), block, "int4")
    wp = rq.prepare_weights(w.cuda(), s.cuda(), block, "int4")
    wb = rq.prepare_weights(w.cuda(), s.cuda(), block, "int4_bytes")
    yp = rq.w4a4_gemm(xq, wp, "int4", out)
    yb = rq.int_gemm(xq, "int4", wb, "int4_bytes", out)
    torch.cuda.synchronize()
    assert torch.equal(yp, yb)
    # and Y against the oracle's W4A4 product, beyond the tie bounds
    xr = hadamard.rotate(parity.bf16_to_f64(x), s.numpy(), block)
    wr = hadamard.rotate(parity.bf16_to_f64(w), s.numpy(), block)
    qx, sx, tx = quant.int4_sym_rows(xr)
    qw, sw, tw = quant.int4_sym_rows(wr)
    ref = gemm.int4_y(gemm.int4_acc(qx, qw), sx, sw)
    xh, dx = parity.int4_tie_bounds(qx, sx, tx)
    wh, dw = parity.int4_tie_bounds(qw, sw, tw)
    if out == "f32":
        parity.check_y_with_ties(parity.to_np(yb), ref, xh, dx, wh, dw)
    rq.get_device_error()
