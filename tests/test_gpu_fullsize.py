"""GPU parity at the benchmarked sizes, in the launch configuration bench.py times.

The bench's own synthetic inputs at full size (q_proj 2048 x 4096 x 4096 with a
full-width rotation, down_proj 4096 x 12288 x 4096 with 128-blocks, the kv4
cache [16, 32, 4096, 128] and a decode step over it), checked on sampled rows
that the oracle computes one by one: the rotated + quantized codes of sampled
activation and weight rows against the oracle's rotation and quantizer, and
sampled rows of Y against exact integer sums of the GPU's own codes (within
one bf16 step); sampled (batch, head) slices of the KV4 cache and of the
attention output against the oracle.
"""

import numpy as np
import pytest
import torch

import parity
from oracle import attention, gemm, hadamard, quant
from rotation_w4a4_quantization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rotation_w4a4_quantization_b200 import rq as m
    m.init(0)
    return m


@pytest.mark.parametrize("name,nrows", [("q_proj_int4", 12), ("down_proj_int4", 8)])
def test_int4_workload_sampled(rq, name, nrows):
    c = syn.WORKLOADS[name]
    x = syn.activations(name, device="cuda")
    w = syn.weights(name, device="cuda")
    s = syn.workload_signs(name)
    xq = rq.rotate_quantize(x, s.cuda(), c["block"], "int4")
    wq = rq.prepare_weights(w, s.cuda(), c["block"], "int4")
    y = rq.w4a4_gemm(xq, wq, "int4", "bf16")
    torch.cuda.synchronize()
    rng = np.random.default_rng(c["index"])
    rows = np.sort(rng.choice(c["M"], nrows, replace=False))
    wrows = np.sort(rng.choice(c["N"], nrows, replace=False))
    # codes and scales of sampled X and W rows against the oracle
    xr = hadamard.rotate(parity.bf16_to_f64(x[rows].cpu()), s.numpy(), c["block"])
    parity.check_int4_quant(parity.to_np(xq[0])[rows], parity.to_np(xq[1])[rows], xr)
    wr = hadamard.rotate(parity.bf16_to_f64(w[wrows].cpu()), s.numpy(), c["block"])
    parity.check_int4_quant(parity.to_np(wq[0])[wrows], parity.to_np(wq[1])[wrows], wr)
    # sampled rows of Y against exact sums of the GPU's codes
    qx = quant.unpack_nibbles(parity.to_np(xq[0])[rows], signed=True)
    qw = quant.unpack_nibbles(parity.to_np(wq[0]), signed=True)
    ref = gemm.int4_y(gemm.int4_acc(qx, qw), parity.to_np(xq[1])[rows], parity.to_np(wq[1]))
    got = y.float().cpu().numpy()[rows].astype(np.float64)
    rb = parity.bf16_round(ref)
    assert np.all(np.abs(got - rb) <= np.abs(rb) * 2.0 ** -7 + 1e-30)
    rq.get_device_error()


def test_kv4_workload_sampled(rq):
    c = syn.WORKLOADS["kv4"]
    s = syn.workload_signs("kv4")
    k = syn.kv(device="cuda", which=0)
    codes, scale, zero = rq.kv_rotate_quantize(k, s.cuda())
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    for b, h in zip(rng.integers(0, c["B"], 4), rng.integers(0, c["H"], 4)):
        kr = hadamard.rotate(parity.bf16_to_f64(k[b, h].cpu()), s.numpy(), 128)
        parity.check_kv4(parity.to_np(codes[b, h]), parity.to_np(scale[b, h]).astype(np.float64),
                         parity.to_np(zero[b, h]).astype(np.float64), kr)
    rq.get_device_error()


def test_kv4_decode_workload_sampled(rq):
    c = syn.WORKLOADS["kv4_decode"]
    s = syn.workload_signs("kv4_decode")
    kc = rq.kv_rotate_quantize(syn.kv(device="cuda", which=0), s.cuda())
    vc = rq.kv_rotate_quantize(syn.kv(device="cuda", which=1), s.cuda())
    g = torch.Generator(device="cuda")
    g.manual_seed(4000 + c["index"])
    q = torch.randn((c["B"], c["H"], c["D"]), generator=g, device="cuda").to(torch.bfloat16)
    out = rq.kv4_decode_attention(q, kc, vc, s.cuda())
    torch.cuda.synchronize()
    rng = np.random.default_rng(6)
    for b, h in zip(rng.integers(0, c["B"], 4), rng.integers(0, c["H"], 4)):
        sl = lambda t: parity.to_np(t[b:b + 1, h:h + 1])
        kq = quant.unpack_nibbles(sl(kc[0]), signed=False)
        vq = quant.unpack_nibbles(sl(vc[0]), signed=False)
        ref = attention.kv4_decode_attention(parity.bf16_to_f64(q[b:b + 1, h:h + 1].cpu()), kq,
                                             sl(kc[1]).astype(np.float64), sl(kc[2]).astype(np.float64), vq,
                                             sl(vc[1]).astype(np.float64), sl(vc[2]).astype(np.float64), s.numpy())
        got = parity.to_np(out[b:b + 1, h:h + 1]).astype(np.float64)
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-5
    rq.get_device_error()
