"""GPU: the hot path captured into a CUDA graph and replayed on new inputs gives
the same bytes as the eager calls (the kernels are deterministic, and their
programmatic-dependent launches become graph edges that keep stream order)."""

import pytest
import torch

from rotation_w4a4_quantization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rotation_w4a4_quantization_b200 import rq as m
    m.init(0)
    return m


@pytest.mark.parametrize("name, block, fmt, gmode", [
    ("q_proj_int4", 0, "int4", "dynamic"),
    ("q_proj_int4", 128, "int4", "dynamic"),
    ("q_proj_mxfp4", 128, "mxfp4", "dynamic"),
    ("q_proj_nvfp4", 128, "nvfp4", "static"),
])
def test_rotate_gemm_graph_replay(rq, name, block, fmt, gmode):
    m, n = 520, 384  # several tiles and a ragged tail in both dimensions
    sg = syn.workload_signs(name).cuda()
    w = syn.weights(name, rows=n).cuda()
    wq = rq.prepare_weights(w, sg, block=block, fmt=fmt)
    x0 = syn.activations(name, rows=m).cuda()
    x1 = syn.activations(name, rows=m, seed_offset=7).cuda()
    gs = None
    if fmt == "nvfp4":  # static per-tensor scale: the one dynamic mode finds for the second input
        gs = rq.rotate_quantize(x1, sg, block=block, fmt=fmt, gmode="dynamic")[2].clone()

    # eager on the second input
    xq_ref = rq.rotate_quantize(x1, sg, block=block, fmt=fmt, gmode=gmode, gscale=gs)
    y_ref = rq.w4a4_gemm(xq_ref, wq, fmt=fmt, out="bf16")
    torch.cuda.synchronize()

    # capture on static buffers holding the first input, then replay on the second
    x = x0.clone()
    codes, scales = torch.empty_like(xq_ref[0]), torch.empty_like(xq_ref[1])
    y = torch.empty_like(y_ref)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # one eager pass to settle one-time set-up outside the capture
        xq = rq.rotate_quantize(x, sg, block=block, fmt=fmt, gmode=gmode, gscale=gs, out=(codes, scales))
        rq.w4a4_gemm(xq, wq, fmt=fmt, out="bf16", y=y)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        xq = rq.rotate_quantize(x, sg, block=block, fmt=fmt, gmode=gmode, gscale=gs, out=(codes, scales))
        rq.w4a4_gemm(xq, wq, fmt=fmt, out="bf16", y=y)
    x.copy_(x1)
    codes.zero_()
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(codes, xq_ref[0])
    assert torch.equal(scales, xq_ref[1])
    assert torch.equal(y, y_ref)
    # and a second replay is idempotent
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    del g


def test_kv4_and_decode_attention_graph_replay(rq):
    b, h, s = 2, 4, 1500
    sg = syn.workload_signs("kv4").cuda()
    k0, v0 = syn.kv(b, h, s, which=0).cuda(), syn.kv(b, h, s, which=1).cuda()
    k1, v1 = syn.kv(b, h, s, which=0, seed_offset=3).cuda(), syn.kv(b, h, s, which=1, seed_offset=3).cuda()
    q1 = syn.kv(b, h, 1, which=0, seed_offset=5).reshape(b, h, 128).cuda()
    kc_ref = rq.kv_rotate_quantize(k1, sg)
    vc_ref = rq.kv_rotate_quantize(v1, sg)
    o_ref = rq.kv4_decode_attention(q1, kc_ref, vc_ref, sg)
    torch.cuda.synchronize()

    kk, vv, q = k0.clone(), v0.clone(), torch.zeros_like(q1)
    kc = tuple(torch.empty_like(t) for t in kc_ref)
    vc = tuple(torch.empty_like(t) for t in vc_ref)
    o = torch.empty_like(o_ref)
    ws = torch.empty((max(int(rq.lib.rq_kv4_attention_workspace_bytes(b, h, s)), 16),), dtype=torch.uint8,
                     device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        rq.kv_rotate_quantize(kk, sg, out=kc)
        rq.kv_rotate_quantize(vv, sg, out=vc)
        rq.kv4_decode_attention(q, kc, vc, sg, out=o, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        rq.kv_rotate_quantize(kk, sg, out=kc)
        rq.kv_rotate_quantize(vv, sg, out=vc)
        rq.kv4_decode_attention(q, kc, vc, sg, out=o, workspace=ws)
    kk.copy_(k1)
    vv.copy_(v1)
    q.copy_(q1)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    for a, r in zip(kc + vc, kc_ref + vc_ref):
        assert torch.equal(a, r)
    assert torch.equal(o, o_ref)
    del g
