"""CPU checks of the C-ABI boundary: the library loads, exports every entry
point that include/rq.h declares, and rejects bad arguments on the host with
the documented status -- before any CUDA call, so no GPU is needed.
"""

import ctypes
import os
import re

import pytest

from conftest import ROOT

rq = pytest.importorskip("rotation_w4a4_quantization_b200.rq")
lib = rq.lib

INVALID, SHAPE, ALIGN = 1, 2, 3
P = ctypes.c_void_p
A16 = P(0x10000)      # a 16-byte aligned fake device address (never dereferenced)
A8 = P(0x10008)


def declared_functions():
    with open(os.path.join(ROOT, "include", "rq.h")) as f:
        text = f.read()
    return re.findall(r"RQ_API\s+[\w\s\*]+?\b(rq_\w+)\s*\(", text)


def test_header_matches_exports():
    names = declared_functions()
    assert sorted(names) == sorted(rq.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for s in range(7):
        assert lib.rq_status_string(s)
    assert lib.rq_status_string(99) == b"unknown status"


def test_workspace_bytes():
    assert lib.rq_workspace_bytes(rq.RQ_INT4) == 0
    assert lib.rq_workspace_bytes(rq.RQ_NVFP4) == 16


def rotq(x=A16, m=4, k=512, ldx=512, signs=A16, block=128, fmt=0, gmode=0, codes=A16, scales=A16, g=A16, ws=A16):
    return lib.rq_rotate_quantize(x, m, k, ldx, signs, block, fmt, gmode, codes, scales, g, ws, None)


def test_rotate_quantize_rejections():
    assert rotq(x=None) == INVALID
    assert rotq(signs=None) == INVALID
    assert rotq(codes=None) == INVALID
    assert rotq(m=-1) == INVALID
    assert rotq(ldx=100) == INVALID                 # ldx < K
    assert rotq(k=500, ldx=500) == SHAPE            # K not a multiple of 128
    assert rotq(k=65536, ldx=65536) == SHAPE        # above the supported K
    assert rotq(block=64) == SHAPE
    assert rotq(k=384, ldx=384, block=0) == SHAPE   # full width needs a power of two
    assert rotq(k=8192, ldx=8192, block=0) == SHAPE
    assert rotq(x=P(0x10002)) == ALIGN
    assert rotq(ldx=516) == ALIGN                   # row pitch not a multiple of 16 bytes
    assert rotq(codes=A8) == ALIGN
    assert rotq(signs=A8) == ALIGN                 # the sign vector is read 16 bytes at a time
    assert rotq(fmt=7) == INVALID
    assert rotq(gmode=5) == INVALID
    assert rotq(fmt=1, block=0) == SHAPE            # NVFP4 needs 128-wide blocks
    assert rotq(fmt=1, g=None) == INVALID
    assert rotq(fmt=1, ws=None) == INVALID          # dynamic NVFP4 needs the workspace
    assert rotq(fmt=1, scales=P(0x10004)) == ALIGN


def test_rotate_quantize_empty_is_noop():
    assert rotq(m=0) == 0


def test_prepare_weights_and_rotate_f32_rejections():
    assert lib.rq_prepare_weights(None, 4, 512, 512, A16, 128, 0, A16, A16, A16, A16, None) == INVALID
    assert lib.rq_prepare_weights(A16, 4, 500, 500, A16, 128, 0, A16, A16, A16, A16, None) == SHAPE
    assert lib.rq_rotate_f32(A16, 4, 512, 512, A16, 128, None, 512, None) == INVALID
    assert lib.rq_rotate_f32(A16, 4, 512, 512, A16, 128, A16, 510, None) == INVALID   # ldo < K
    assert lib.rq_rotate_f32(A16, 4, 512, 512, A16, 128, A16, 514, None) == ALIGN
    assert lib.rq_rotate_f32(A16, 0, 512, 512, A16, 128, A16, 512, None) == 0


def gemm(xc=A16, xs=A16, xg=A16, wc=A16, ws=A16, wg=A16, m=128, n=256, k=512, fmt=0, y=A16, ldy=256, out=0):
    return lib.rq_w4a4_gemm(xc, xs, xg, wc, ws, wg, m, n, k, fmt, y, ldy, out, None)


def test_gemm_rejections():
    assert gemm(xc=None) == INVALID
    assert gemm(y=None) == INVALID
    assert gemm(m=-1) == INVALID
    assert gemm(ldy=100) == INVALID
    assert gemm(fmt=3) == INVALID
    assert gemm(out=9) == INVALID
    assert gemm(fmt=1, out=2) == INVALID           # raw accumulators are INT4 only
    assert gemm(fmt=1, xg=None) == INVALID
    assert gemm(k=192) == SHAPE                    # INT4 K multiple of 128
    assert gemm(fmt=1, k=384) == SHAPE             # NVFP4 K multiple of 256
    assert gemm(k=131072) == SHAPE
    assert gemm(xc=A8) == ALIGN
    assert gemm(y=P(0x10002)) == ALIGN             # fp32 Y must be 4-byte aligned
    assert gemm(m=0) == 0 and gemm(n=0) == 0


def kv(x=A16, b=2, h=2, s=8, d=128, strides=(4096, 1024, 128), signs=A16, codes=A16, sc=A16, zr=A16):
    arr = None if strides is None else (ctypes.c_int64 * 3)(*strides)
    return lib.rq_kv_rotate_quantize(x, b, h, s, d, arr, signs, codes, sc, zr, None)


def test_kv_rejections():
    assert kv(x=None) == INVALID
    assert kv(strides=None) == INVALID
    assert kv(b=-1) == INVALID
    assert kv(d=64) == SHAPE
    assert kv(strides=(4096, 1024, 130)) == ALIGN  # vectors must stay 16-byte aligned
    assert kv(sc=P(0x10001)) == ALIGN
    assert kv(signs=A8) == ALIGN
    assert kv(strides=(4096, -1, 128)) == INVALID
    assert kv(s=0) == 0


def test_init_without_gpu_reports_unsupported_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert lib.rq_init(0) == 4


def igemm(xc=A16, xs=A16, xf=3, wc=A16, ws=A16, wf=0, m=256, n=256, k=512, y=A16, ldy=256, out=0):
    return lib.rq_int_gemm(xc, xs, xf, wc, ws, wf, m, n, k, y, ldy, out, None)


def test_int_gemm_rejections():
    assert igemm(xf=1) == INVALID                  # NVFP4 is not an integer format
    assert igemm(wf=5) == INVALID                  # per-group asymmetric codes have no GEMM
    assert igemm(xf=0, wf=3) == SHAPE              # 4-bit activations with wider weights
    assert igemm(xf=3, wf=6) == INVALID            # the byte layout of INT4 weights pairs with INT4 activations
    assert igemm(xf=0, wf=6, k=192) == SHAPE       # W4A4 with byte weights: K a multiple of 128
    assert igemm(xf=0, wf=6, m=0) == 0
    assert igemm(xf=0, wf=0, k=192) == SHAPE       # W4A4 goes through the W4A4 GEMM's checks
    assert igemm(ldy=100) == INVALID
    assert igemm(out=9) == INVALID
    assert igemm(xc=None) == INVALID
    assert igemm(k=192) == SHAPE
    assert igemm(k=65536 + 128) == SHAPE
    assert igemm(xc=A8) == ALIGN
    assert igemm(y=P(0x10002)) == ALIGN            # fp32 Y 4-byte aligned
    assert igemm(ws=P(0x10004)) == ALIGN           # weight scales read 16 bytes at a time
    assert igemm(m=0) == 0 and igemm(n=0) == 0


def attn(q=A16, b=2, h=4, s=1500, kc=A16, ks=A16, kz=A16, vc=A16, vs=A16, vz=A16, signs=A16, scale=0.0, o=A16,
         out=0, ws=A16):
    return lib.rq_kv4_decode_attention(q, b, h, s, kc, ks, kz, vc, vs, vz, signs, scale, o, out, ws, None)


def test_decode_attention_rejections():
    assert attn(b=-1) == INVALID
    assert attn(out=2) == INVALID                  # fp32 or bf16 output only
    assert attn(scale=-1.0) == INVALID
    assert attn(scale=float("inf")) == INVALID
    assert attn(scale=float("nan")) == INVALID
    assert attn(b=0) == 0 and attn(h=0) == 0       # nothing to do
    assert attn(s=0) == INVALID                    # a softmax over no tokens
    assert attn(q=None) == INVALID
    assert attn(ws=None) == INVALID
    assert attn(vz=None) == INVALID
    assert attn(q=A8) == ALIGN
    assert attn(ks=P(0x10001)) == ALIGN
    assert attn(o=P(0x10002)) == ALIGN             # fp32 output 4-byte aligned
    assert attn(o=P(0x10001), out=1) == ALIGN      # bf16 output 2-byte aligned
    assert attn(b=1 << 20, h=1 << 11, s=1024) == SHAPE   # more partial records than a grid holds


def test_decode_attention_workspace_bytes():
    wsb = lib.rq_kv4_attention_workspace_bytes
    assert wsb(0, 4, 100) == 0 and wsb(2, 0, 100) == 0 and wsb(2, 4, 0) == 0
    one = wsb(1, 1, 1)
    assert one > 0 and one % 16 == 0
    assert wsb(1, 1, 1024) == one                  # one record per 1024 cached tokens
    assert wsb(1, 1, 1025) == 2 * one
    assert wsb(2, 4, 1500) == 2 * 4 * 2 * one


def test_noalloc_and_selftest_rejections():
    f = lib.rq_rotate_quantize_nvfp4_noalloc
    assert f(None, 4, 512, 512, A16, A16, A16, A16, None) == INVALID
    assert f(A16, 4, 500, 500, A16, A16, A16, A16, None) == SHAPE
    assert f(A16, 0, 512, 512, A16, A16, A16, A16, None) == 0
    assert lib.rq_selftest_wait_timeout(0, None) == INVALID
    assert lib.rq_selftest_wait_timeout(-5, None) == INVALID
    assert lib.rq_selftest_wait_timeout(1 << 40, None) == INVALID    # above the kernels' own limit


def test_rotate_quantize_format_rules():
    assert rotq(fmt=7) == INVALID                  # no such format
    assert rotq(fmt=6, m=0) == 0                   # INT4 codes one per byte
    assert rotq(fmt=6, scales=P(0x10002)) == ALIGN  # its fp32 scales
    assert rotq(fmt=2, block=0) == SHAPE           # MXFP4 needs block-diagonal rotation
    assert rotq(fmt=5, block=0) == SHAPE           # so do per-group asymmetric codes
    assert rotq(fmt=3, block=64) == SHAPE          # blocks of 16, 32, 128 or the full width
    assert rotq(fmt=3, m=0) == 0 and rotq(fmt=4, m=0) == 0 and rotq(fmt=5, m=0) == 0
    assert rotq(fmt=3, scales=P(0x10002)) == ALIGN  # fp32 scales


# ---------------------------------------------------------------- the binding's own checks
# The Python binding checks what the C ABI cannot see -- dtypes, inner strides
# and the sizes of caller-passed buffers -- and raises ValueError before any
# library call.  These run on CPU tensors: the checks come before the
# CUDA-tensor check, so each message names the real problem.
import torch  # noqa: E402


def _bf16(m, k):
    return torch.zeros((m, k), dtype=torch.bfloat16)


def _s(k):
    return torch.ones(k, dtype=torch.int8)


def _raises(match, fn, *a, **kw):
    with pytest.raises(ValueError, match=match):
        fn(*a, **kw)


def test_binding_checks_rotate_quantize_inputs():
    _raises("bfloat16", rq.rotate_quantize, torch.zeros((4, 512)), _s(512))              # fp32 X
    _raises("stride", rq.rotate_quantize, _bf16(512, 4).t(), _s(512))                   # column-strided X
    _raises("2-D", rq.rotate_quantize, torch.zeros((2, 4, 512), dtype=torch.bfloat16), _s(512))
    _raises("signs", rq.rotate_quantize, _bf16(4, 512), _s(256))                        # short signs
    _raises("signs", rq.rotate_quantize, _bf16(4, 512), torch.ones(512, dtype=torch.int32))
    _raises("CUDA", rq.rotate_quantize, _bf16(4, 512), _s(512))                         # all right but on the host


def test_binding_checks_rotate_quantize_outputs():
    x, s = _bf16(4, 512), _s(512)
    ok_codes = torch.empty((4, 256), dtype=torch.uint8)
    _raises("codes", rq.rotate_quantize, x, s, out=(torch.empty((4, 255), dtype=torch.uint8),
                                                    torch.empty(4, dtype=torch.float32)))
    _raises("scales", rq.rotate_quantize, x, s, out=(ok_codes, torch.empty(3, dtype=torch.float32)))
    _raises("scales", rq.rotate_quantize, x, s, fmt="nvfp4", out=(ok_codes, torch.empty((4, 16), dtype=torch.uint8)))
    _raises("codes", rq.rotate_quantize, x, s, fmt="int8", out=(ok_codes, torch.empty(4, dtype=torch.float32)))
    _raises("workspace", rq.rotate_quantize, x, s, fmt="nvfp4", workspace=torch.empty(8, dtype=torch.uint8))
    _raises("gscale", rq.rotate_quantize, x, s, fmt="nvfp4", gscale=torch.empty(1, dtype=torch.float64))
    _raises("gscale", rq.rotate_quantize, x, s, fmt="nvfp4", gmode="static")
    _raises("codes", rq.prepare_weights, x, s, out=(torch.empty((256, 4), dtype=torch.uint8).t(),
                                                    torch.empty(4, dtype=torch.float32)))


def test_binding_checks_gemm_operands():
    xq = (torch.empty((8, 256), dtype=torch.uint8), torch.empty(8, dtype=torch.float32), None)
    wq = (torch.empty((16, 256), dtype=torch.uint8), torch.empty(16, dtype=torch.float32), None)
    wq_k = (torch.empty((16, 128), dtype=torch.uint8), torch.empty(16, dtype=torch.float32), None)
    _raises("disagree on K", rq.w4a4_gemm, xq, wq_k, "int4")
    _raises("scales", rq.w4a4_gemm, xq, (wq[0], torch.empty(15, dtype=torch.float32), None), "int4")
    _raises("scales", rq.w4a4_gemm, xq, wq, "nvfp4")                                    # INT4 scales as NVFP4
    _raises("gscale", rq.w4a4_gemm, (xq[0], torch.empty((8, 32), dtype=torch.uint8), None),
            (wq[0], torch.empty((16, 32), dtype=torch.uint8), None), "nvfp4")
    _raises("y must be", rq.w4a4_gemm, xq, wq, "int4", "f32", y=torch.empty((8, 15), dtype=torch.float32))
    _raises("y must be", rq.w4a4_gemm, xq, wq, "int4", "bf16", y=torch.empty((8, 16), dtype=torch.float32))
    _raises("int4, nvfp4 or mxfp4", rq.w4a4_gemm, xq, wq, "int8")
    _raises("CUDA", rq.w4a4_gemm, xq, wq, "int4")
    x8 = (torch.empty((8, 512), dtype=torch.int8), torch.empty(8, dtype=torch.float32))
    _raises("disagree on K", rq.int_gemm, x8, "int8", wq_k, "int4")
    _raises("codes", rq.int_gemm, (torch.empty((8, 512), dtype=torch.uint8), x8[1]), "int8", wq, "int4")
    _raises("CUDA", rq.int_gemm, x8, "int8", wq, "int4")
    # INT4 weights in the byte layout: one int8 code per channel, K columns
    x4 = (torch.empty((8, 256), dtype=torch.uint8), torch.empty(8, dtype=torch.float32))
    wb = (torch.empty((16, 512), dtype=torch.int8), torch.empty(16, dtype=torch.float32))
    _raises("disagree on K", rq.int_gemm, x4, "int4", (torch.empty((16, 256), dtype=torch.int8), wb[1]),
            "int4_bytes")                                                            # packed width passed as bytes
    _raises("codes", rq.int_gemm, x4, "int4", (torch.empty((16, 512), dtype=torch.uint8), wb[1]), "int4_bytes")
    _raises("int4, int6 or int8", rq.int_gemm, wb, "int4_bytes", wb, "int4_bytes")     # activations never bytes
    _raises("CUDA", rq.int_gemm, x4, "int4", wb, "int4_bytes")


def test_binding_checks_kv_and_attention():
    kv = torch.zeros((1, 2, 8, 128), dtype=torch.bfloat16)
    _raises("head_dim", rq.kv_rotate_quantize, torch.zeros((1, 2, 8, 64), dtype=torch.bfloat16), _s(64))
    _raises("bf16", rq.kv_rotate_quantize, kv.float(), _s(128))
    _raises("signs", rq.kv_rotate_quantize, kv, _s(64))
    _raises("scale", rq.kv_rotate_quantize, kv, _s(128), out=(torch.empty((1, 2, 8, 64), dtype=torch.uint8),
                                                              torch.empty((1, 2, 7), dtype=torch.float16),
                                                              torch.empty((1, 2, 8), dtype=torch.float16)))
    cache = (torch.empty((1, 2, 8, 64), dtype=torch.uint8), torch.empty((1, 2, 8), dtype=torch.float16),
             torch.empty((1, 2, 8), dtype=torch.float16))
    q = torch.zeros((1, 2, 128), dtype=torch.bfloat16)
    _raises("q", rq.kv4_decode_attention, q.float(), cache, cache, _s(128))
    _raises("v codes", rq.kv4_decode_attention, q, cache, (cache[0][:, :, :4], cache[1], cache[2]), _s(128))
    _raises("workspace", rq.kv4_decode_attention, q, cache, cache, _s(128), workspace=torch.empty(16, dtype=torch.uint8))
    _raises("out", rq.kv4_decode_attention, q, cache, cache, _s(128), out=torch.empty((1, 2, 128), dtype=torch.bfloat16))
    _raises("CUDA", rq.kv4_decode_attention, q, cache, cache, _s(128))


def test_binding_checks_rotate_f32_and_noalloc():
    _raises("out", rq.rotate_f32, _bf16(4, 512), _s(512), out=torch.empty((4, 500), dtype=torch.float32))
    _raises("signs", rq.rotate_f32, _bf16(4, 512), _s(128))
    _raises("scales", rq.rotate_quantize_nvfp4_noalloc, _bf16(4, 512), _s(512),
            out=(torch.empty((4, 256), dtype=torch.uint8), torch.empty((4, 16), dtype=torch.uint8)))
    _raises("CUDA", rq.rotate_quantize_nvfp4_noalloc, _bf16(4, 512), _s(512))
