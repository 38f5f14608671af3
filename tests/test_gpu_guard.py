"""GPU: guard bands around every output (compute-sanitizer is closed here).

Each output is a view into a larger buffer whose surroundings -- 4 KiB before
and after, and the padding columns of a strided Y -- are filled with 0xA5; after
the call every guard byte must be intact, for ragged shapes (rows and columns
that are not multiples of the tiles) of every entry point.  The values
themselves are checked by the parity tests.
"""

import pytest
import torch

from rotation_w4a4_quantization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

PAD = 4096
CANARY = 0xA5


@pytest.fixture(scope="module")
def rq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rotation_w4a4_quantization_b200 import rq as m
    m.init(0)
    return m


class Guarded:
    """A tensor of `shape` / `dtype` (last dimension padded to `ld` elements)
    carved out of a canary-filled byte buffer."""

    def __init__(self, shape, dtype, ld=None):
        esz = torch.empty((), dtype=dtype).element_size()
        rows = 1
        for d in shape[:-1]:
            rows *= d
        self.ld = ld or shape[-1]
        nbytes = rows * self.ld * esz
        self.buf = torch.full((PAD + nbytes + PAD,), CANARY, dtype=torch.uint8, device="cuda")
        flat = self.buf[PAD:PAD + nbytes].view(dtype)
        full = flat.view(*shape[:-1], self.ld)
        self.t = full[..., :shape[-1]]
        self.full_bytes = self.buf[PAD:PAD + nbytes].view(rows, self.ld * esz)
        self.inner = shape[-1] * esz

    def intact(self):
        torch.cuda.synchronize()
        ok = bool((self.buf[:PAD] == CANARY).all()) and bool((self.buf[-PAD:] == CANARY).all())
        if self.inner < self.full_bytes.shape[1]:
            ok = ok and bool((self.full_bytes[:, self.inner:] == CANARY).all())
        return ok


def _x(m, k, seed=1):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((m, k), generator=g)
    x[:, 3] *= 30
    return x.to(torch.bfloat16).cuda()


@pytest.mark.parametrize("fmt,block,m,k", [("int4", 128, 37, 512), ("int4", 0, 33, 4096), ("int4", 0, 5, 1024),
                                           ("int8", 128, 37, 384), ("int8", 0, 70, 4096), ("nvfp4", 128, 37, 512),
                                           ("nvfp4", 16, 301, 4096), ("mxfp4", 32, 37, 512),
                                           ("int4_asym", 128, 37, 640)])
def test_rotate_quantize_guards(rq, fmt, block, m, k):
    x = _x(m, k)
    s = syn.signs(k, 3).cuda()
    if fmt in ("int8",):
        codes, scales = Guarded((m, k), torch.int8), Guarded((m,), torch.float32)
    elif fmt == "int4_asym":
        codes, scales = Guarded((m, k // 2), torch.uint8), Guarded((m, k // 128, 2), torch.float16)
    else:
        codes = Guarded((m, k // 2), torch.uint8)
        scales = Guarded((m,), torch.float32) if fmt == "int4" else \
            Guarded((m, k // (16 if fmt == "nvfp4" else 32)), torch.uint8)
    g = Guarded((1,), torch.float32)
    rq.rotate_quantize(x, s, block, fmt, gscale=g.t if fmt == "nvfp4" else None, out=(codes.t, scales.t))
    assert codes.intact() and scales.intact() and g.intact()
    rq.get_device_error()


@pytest.mark.parametrize("block,m,k", [(128, 37, 512), (0, 33, 4096), (16, 9, 256)])
def test_rotate_f32_guards_strided(rq, block, m, k):
    x = _x(m, k, 5)
    s = syn.signs(k, 6).cuda()
    out = Guarded((m, k), torch.float32, ld=k + 36)
    rq.rotate_f32(x, s, block, out=out.t)
    assert out.intact()


GEMM_CASES = [(fmt, m, n, k, out) for fmt, m, n, k in [("int4", 300, 520, 512), ("int4", 100, 264, 256),
                                                        ("nvfp4", 300, 520, 512), ("mxfp4", 300, 264, 1024)]
              for out in (("f32", "bf16", "i32") if fmt == "int4" else ("f32", "bf16"))]


@pytest.mark.parametrize("fmt,m,n,k,out", GEMM_CASES)
def test_gemm_guards(rq, fmt, m, n, k, out):
    s = syn.signs(k, 7).cuda()
    xq = rq.rotate_quantize(_x(m, k, 8), s, 128, fmt)
    wq = rq.prepare_weights(_x(n, k, 9), s, 128, fmt)
    dt = {"f32": torch.float32, "bf16": torch.bfloat16, "i32": torch.int32}[out]
    y = Guarded((m, n), dt, ld=n + 24)
    rq.w4a4_gemm(xq, wq, fmt, out, y=y.t)
    assert y.intact()
    rq.get_device_error()


@pytest.mark.parametrize("xf,wf", [("int8", "int4"), ("int8", "int8")])
def test_int_gemm_guards(rq, xf, wf):
    m, n, k = 300, 520, 512
    s = syn.signs(k, 10).cuda()
    xq = rq.rotate_quantize(_x(m, k, 11), s, 128, xf)
    wq = rq.prepare_weights(_x(n, k, 12), s, 128, wf)
    y = Guarded((m, n), torch.bfloat16, ld=n + 8)
    rq.int_gemm(xq, xf, wq, wf, "bf16", y=y.t)
    assert y.intact()


def test_kv_and_attention_guards(rq):
    b, h, t = 2, 3, 1100
    s = syn.signs(128, 13).cuda()
    k = syn.kv(batch=b, heads=h, seq=t, which=0).cuda()
    v = syn.kv(batch=b, heads=h, seq=t, which=1).cuda()
    kc = (Guarded((b, h, t, 64), torch.uint8), Guarded((b, h, t), torch.float16), Guarded((b, h, t), torch.float16))
    rq.kv_rotate_quantize(k, s, out=tuple(g.t for g in kc))
    assert all(g.intact() for g in kc)
    vc = rq.kv_rotate_quantize(v, s)
    q = torch.randn((b, h, 128), device="cuda").to(torch.bfloat16)
    nws = int(rq.lib.rq_kv4_attention_workspace_bytes(b, h, t))
    ws = Guarded((nws,), torch.uint8)
    out = Guarded((b, h, 128), torch.float32)
    rq.kv4_decode_attention(q, tuple(g.t for g in kc), vc, s, out=out.t, workspace=ws.t)
    assert out.intact() and ws.intact()
    rq.get_device_error()
