"""Thin Python binding of librq (include/rq.h): argument marshalling only.

Every computation runs in the CUDA kernels of librq.so; this module only
allocates output tensors with PyTorch, passes raw device pointers, sizes and
the current CUDA stream, and turns status codes into exceptions.  There is no
CPU fallback: if librq.so is missing or fails to load, importing this module
raises.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librq.so")

RQ_INT4, RQ_NVFP4, RQ_MXFP4, RQ_INT8, RQ_INT6, RQ_INT4_ASYM, RQ_INT4_BYTES = 0, 1, 2, 3, 4, 5, 6
RQ_OUT_F32, RQ_OUT_BF16, RQ_OUT_I32_ACC = 0, 1, 2
RQ_SCALE_DYNAMIC, RQ_SCALE_STATIC = 0, 1
STATUS = {0: "RQ_OK", 1: "RQ_ERR_INVALID_ARG", 2: "RQ_ERR_UNSUPPORTED_SHAPE", 3: "RQ_ERR_ALIGNMENT",
          4: "RQ_ERR_UNSUPPORTED_DEVICE", 5: "RQ_ERR_CUDA", 6: "RQ_ERR_TIMEOUT"}
EXPORTED = ["rq_init", "rq_status_string", "rq_workspace_bytes", "rq_rotate_quantize", "rq_prepare_weights",
            "rq_w4a4_gemm", "rq_kv_rotate_quantize", "rq_rotate_f32", "rq_get_device_error",
            "rq_rotate_quantize_nvfp4_noalloc", "rq_kv4_attention_workspace_bytes", "rq_kv4_decode_attention",
            "rq_int_gemm", "rq_selftest_wait_timeout"]

if not os.path.exists(LIB_PATH):
    raise ImportError("librq.so not built: run `python -m rotation_w4a4_quantization_b200.build`")
lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_i = ctypes.c_int
lib.rq_init.argtypes = [_i]
lib.rq_init.restype = _i
lib.rq_status_string.argtypes = [_i]
lib.rq_status_string.restype = ctypes.c_char_p
lib.rq_workspace_bytes.argtypes = [_i]
lib.rq_workspace_bytes.restype = ctypes.c_size_t
lib.rq_rotate_quantize.argtypes = [_p, _i64, _i64, _i64, _p, _i, _i, _i, _p, _p, _p, _p, _p]
lib.rq_rotate_quantize.restype = _i
lib.rq_prepare_weights.argtypes = [_p, _i64, _i64, _i64, _p, _i, _i, _p, _p, _p, _p, _p]
lib.rq_prepare_weights.restype = _i
lib.rq_w4a4_gemm.argtypes = [_p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i, _p, _i64, _i, _p]
lib.rq_w4a4_gemm.restype = _i
lib.rq_int_gemm.argtypes = [_p, _p, _i, _p, _p, _i, _i64, _i64, _i64, _p, _i64, _i, _p]
lib.rq_int_gemm.restype = _i
lib.rq_kv_rotate_quantize.argtypes = [_p, _i64, _i64, _i64, _i64, ctypes.POINTER(_i64), _p, _p, _p, _p, _p]
lib.rq_kv_rotate_quantize.restype = _i
lib.rq_rotate_f32.argtypes = [_p, _i64, _i64, _i64, _p, _i, _p, _i64, _p]
lib.rq_rotate_f32.restype = _i
lib.rq_rotate_quantize_nvfp4_noalloc.argtypes = [_p, _i64, _i64, _i64, _p, _p, _p, _p, _p]
lib.rq_rotate_quantize_nvfp4_noalloc.restype = _i
lib.rq_kv4_attention_workspace_bytes.argtypes = [_i64, _i64, _i64]
lib.rq_kv4_attention_workspace_bytes.restype = ctypes.c_size_t
lib.rq_kv4_decode_attention.argtypes = [_p, _i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, ctypes.c_float, _p, _i, _p, _p]
lib.rq_kv4_decode_attention.restype = _i
lib.rq_selftest_wait_timeout.argtypes = [_i64, _p]
lib.rq_selftest_wait_timeout.restype = _i
lib.rq_get_device_error.argtypes = [_p]
lib.rq_get_device_error.restype = _i


class RQError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        msg = lib.rq_status_string(status).decode()
        super().__init__("%s failed: %s (%s)" % (what, STATUS.get(status, status), msg))


def _check(status, what):
    if status != 0:
        raise RQError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t=None):
    dev = t.device if t is not None else torch.device("cuda")
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _fmt(fmt):
    if isinstance(fmt, str):
        return {"int4": RQ_INT4, "nvfp4": RQ_NVFP4, "mxfp4": RQ_MXFP4, "int8": RQ_INT8, "int6": RQ_INT6,
                "int4_asym": RQ_INT4_ASYM, "int4_bytes": RQ_INT4_BYTES}[fmt]
    return int(fmt)


def init(device=0):
    _check(lib.rq_init(int(device)), "rq_init")


def workspace_bytes(fmt):
    return int(lib.rq_workspace_bytes(_fmt(fmt)))


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("librq takes CUDA tensors only")


# Host-side checks of what the C ABI cannot see (dtypes, inner strides and the
# sizes of caller-passed buffers), so that a mismatch raises ValueError here
# instead of making a kernel read or write out of bounds.
def _expect(t, shape, dtype, name, contiguous=True):
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if contiguous and not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _expect_matrix_bf16(x, name):
    if x.dim() != 2:
        raise ValueError("%s must be 2-D [rows, K], got %d-D" % (name, x.dim()))
    if x.dtype != torch.bfloat16:
        raise ValueError("%s must be torch.bfloat16, got %s" % (name, x.dtype))
    if x.shape[0] > 0 and x.stride(1) != 1:
        raise ValueError("%s rows must be contiguous (stride(1) == 1)" % name)


def _expect_signs(signs, k):
    _expect(signs, (k,), torch.int8, "signs")


def _expect_bytes(t, nbytes, name):
    if not t.is_contiguous() or t.numel() * t.element_size() < nbytes:
        raise ValueError("%s must be a contiguous buffer of at least %d bytes" % (name, nbytes))


def _quant_shapes(rows, k, fmt):
    """(codes shape, codes dtype, scales shape, scales dtype) that a format writes."""
    if fmt in (RQ_INT8, RQ_INT6, RQ_INT4_BYTES):
        return (rows, k), torch.int8, (rows,), torch.float32
    if fmt == RQ_INT4_ASYM:
        return (rows, k // 2), torch.uint8, (rows, k // 128, 2), torch.float16
    if fmt == RQ_INT4:
        return (rows, k // 2), torch.uint8, (rows,), torch.float32
    if fmt == RQ_NVFP4:
        return (rows, k // 2), torch.uint8, (rows, k // 16), torch.uint8
    if fmt == RQ_MXFP4:
        return (rows, k // 2), torch.uint8, (rows, k // 32), torch.uint8
    raise ValueError("unknown format %r" % fmt)


def _expect_quant_outputs(out, rows, k, fmt):
    cs, cd, ss, sd = _quant_shapes(rows, k, fmt)
    codes, scales = out
    _expect(codes, cs, cd, "codes")
    _expect(scales, ss, sd, "scales")


def _expect_quantized(q, rows, k, fmt, name):
    """A (codes, scales, gscale) triple as rotate_quantize / prepare_weights return it."""
    _expect_quant_outputs((q[0], q[1]), rows, k, fmt)
    if fmt == RQ_NVFP4:
        if q[2] is None:
            raise ValueError("%s: NVFP4 needs its per-tensor scale (gscale)" % name)
        _expect(q[2].reshape(-1)[:1], (1,), torch.float32, name + " gscale", contiguous=False)


def _expect_output_matrix(y, m, n, dtype):
    if y.dtype != dtype or y.dim() != 2 or y.shape[0] != m or y.shape[1] < n or (m > 0 and y.stride(1) != 1):
        raise ValueError("y must be %s [M, >= N] with contiguous rows" % dtype)


def _alloc_quant_outputs(rows, k, fmt, device):
    if fmt in (RQ_INT8, RQ_INT6, RQ_INT4_BYTES):  # one int8 code per byte
        return (torch.empty((rows, k), dtype=torch.int8, device=device),
                torch.empty((rows,), dtype=torch.float32, device=device))
    codes = torch.empty((rows, k // 2), dtype=torch.uint8, device=device)
    if fmt == RQ_INT4_ASYM:  # fp16 (scale, zero) per group of 128
        return codes, torch.empty((rows, k // 128, 2), dtype=torch.float16, device=device)
    if fmt == RQ_INT4:
        scales = torch.empty((rows,), dtype=torch.float32, device=device)
    elif fmt == RQ_NVFP4:
        scales = torch.empty((rows, k // 16), dtype=torch.uint8, device=device)
    else:
        scales = torch.empty((rows, k // 32), dtype=torch.uint8, device=device)
    return codes, scales


def rotate_quantize(x, signs, block=128, fmt="int4", gmode="dynamic", gscale=None, out=None, workspace=None):
    """X [M, K] bf16 (row stride ldx) -> (codes, scales, gscale).

    INT4: codes uint8 [M, K/2], scales fp32 [M], gscale None.
    NVFP4: codes uint8 [M, K/2] (E2M1), scales uint8 [M, K/16] (E4M3), gscale fp32 [1].
    MXFP4: codes uint8 [M, K/2] (E2M1), scales uint8 [M, K/32] (E8M0), gscale None.
    INT8 / INT6: codes int8 [M, K] (one code per byte), scales fp32 [M], gscale None.
    INT4_ASYM: codes uint8 [M, K/2] (unsigned nibbles), scales fp16 [M, K/128, 2] = (scale, zero).
    """
    f = _fmt(fmt)
    _expect_matrix_bf16(x, "x")
    m, k = x.shape
    _expect_signs(signs, k)
    if out is not None:
        _expect_quant_outputs(out, m, k, f)
    if gmode not in ("dynamic", "static"):
        raise ValueError("gmode must be 'dynamic' or 'static'")
    gm = RQ_SCALE_DYNAMIC if gmode == "dynamic" else RQ_SCALE_STATIC
    if gscale is not None:
        _expect_bytes(gscale, 4, "gscale")
        if gscale.dtype != torch.float32:
            raise ValueError("gscale must be torch.float32")
    if workspace is not None:
        _expect_bytes(workspace, workspace_bytes(f), "workspace")
    if f == RQ_NVFP4 and gscale is None and gm == RQ_SCALE_STATIC:
        raise ValueError("static NVFP4 scaling needs gscale")
    _require_cuda(x, signs, gscale, workspace, *(out or ()))
    codes, scales = out if out is not None else _alloc_quant_outputs(m, k, f, x.device)
    if f == RQ_NVFP4:
        if gscale is None:
            gscale = torch.empty((1,), dtype=torch.float32, device=x.device)
        if workspace is None and gm == RQ_SCALE_DYNAMIC:
            workspace = torch.empty((16,), dtype=torch.uint8, device=x.device)
    _check(lib.rq_rotate_quantize(_ptr(x), m, k, x.stride(0), _ptr(signs), int(block), f, gm, _ptr(codes),
                                  _ptr(scales), _ptr(gscale), _ptr(workspace), _stream(x)), "rq_rotate_quantize")
    return codes, scales, gscale


def prepare_weights(w, signs, block=128, fmt="int4", out=None, workspace=None):
    """W [N, K] bf16 -> (codes, scales, gscale), the offline weight side."""
    f = _fmt(fmt)
    _expect_matrix_bf16(w, "w")
    n, k = w.shape
    _expect_signs(signs, k)
    if out is not None:
        _expect_quant_outputs(out, n, k, f)
    if workspace is not None:
        _expect_bytes(workspace, workspace_bytes(f), "workspace")
    _require_cuda(w, signs, workspace, *(out or ()))
    codes, scales = out if out is not None else _alloc_quant_outputs(n, k, f, w.device)
    gscale = torch.empty((1,), dtype=torch.float32, device=w.device) if f == RQ_NVFP4 else None
    if f == RQ_NVFP4 and workspace is None:
        workspace = torch.empty((16,), dtype=torch.uint8, device=w.device)
    _check(lib.rq_prepare_weights(_ptr(w), n, k, w.stride(0), _ptr(signs), int(block), f, _ptr(codes), _ptr(scales),
                                  _ptr(gscale), _ptr(workspace), _stream(w)), "rq_prepare_weights")
    return codes, scales, gscale


def w4a4_gemm(xq, wq, fmt="int4", out="f32", y=None):
    """Y = deq(xq) . deq(wq)^T with xq / wq the (codes, scales, gscale) triples."""
    xc, xs, xg = xq
    wc, ws, wg = wq
    f = _fmt(fmt)
    if f not in (RQ_INT4, RQ_NVFP4, RQ_MXFP4):
        raise ValueError("w4a4_gemm takes int4, nvfp4 or mxfp4 codes")
    o = {"f32": RQ_OUT_F32, "bf16": RQ_OUT_BF16, "i32": RQ_OUT_I32_ACC}[out]
    if xc.dim() != 2 or wc.dim() != 2:
        raise ValueError("codes must be 2-D")
    m, kh = xc.shape
    n = wc.shape[0]
    if wc.shape[1] != kh:
        raise ValueError("X and W codes disagree on K: %d vs %d" % (2 * kh, 2 * wc.shape[1]))
    _expect_quantized(xq, m, 2 * kh, f, "xq")
    _expect_quantized(wq, n, 2 * kh, f, "wq")
    dt = {RQ_OUT_F32: torch.float32, RQ_OUT_BF16: torch.bfloat16, RQ_OUT_I32_ACC: torch.int32}[o]
    if y is not None:
        _expect_output_matrix(y, m, n, dt)
    _require_cuda(xc, xs, xg, wc, ws, wg, y)
    if y is None:
        y = torch.empty((m, n), dtype=dt, device=xc.device)
    _check(lib.rq_w4a4_gemm(_ptr(xc), _ptr(xs), _ptr(xg), _ptr(wc), _ptr(ws), _ptr(wg), m, n, 2 * kh, f, _ptr(y),
                            y.stride(0), o, _stream(xc)), "rq_w4a4_gemm")
    return y


def int_gemm(xq, xfmt, wq, wfmt, out="f32", y=None):
    """Y = deq(xq) . deq(wq)^T for integer codes of different widths (W4A8, W6A6,
    W8A8, W4A4): xq / wq are (codes, scales, _) triples from rotate_quantize /
    prepare_weights with formats xfmt / wfmt in {"int4", "int6", "int8"}; W4A4
    also takes wfmt "int4_bytes" (the INT4 weight codes one per byte)."""
    xc, xs = xq[0], xq[1]
    wc, ws = wq[0], wq[1]
    fx, fw = _fmt(xfmt), _fmt(wfmt)
    if fx not in (RQ_INT4, RQ_INT6, RQ_INT8) or fw not in (RQ_INT4, RQ_INT6, RQ_INT8, RQ_INT4_BYTES):
        raise ValueError("int_gemm takes int4, int6 or int8 codes (int4_bytes for the weights)")
    o = {"f32": RQ_OUT_F32, "bf16": RQ_OUT_BF16, "i32": RQ_OUT_I32_ACC}[out]
    if xc.dim() != 2 or wc.dim() != 2:
        raise ValueError("codes must be 2-D")
    m, n = xc.shape[0], wc.shape[0]
    k = xc.shape[1] * (2 if fx == RQ_INT4 else 1)
    kw = wc.shape[1] * (2 if fw == RQ_INT4 else 1)
    if kw != k:
        raise ValueError("X and W codes disagree on K: %d vs %d" % (k, kw))
    _expect_quant_outputs((xc, xs), m, k, fx)
    _expect_quant_outputs((wc, ws), n, k, fw)
    dt = {RQ_OUT_F32: torch.float32, RQ_OUT_BF16: torch.bfloat16, RQ_OUT_I32_ACC: torch.int32}[o]
    if y is not None:
        _expect_output_matrix(y, m, n, dt)
    _require_cuda(xc, xs, wc, ws, y)
    if y is None:
        y = torch.empty((m, n), dtype=dt, device=xc.device)
    _check(lib.rq_int_gemm(_ptr(xc), _ptr(xs), fx, _ptr(wc), _ptr(ws), fw, m, n, k, _ptr(y), y.stride(0), o,
                           _stream(xc)), "rq_int_gemm")
    return y


def kv_rotate_quantize(kv, signs, out=None):
    """K or V [B, H, S, 128] bf16 (head_dim contiguous) -> (codes [B,H,S,64], scale fp16 [B,H,S], zero fp16 [B,H,S])."""
    if kv.dim() != 4 or kv.dtype != torch.bfloat16:
        raise ValueError("kv must be bf16 [B, H, S, 128]")
    b, h, s, d = kv.shape
    if d != 128:
        raise ValueError("head_dim must be 128")
    if kv.stride(3) != 1:
        raise ValueError("head_dim must be contiguous")
    _expect_signs(signs, d)
    if out is not None:
        _expect(out[0], (b, h, s, d // 2), torch.uint8, "codes")
        _expect(out[1], (b, h, s), torch.float16, "scale")
        _expect(out[2], (b, h, s), torch.float16, "zero")
    _require_cuda(kv, signs, *(out or ()))
    if out is None:
        codes = torch.empty((b, h, s, d // 2), dtype=torch.uint8, device=kv.device)
        scale = torch.empty((b, h, s), dtype=torch.float16, device=kv.device)
        zero = torch.empty((b, h, s), dtype=torch.float16, device=kv.device)
    else:
        codes, scale, zero = out
    strides = (ctypes.c_int64 * 3)(kv.stride(0), kv.stride(1), kv.stride(2))
    _check(lib.rq_kv_rotate_quantize(_ptr(kv), b, h, s, d, strides, _ptr(signs), _ptr(codes), _ptr(scale),
                                     _ptr(zero), _stream(kv)), "rq_kv_rotate_quantize")
    return codes, scale, zero


def rotate_f32(x, signs, block=128, out=None):
    """X.Q as fp32 [M, K]."""
    _expect_matrix_bf16(x, "x")
    m, k = x.shape
    _expect_signs(signs, k)
    if out is not None:
        if out.dtype != torch.float32 or out.dim() != 2 or out.shape[0] != m or out.shape[1] < k or (
                m > 0 and out.stride(1) != 1):
            raise ValueError("out must be fp32 [M, >= K] with contiguous rows")
    _require_cuda(x, signs, out)
    if out is None:
        out = torch.empty((m, k), dtype=torch.float32, device=x.device)
    _check(lib.rq_rotate_f32(_ptr(x), m, k, x.stride(0), _ptr(signs), int(block), _ptr(out), out.stride(0),
                             _stream(x)), "rq_rotate_f32")
    return out


def rotate_quantize_nvfp4_noalloc(x, signs, out=None, gscale=None):
    """NVFP4 (128-wide blocks, dynamic per-tensor scale) without any device
    workspace: for callers that cannot allocate device memory.  Returns
    (codes, scales, gscale) like rotate_quantize; outputs may be passed in."""
    _expect_matrix_bf16(x, "x")
    m, k = x.shape
    _expect_signs(signs, k)
    if out is not None:
        _expect_quant_outputs(out, m, k, RQ_NVFP4)
    if gscale is not None:
        _expect_bytes(gscale, 4, "gscale")
    _require_cuda(x, signs, gscale, *(out or ()))
    codes, scales = out if out is not None else _alloc_quant_outputs(m, k, RQ_NVFP4, x.device)
    if gscale is None:
        gscale = torch.empty((1,), dtype=torch.float32, device=x.device)
    _check(lib.rq_rotate_quantize_nvfp4_noalloc(_ptr(x), m, k, x.stride(0), _ptr(signs), _ptr(codes), _ptr(scales),
                                                _ptr(gscale), _stream(x)), "rq_rotate_quantize_nvfp4_noalloc")
    return codes, scales, gscale


def kv4_decode_attention(q, kcache, vcache, signs, softmax_scale=0.0, out_dtype="f32", out=None, workspace=None):
    """One decode step over the KV4 cache.  q bf16 [B, H, 128]; kcache / vcache
    the (codes [B,H,S,64], scale fp16 [B,H,S], zero fp16 [B,H,S]) triples of
    kv_rotate_quantize.  Returns o [B, H, 128] (fp32 or bf16) in the original
    basis."""
    kc, ks, kz = kcache
    vc, vs, vz = vcache
    if q.dim() != 3 or kc.dim() != 4:
        raise ValueError("q must be [B, H, 128] and the cache codes [B, H, S, 64]")
    b, h, d = q.shape
    s = kc.shape[2]
    _expect(q, (b, h, 128), torch.bfloat16, "q")
    for c, sc, z, nm in ((kc, ks, kz, "k"), (vc, vs, vz, "v")):
        _expect(c, (b, h, s, 64), torch.uint8, nm + " codes")
        _expect(sc, (b, h, s), torch.float16, nm + " scale")
        _expect(z, (b, h, s), torch.float16, nm + " zero")
    _expect_signs(signs, 128)
    o = {"f32": RQ_OUT_F32, "bf16": RQ_OUT_BF16}[out_dtype]
    odt = torch.float32 if o == RQ_OUT_F32 else torch.bfloat16
    if out is not None:
        _expect(out, (b, h, d), odt, "out")
    nb = int(lib.rq_kv4_attention_workspace_bytes(b, h, s))
    if workspace is not None:
        _expect_bytes(workspace, nb, "workspace")
    _require_cuda(q, kc, ks, kz, vc, vs, vz, signs, out, workspace)
    if out is None:
        out = torch.empty((b, h, d), dtype=odt, device=q.device)
    if workspace is None:
        workspace = torch.empty((max(nb, 16),), dtype=torch.uint8, device=q.device)
    _check(lib.rq_kv4_decode_attention(_ptr(q), b, h, s, _ptr(kc), _ptr(ks), _ptr(kz), _ptr(vc), _ptr(vs), _ptr(vz),
                                       _ptr(signs), float(softmax_scale), _ptr(out), o, _ptr(workspace), _stream(q)),
           "rq_kv4_decode_attention")
    return out


def selftest_wait_timeout(limit_cycles=1_000_000):
    """Launch the self-test kernel whose bounded wait runs out (see rq.h)."""
    _check(lib.rq_selftest_wait_timeout(int(limit_cycles), _stream()), "rq_selftest_wait_timeout")


def get_device_error(stream=None):
    """Synchronize the stream and raise if a kernel recorded a device-side timeout."""
    s = ctypes.c_void_p(stream) if stream is not None else _stream()
    _check(lib.rq_get_device_error(s), "rq_get_device_error")
