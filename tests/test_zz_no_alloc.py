"""The no-allocation NVFP4 entry point, checked against the regular one.

rq_rotate_quantize_nvfp4_noalloc serves callers that cannot allocate device
memory (fixed arenas, plugin APIs without workspaces, hosts that avoid
cudaMalloc after start-up): its scratch lives in a static device array inside
librq.  This file runs last so that a failure here leaves every other test's
result standing.  It calls the C ABI directly and compares the outputs with
rq_rotate_quantize's (same kernels, so the match must be exact) on two calls
in a row, the second with a smaller per-tensor maximum so that a scratch word
left over from the first call would show; a third call, again with a smaller
maximum, has more rows than the SMs' shared memory holds, so the scratch goes
through the two-pass path (a max pass that gathers into it, then a quantize
pass that reads it).
"""

import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(rq, x, s):
    m, k = x.shape
    codes = torch.empty((m, k // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((m, k // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty((1,), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = rq.lib.rq_rotate_quantize_nvfp4_noalloc(_ptr(x), m, k, x.stride(0), _ptr(s), _ptr(codes), _ptr(scales),
                                                 _ptr(g), stream)
    assert st == 0, rq.lib.rq_status_string(st)
    return codes, scales, g


def test_noalloc_matches_regular_entry_point_in_a_row():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rotation_w4a4_quantization_b200 import rq
    from rotation_w4a4_quantization_b200 import synthetic as syn
    rq.init(0)
    k = 4096
    s = syn.signs(k, 91).cuda()
    gen = torch.Generator().manual_seed(92)
    x1 = (torch.randn((333, k), generator=gen) * 3.0).to(torch.bfloat16).cuda()
    x2 = (torch.randn((2048, k), generator=gen) * 0.5).to(torch.bfloat16).cuda()   # smaller max than x1
    x3 = (torch.randn((4100, k), generator=gen) * 0.25).to(torch.bfloat16).cuda()  # two-pass, smaller again
    for x in (x1, x2, x3):
        got = _call_noalloc(rq, x, s)
        ref = rq.rotate_quantize(x, s, 128, "nvfp4", "dynamic")
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    rq.get_device_error()


def test_noalloc_rejects_what_the_regular_entry_point_rejects():
    from rotation_w4a4_quantization_b200 import rq
    a16 = ctypes.c_void_p(0x10000)
    assert rq.lib.rq_rotate_quantize_nvfp4_noalloc(None, 4, 512, 512, a16, a16, a16, a16, None) == 1
    assert rq.lib.rq_rotate_quantize_nvfp4_noalloc(a16, 4, 500, 500, a16, a16, a16, a16, None) == 2
    assert rq.lib.rq_rotate_quantize_nvfp4_noalloc(a16, 0, 512, 512, a16, a16, a16, a16, None) == 0
