"""GPU parity of the KV4 decode attention (the consumer of the 4-bit KV cache)
against the fp64 oracle; all calls go through the C ABI.

"QuaRot (rotation-based outlier removal, W4A4KV4)", "Activation scheme" (the
cache is stored rotated); "Rotations for 4-Bit Activations: QuaRot, SpinQuant,
and Friends", "A rotation changes nothing, and that is the point".
"""

import numpy as np
import pytest
import torch

import parity
from oracle import attention, quant
from rotation_w4a4_quantization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from rotation_w4a4_quantization_b200 import rq as m
    m.init(0)
    return m


def _cache_from_oracle(x, s):
    """Oracle KV4 cache of x [B, H, S, 128] (rotated with signs s)."""
    b, h, t, d = x.shape
    xr = attention.rotate_heads(x, s)
    q, sh, zh, _, _ = quant.kv4_vectors(xr.reshape(-1, d))
    return q.reshape(b, h, t, d), sh.reshape(b, h, t), zh.reshape(b, h, t)


def _dev_cache(q, sh, zh):
    b, h, t, d = q.shape
    codes = quant.pack_nibbles(q.reshape(-1, d)).reshape(b, h, t, d // 2)
    return (torch.from_numpy(codes).cuda(), torch.from_numpy(sh.astype(np.float16)).cuda(),
            torch.from_numpy(zh.astype(np.float16)).cuda())


def _inputs(b, h, t, seed, outliers=True):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn((b, h, t, 128), generator=g)
    v = torch.randn((b, h, t, 128), generator=g)
    if outliers:
        k[..., 5] *= 30
        v[..., 77] *= 20
    qv = torch.randn((b, h, 128), generator=g).to(torch.bfloat16)
    return (parity.bf16_to_f64(k.to(torch.bfloat16)), parity.bf16_to_f64(v.to(torch.bfloat16)), qv)


@pytest.mark.parametrize("b,h,t", [(1, 2, 300), (2, 4, 4096), (1, 1, 1), (1, 3, 256), (4, 8, 1000), (1, 2, 257)])
def test_decode_attention_on_oracle_cache(rq, b, h, t):
    k, v, qv = _inputs(b, h, t, 10 + t)
    s = syn.signs(128, 900 + t)
    kq, ksh, kzh = _cache_from_oracle(k, s.numpy())
    vq, vsh, vzh = _cache_from_oracle(v, s.numpy())
    out = rq.kv4_decode_attention(qv.cuda(), _dev_cache(kq, ksh, kzh), _dev_cache(vq, vsh, vzh), s.cuda())
    torch.cuda.synchronize()
    ref = attention.kv4_decode_attention(parity.bf16_to_f64(qv), kq, ksh, kzh, vq, vsh, vzh, s.numpy())
    got = parity.to_np(out).astype(np.float64)
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err < 1e-5, err
    assert np.all(np.abs(got - ref) <= 1e-4 * np.abs(ref).max(axis=-1, keepdims=True))


def test_decode_attention_bf16_out_and_scale(rq):
    b, h, t = 2, 2, 700
    k, v, qv = _inputs(b, h, t, 3)
    s = syn.signs(128, 4)
    kq, ksh, kzh = _cache_from_oracle(k, s.numpy())
    vq, vsh, vzh = _cache_from_oracle(v, s.numpy())
    out = rq.kv4_decode_attention(qv.cuda(), _dev_cache(kq, ksh, kzh), _dev_cache(vq, vsh, vzh), s.cuda(),
                                  softmax_scale=0.05, out_dtype="bf16")
    ref = attention.kv4_decode_attention(parity.bf16_to_f64(qv), kq, ksh, kzh, vq, vsh, vzh, s.numpy(), scale=0.05)
    got = out.float().cpu().numpy().astype(np.float64)
    rb = parity.bf16_round(ref)
    assert np.all(np.abs(got - rb) <= np.abs(rb) * 2.0 ** -7 + 1e-4 * np.abs(ref).max())


def test_decode_attention_end_to_end(rq):
    # the GPU writes the cache (rq_kv_rotate_quantize), the GPU reads it; the
    # oracle attends over the GPU's own cache, and the result stays close to
    # attention over the unquantized bf16 K, V
    b, h, t = 2, 4, 1024
    kv = syn.kv(batch=b, heads=h, seq=t, which=0)
    vv = syn.kv(batch=b, heads=h, seq=t, which=1)
    s = syn.workload_signs("kv4")
    kc = rq.kv_rotate_quantize(kv.cuda(), s.cuda())
    vc = rq.kv_rotate_quantize(vv.cuda(), s.cuda())
    g = torch.Generator().manual_seed(5)
    qv = torch.randn((b, h, 128), generator=g).to(torch.bfloat16)
    out = rq.kv4_decode_attention(qv.cuda(), kc, vc, s.cuda())
    torch.cuda.synchronize()

    def host(c):
        codes = quant.unpack_nibbles(c[0].cpu().numpy().reshape(-1, 64), signed=False).reshape(b, h, t, 128)
        return codes, c[1].cpu().numpy().astype(np.float64), c[2].cpu().numpy().astype(np.float64)

    ref = attention.kv4_decode_attention(parity.bf16_to_f64(qv), *host(kc), *host(vc), s.numpy())
    got = parity.to_np(out).astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-5
    exact, _ = attention.attention(parity.bf16_to_f64(qv), parity.bf16_to_f64(kv), parity.bf16_to_f64(vv),
                                   1 / np.sqrt(128))
    assert np.linalg.norm(got - exact) / np.linalg.norm(exact) < 0.5
    rq.get_device_error()


def test_decode_attention_rejects_bad_arguments(rq):
    b, h, t = 1, 1, 4
    k, v, qv = _inputs(b, h, t, 1)
    s = syn.signs(128, 1)
    kq, ksh, kzh = _cache_from_oracle(k, s.numpy())
    kc = _dev_cache(kq, ksh, kzh)
    empty = (kc[0][:, :, :0], kc[1][:, :, :0], kc[2][:, :, :0])
    with pytest.raises(rq.RQError) as e:
        rq.kv4_decode_attention(qv.cuda(), empty, empty, s.cuda())
    assert e.value.status == 1
    with pytest.raises(rq.RQError) as e:
        rq.kv4_decode_attention(qv.cuda(), kc, kc, s.cuda(), softmax_scale=-1.0)
    assert e.value.status == 1
