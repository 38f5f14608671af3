"""Pins for the decode-attention oracle over the 4-bit KV cache (CPU only).

Rotation invariance against plain attention (the closed form the QuaRot page
relies on), softmax against explicit loops, the dequantization identity, the
inverse rotation, and the claim that rotating before the 4-bit KV
quantization lowers the attention error on vectors with outlier dimensions.
"""

import math

import numpy as np

from oracle import attention, hadamard, quant


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_attention_matches_explicit_loops():
    q = _rand((1, 1, 4), 1)
    k = _rand((1, 1, 5, 4), 2)
    v = _rand((1, 1, 5, 4), 3)
    o, p = attention.attention(q, k, v, 0.7)
    sc = [0.7 * sum(q[0, 0, d] * k[0, 0, t, d] for d in range(4)) for t in range(5)]
    m = max(sc)
    e = [math.exp(x - m) for x in sc]
    tot = sum(e)
    for t in range(5):
        assert abs(p[0, 0, t] - e[t] / tot) < 1e-15
    for d in range(4):
        assert abs(o[0, 0, d] - sum(e[t] / tot * v[0, 0, t, d] for t in range(5))) < 1e-14


def test_unrotate_inverts_rotate():
    s = np.where(np.random.default_rng(4).integers(0, 2, 128) == 0, -1.0, 1.0)
    x = _rand((3, 5, 128), 5)
    assert np.abs(attention.unrotate_heads(attention.rotate_heads(x, s), s) - x).max() < 1e-13


def test_rotated_attention_equals_plain_attention():
    # with the cache stored rotated and unquantized, rotating q and rotating
    # the output back gives exactly the plain attention output
    s = np.where(np.random.default_rng(6).integers(0, 2, 128) == 0, -1.0, 1.0)
    q, k, v = _rand((2, 3, 128), 7), _rand((2, 3, 9, 128), 8), _rand((2, 3, 9, 128), 9)
    ref, _ = attention.attention(q, k, v, 1 / np.sqrt(128))
    o_rot, _ = attention.attention(attention.rotate_heads(q, s), attention.rotate_heads(k, s),
                                   attention.rotate_heads(v, s), 1 / np.sqrt(128))
    assert np.abs(attention.unrotate_heads(o_rot, s) - ref).max() < 1e-12


def test_dequant_identity():
    c = np.arange(16)[None, :].repeat(2, 0)
    x = attention.kv4_dequant(np.pad(c, ((0, 0), (0, 112))), np.array([0.5, 2.0]), np.array([-1.0, 3.0]))
    assert np.array_equal(x[0, :16], -1.0 + 0.5 * np.arange(16))
    assert np.array_equal(x[1, :16], 3.0 + 2.0 * np.arange(16))


def _kv4(x, s):
    """Quantize [B, H, S, 128] vectors with kv4_vectors (after rotating them when s is given)."""
    shp = x.shape
    xr = attention.rotate_heads(x, s) if s is not None else x
    q, sh, zh, _, _ = quant.kv4_vectors(xr.reshape(-1, 128))
    return q.reshape(shp), sh.reshape(shp[:-1]), zh.reshape(shp[:-1])


def test_rotation_lowers_kv4_attention_error():
    # KV vectors with two outlier dimensions per head (x30, the kv4 workload's
    # recipe): 4-bit asymmetric quantization with a rotation first loses less
    rng = np.random.default_rng(10)
    b, h, t = 1, 4, 256
    k = rng.standard_normal((b, h, t, 128))
    v = rng.standard_normal((b, h, t, 128))
    for hh in range(h):
        dims = rng.choice(128, 2, replace=False)
        k[:, hh, :, dims] *= 30
        v[:, hh, :, dims] *= 30
    q = rng.standard_normal((b, h, 128))
    s = np.where(rng.integers(0, 2, 128) == 0, -1.0, 1.0)
    ref, _ = attention.attention(q, k, v, 1 / np.sqrt(128))
    kc, ksh, kzh = _kv4(k, s)
    vc, vsh, vzh = _kv4(v, s)
    o_rot = attention.kv4_decode_attention(q, kc, ksh, kzh, vc, vsh, vzh, s)
    kc0, ksh0, kzh0 = _kv4(k, None)
    vc0, vsh0, vzh0 = _kv4(v, None)
    o_plain, _ = attention.attention(q, attention.kv4_dequant(kc0, ksh0, kzh0),
                                     attention.kv4_dequant(vc0, vsh0, vzh0), 1 / np.sqrt(128))
    e_rot = np.linalg.norm(o_rot - ref) / np.linalg.norm(ref)
    e_plain = np.linalg.norm(o_plain - ref) / np.linalg.norm(ref)
    # (0.32 vs 1.37 here: the outlier dimensions make the softmax sharp, so the
    # output error is far above the cache's own ~7% / ~24% error)
    assert e_rot < 0.5 * e_plain
