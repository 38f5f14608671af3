"""Oracle: one decoding step of attention over the 4-bit KV cache, in fp64.

Test infrastructure only (see ``oracle/__init__.py``).

Sources on the pages:

* "QuaRot (rotation-based outlier removal, W4A4KV4)", field "Activation
  scheme": the rotation is applied to the KV cache too, so keys and values are
  stored rotated (and quantized to 4 bits: the KV4 of W4A4KV4).
* "SpinQuant (learned rotations + W4A4KV4)", field "Activation scheme":
  per-group asymmetric INT4 for the KV cache (a scale and a zero point).
* "Rotations for 4-Bit Activations: QuaRot, SpinQuant, and Friends", section
  "A rotation changes nothing, and that is the point": for orthogonal Q,
  q.K^T = (q.Q).(K.Q)^T, so the query is rotated with the same per-head Q
  (diag(s) . H_128 / sqrt(128)) and scores need no de-rotation; the weighted
  sum of rotated values is rotated back, (p.(V.Q)).Q^T = p.V.

Readings where the pages are silent: a decode step is one query per
(batch, head) attending to all S cached tokens (no mask); softmax with scale
1/sqrt(128) unless given; the cache entries dequantize as z_h + s_h * q with
the stored fp16 scale s_h and zero z_h; the output is returned in the
original (unrotated) basis.
"""

import numpy as np

from . import hadamard

HEAD_DIM = 128


def kv4_dequant(codes, s_h, z_h):
    """z + s * q per cached vector: codes [..., 128] (0..15), s_h / z_h [...]."""
    codes = np.asarray(codes, dtype=np.float64)
    return (np.asarray(z_h, dtype=np.float64)[..., None]
            + np.asarray(s_h, dtype=np.float64)[..., None] * codes)


def rotate_heads(x, signs):
    """x [..., 128] -> x . diag(s) . H_128 / sqrt(128) per head vector."""
    x = np.asarray(x, dtype=np.float64)
    shp = x.shape
    return hadamard.rotate(x.reshape(-1, HEAD_DIM), signs, HEAD_DIM).reshape(shp)


def unrotate_heads(y, signs):
    """The inverse of rotate_heads: y . H_128 / sqrt(128) . diag(s) (H symmetric, Q orthogonal)."""
    y = np.asarray(y, dtype=np.float64)
    h = hadamard.sylvester(HEAD_DIM) / np.sqrt(HEAD_DIM)
    return (y.reshape(-1, HEAD_DIM) @ h * np.asarray(signs, dtype=np.float64)[None, :]).reshape(y.shape)


def attention(q, k, v, scale):
    """softmax(q . k^T * scale) . v for one query per (batch, head).

    q [B, H, D], k / v [B, H, S, D] -> [B, H, D]; also the probabilities [B, H, S].
    """
    q = np.asarray(q, dtype=np.float64)
    s = np.einsum("bhd,bhsd->bhs", q, np.asarray(k, dtype=np.float64)) * scale
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    return np.einsum("bhs,bhsd->bhd", p, np.asarray(v, dtype=np.float64)), p


def kv4_decode_attention(q, kc, ks, kz, vc, vs, vz, signs, scale=None):
    """Decode attention over the KV4 cache.

    q [B, H, 128] (real query, unrotated); kc / vc [B, H, S, 128] codes 0..15;
    ks, kz, vs, vz [B, H, S] fp16 scale / zero values.  Returns o [B, H, 128]
    in the original basis.
    """
    if scale is None:
        scale = 1.0 / np.sqrt(HEAD_DIM)
    q_rot = rotate_heads(q, signs)
    o_rot, _ = attention(q_rot, kv4_dequant(kc, ks, kz), kv4_dequant(vc, vs, vz), scale)
    return unrotate_heads(o_rot, signs)
