"""Oracle: the 4-bit quantizers and the nibble packing, step by step in fp64.

Test infrastructure only (see ``oracle/__init__.py``).

Sources on the pages:

* INT4 symmetric, one scale per token (activations) and one per output channel
  (weights): "Rotations for 4-Bit Activations: QuaRot, SpinQuant, and Friends",
  section "What it buys in 4 bits, and what it doesn't"; round to nearest per
  section "Gotchas" ("These checkpoints use round to nearest").
* NVFP4 -- E2M1 values with an FP8 (E4M3) scale for every block of 16 values:
  same section.  The fp32 per-tensor scale is the second level of NVFP4's
  two-level scaling.
* MXFP4 -- E2M1 values whose scales are powers of two shared by 32 values:
  same article, section "The full model in NVFP4, on vLLM" (the FP4 study it
  cites) and section "When to rotate".
* 6- and 8-bit symmetric round to nearest (W8A8, W6A6) and W4A8:
  "QuaRot (rotation-based outlier removal, W4A4KV4)", field "Bits" (lossless
  6-bit and 8-bit round-to-nearest, no calibration data) and "SpinQuant
  (learned rotations + W4A4KV4)", field "Activation scheme" (also reported
  at W4A8).
* Per-group asymmetric INT4 for activations and weights: "SpinQuant (learned
  rotations + W4A4KV4)", field "Activation scheme" (per-group INT4
  asymmetric quantization of weights, activations and KV cache).
* KV cache at 4 bits, asymmetric: "SpinQuant (learned rotations + W4A4KV4)",
  field "Activation scheme" (per-group INT4 asymmetric for the KV cache), and
  "QuaRot (rotation-based outlier removal, W4A4KV4)", field "Activation scheme"
  (rotations applied to the KV cache too).

Readings where the pages are silent (each also listed in the design notes):

* INT4: s = fp32(fp32(amax)/7); q = clamp(rint(x/s), -8, 7) with rint
  half-to-even; so -8 is never produced.  amax = 0 -> s = 0, q = 0.
* INT6 / INT8: the INT4 rule with qmax = 2^(b-1) - 1 = 31 / 127 in place
  of 7: s = fp32(fp32(amax)/qmax), q = clamp(rint(x/s), -qmax-1, qmax), one
  scale per token (activations) or output channel (weights); the codes are
  stored one per byte (two's complement).
* NVFP4: g = fp32(fp32(amax(X~)) / (6*448)) over the whole rotated tensor
  (dynamic) or given by the caller (static).  Per block b of 16 along K:
  S_b = E4M3_rn_satfinite(amax_b / (6 g)); e = E2M1_rn_satfinite(x / (S_b g));
  S_b = 0 -> e = 0.
* MXFP4: per block b of 32 along K, the E8M0 scale 2^e with
  e = floor(log2(amax_b)) - 2 (2 = the exponent of E2M1's largest value 6),
  clamped to E8M0's range [-127, 127]; e = E2M1_rn_satfinite(x / 2^e).  The
  pages give no scale rule; this is the shared-exponent rule of the OCP
  Microscaling formats.  amax_b = 0 -> scale code 0 (2^-127), e = 0.  There
  is no per-tensor scale.
* Per-group asymmetric INT4 of X / W: the KV4 rule below on every group of
  128 consecutive channels of a row (the pages give no group width; 128 is
  the rotation block).
* KV4 per (batch, head, token) vector of head_dim after the Hadamard:
  z = min, s = (max - min)/15, z_h = fp16(z), s_h = fp16(s);
  q = clamp(rint((x - z_h)/s_h), 0, 15); s_h = 0 -> q = 0.
* Packing: element 2i in the low nibble of byte i, 2i+1 in the high nibble.
  INT4 nibbles are two's complement, KV nibbles unsigned, E2M1 nibbles carry
  the sign in bit 3.

Tie accounting: each quantizer also returns a boolean mask of "tie-risk"
decisions -- inputs whose scaled value lies within ``TIE_EPS * max(1, |v|)`` of
a rounding midpoint.  A GPU computing the same steps in fp32 may round those
the other way; everywhere else it must agree exactly.
"""

import numpy as np

from . import formats

# Relative width of the rounding-boundary band.  The fp32 butterflies of a
# log2(n)-stage transform carry a relative error of order log2(n) * 2^-24 of the
# block's partial sums; scaled into code units this stays below ~1e-5, so a
# band of 2^-15 (3.05e-5) covers it with margin.
TIE_EPS = 2.0 ** -15

INT4_QMAX = 7
NVFP4_BLOCK = 16
MXFP4_BLOCK = 32
E2M1_EMAX = 2          # 6 = 1.5 * 2^2
E8M0_EMIN, E8M0_EMAX = -127, 127
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def _near_half(v, eps=TIE_EPS):
    """True where v is within eps*max(1,|v|) of k + 1/2 for an integer k."""
    frac_dist = np.abs(v - (np.floor(v) + 0.5))
    return frac_dist <= eps * np.maximum(1.0, np.abs(v))


def int4_sym_rows(xr):
    """Per-row (per-token / per-output-channel) symmetric INT4.

    xr: fp64 [rows, K].  Returns (q int64 [rows, K] in [-8, 7],
    scale fp32 [rows], tie bool [rows, K]).
    """
    xr = np.asarray(xr, dtype=np.float64)
    amax = np.abs(xr).max(axis=1).astype(np.float32)
    scale = amax / np.float32(INT4_QMAX)                    # fp32 / fp32, correctly rounded
    s64 = scale.astype(np.float64)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s64 > 0, xr / np.where(s64 > 0, s64, 1.0), 0.0)
    q = np.clip(np.rint(v), -8, INT4_QMAX).astype(np.int64)
    tie = _near_half(v) & (s64 > 0)
    return q, scale, tie


def int_sym_rows(xr, bits):
    """Per-row symmetric round-to-nearest with b-bit signed codes, b in 4..8.

    qmax = 2^(b-1) - 1.  xr: fp64 [rows, K].  Returns (q int64 [rows, K] in
    [-qmax-1, qmax], scale fp32 [rows], tie bool [rows, K]).
    """
    if not 4 <= bits <= 8:
        raise ValueError("bits must be in 4..8")
    qmax = 2 ** (bits - 1) - 1
    xr = np.asarray(xr, dtype=np.float64)
    amax = np.abs(xr).max(axis=1).astype(np.float32)
    scale = amax / np.float32(qmax)                          # fp32 / fp32, correctly rounded
    s64 = scale.astype(np.float64)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s64 > 0, xr / np.where(s64 > 0, s64, 1.0), 0.0)
    q = np.clip(np.rint(v), -qmax - 1, qmax).astype(np.int64)
    tie = _near_half(v) & (s64 > 0)
    return q, scale, tie


def int4_dequant(q, scale):
    return np.asarray(q, dtype=np.float64) * np.asarray(scale, dtype=np.float64)[:, None]


def nvfp4_global_scale(xr):
    """Dynamic per-tensor scale g = fp32(fp32(amax) / (6 * 448)) of the rotated tensor."""
    amax = np.float32(np.abs(np.asarray(xr, dtype=np.float64)).max())
    return np.float32(amax / np.float32(E2M1_MAX * E4M3_MAX))


def nvfp4_rows(xr, g):
    """NVFP4 quantization of fp64 [rows, K] with per-tensor scale g (fp32).

    Returns (e codes int64 [rows, K] (sign in bit 3), S codes int64
    [rows, K/16] (E4M3 bits), tie_e bool [rows, K], tie_s bool [rows, K/16]).
    """
    xr = np.asarray(xr, dtype=np.float64)
    rows, k = xr.shape
    if k % NVFP4_BLOCK:
        raise ValueError("K must be a multiple of 16")
    g = np.float64(np.float32(g))
    blocks = xr.reshape(rows, k // NVFP4_BLOCK, NVFP4_BLOCK)
    amax_b = np.abs(blocks).max(axis=2)
    if g > 0:
        w = amax_b / (E2M1_MAX * g)
    else:
        w = np.zeros_like(amax_b)
    s_codes, s_tie_dist = formats.e4m3_round_unsigned(w)
    tie_s = (s_tie_dist <= TIE_EPS * np.maximum(1.0, w)) & (w > 0)
    s_val = formats.e4m3_values(s_codes)                     # exact decoded scale
    denom = (s_val * g)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(denom > 0, blocks / np.where(denom > 0, denom, 1.0), 0.0)
    e_codes, e_tie_dist = formats.e2m1_round(v)
    tie_e = (e_tie_dist <= TIE_EPS * np.maximum(1.0, np.abs(v))) & (denom > 0)
    return (e_codes.reshape(rows, k), s_codes, tie_e.reshape(rows, k), tie_s)


def nvfp4_dequant(e_codes, s_codes, g):
    e = formats.e2m1_values(e_codes)
    rows, k = e.shape
    s = formats.e4m3_values(s_codes)
    return (e.reshape(rows, k // NVFP4_BLOCK, NVFP4_BLOCK) * s[:, :, None]
            * np.float64(np.float32(g))).reshape(rows, k)


def mxfp4_rows(xr):
    """MXFP4 quantization of fp64 [rows, K].

    Returns (e codes int64 [rows, K] (sign in bit 3), scale codes int64
    [rows, K/32] (E8M0 bits), tie_e bool [rows, K], tie_s bool [rows, K/32]).
    tie_s flags blocks whose amax lies within the tie band of a power of two,
    where floor(log2(amax)) flips between neighbours under fp32 rounding.
    """
    xr = np.asarray(xr, dtype=np.float64)
    rows, k = xr.shape
    if k % MXFP4_BLOCK:
        raise ValueError("K must be a multiple of 32")
    blocks = xr.reshape(rows, k // MXFP4_BLOCK, MXFP4_BLOCK)
    amax_b = np.abs(blocks).max(axis=2)
    pos = amax_b > 0
    with np.errstate(divide="ignore"):
        # frexp gives amax = f * 2^p with f in [0.5, 1): floor(log2(amax)) = p - 1 exactly
        _, p2 = np.frexp(np.where(pos, amax_b, 1.0))
    e = np.where(pos, p2.astype(np.int64) - 1 - E2M1_EMAX, E8M0_EMIN)
    e = np.clip(e, E8M0_EMIN, E8M0_EMAX)
    s_codes = (e + 127).astype(np.int64)
    # within the band of a power of two: fp32 rounding of amax may change floor(log2)
    pw = np.ldexp(1.0, np.where(pos, p2.astype(np.int64) - 1, 0))
    near = (np.abs(amax_b - pw) <= TIE_EPS * amax_b) | (np.abs(amax_b - 2 * pw) <= TIE_EPS * amax_b)
    tie_s = near & pos
    v = blocks / np.ldexp(1.0, e)[:, :, None]                 # exact: a power-of-two division
    e_codes, e_tie_dist = formats.e2m1_round(v)
    tie_e = (e_tie_dist <= TIE_EPS * np.maximum(1.0, np.abs(v))) & pos[:, :, None]
    return (e_codes.reshape(rows, k), s_codes, tie_e.reshape(rows, k), tie_s)


def mxfp4_dequant(e_codes, s_codes):
    e = formats.e2m1_values(e_codes)
    rows, k = e.shape
    s = formats.e8m0_values(s_codes)
    return (e.reshape(rows, k // MXFP4_BLOCK, MXFP4_BLOCK) * s[:, :, None]).reshape(rows, k)


def _fp16_tie(v):
    """True where fp64 v lies within a relative TIE_EPS of an fp16 rounding midpoint."""
    v = np.asarray(v, dtype=np.float64)
    h = v.astype(np.float16)
    up = np.nextafter(h, np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(h, np.float16(-np.inf)).astype(np.float64)
    hv = h.astype(np.float64)
    d = np.minimum(np.abs(v - 0.5 * (hv + up)), np.abs(v - 0.5 * (hv + dn)))
    return d <= TIE_EPS * np.maximum(np.abs(v), 2.0 ** -24)


def kv4_vectors(xr):
    """Asymmetric 4-bit quantization of each last-axis vector of rotated fp64 xr.

    Returns (q int64 [..., D] in [0, 15], scale fp16-valued fp64 [...],
    zero fp16-valued fp64 [...], tie bool [..., D], tie_sz bool [...]).
    """
    xr = np.asarray(xr, dtype=np.float64)
    lo = xr.min(axis=-1)
    hi = xr.max(axis=-1)
    s = (hi - lo) / 15.0
    z_h = formats.to_fp16(lo)
    s_h = formats.to_fp16(s)
    sh = s_h[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(sh > 0, (xr - z_h[..., None]) / np.where(sh > 0, sh, 1.0), 0.0)
    q = np.clip(np.rint(v), 0, 15).astype(np.int64)
    tie = _near_half(v) & (sh > 0)
    tie_sz = _fp16_tie(lo) | (_fp16_tie(s) & (s > 0))
    return q, s_h, z_h, tie, tie_sz


def asym_int4_groups(xr, group=128):
    """Per-group asymmetric INT4 along the last axis of rotated fp64 xr [rows, K]:
    each group of `group` channels is quantized by the KV4 rule (z = min,
    s = (max - min)/15 as fp16, q = clamp(rint((x - z_h)/s_h), 0, 15)).

    Returns (q int64 [rows, K], s_h [rows, K/group], z_h [rows, K/group],
    tie bool [rows, K], tie_sz bool [rows, K/group]).
    """
    xr = np.asarray(xr, dtype=np.float64)
    rows, k = xr.shape
    if k % group:
        raise ValueError("K must be a multiple of the group")
    q, s_h, z_h, tie, tie_sz = kv4_vectors(xr.reshape(rows, k // group, group))
    return q.reshape(rows, k), s_h, z_h, tie.reshape(rows, k), tie_sz


def asym_int4_dequant(q, s_h, z_h, group=128):
    rows, k = np.shape(q)
    qg = np.asarray(q, dtype=np.float64).reshape(rows, k // group, group)
    return (qg * np.asarray(s_h)[..., None] + np.asarray(z_h)[..., None]).reshape(rows, k)


def kv4_dequant(q, s_h, z_h):
    return np.asarray(q, dtype=np.float64) * s_h[..., None] + z_h[..., None]


def pack_nibbles(codes):
    """Pack int codes [..., K] (K even) into uint8 [..., K/2], element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed, signed):
    """Inverse of pack_nibbles; signed=True reads two's-complement INT4."""
    p = np.asarray(packed, dtype=np.int64)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    out = np.stack([lo, hi], axis=-1).reshape(*p.shape[:-1], p.shape[-1] * 2)
    if signed:
        out = np.where(out >= 8, out - 16, out)
    return out
