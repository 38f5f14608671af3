"""Comparison helpers for the GPU-vs-oracle parity tests.

Acceptance (from the method's statement of what counts as a match):
* rotated fp32 values within 1e-5 relative (Frobenius over the tensor, and per
  element relative to the row's largest magnitude);
* packed codes and scales identical except at rounding-boundary ties flagged
  by the oracle, which must be at most 1e-4 of the elements and off by one
  code step;
* INT4 int32 accumulators bit-exact on identical codes;
* Y within 1e-3 relative Frobenius error.
"""

import numpy as np
import torch

from oracle import formats, quant

ROT_TOL = 1e-5
Y_TOL = 1e-3
TIE_FRACTION = 1e-4
SCALE_RTOL = 2.0 ** -20


def to_np(t):
    return t.detach().cpu().numpy()


def bf16_to_f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


def check_rotation(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    fro = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300)
    assert fro <= ROT_TOL, fro
    rowmax = np.abs(ref).max(axis=-1, keepdims=True)
    elem = np.abs(gpu - ref) <= ROT_TOL * np.maximum(rowmax, 1e-300)
    assert elem.all(), np.argwhere(~elem)[:5]
    return fro


def check_codes(gpu_codes, ref_codes, tie, rank=None, excused=None, what="codes"):
    """Integer codes: equal except at tie-risk positions, off by <= 1 step.

    rank maps a code to its position on the value axis (identity by default).
    excused marks positions whose scale legitimately differed (not counted).
    Returns the number of mismatches.
    """
    g = np.asarray(gpu_codes)
    r = np.asarray(ref_codes)
    if rank is not None:
        g, r = rank(g), rank(r)
    mism = g != r
    if excused is not None:
        mism &= ~excused
    bad = mism & ~tie
    assert not bad.any(), "%s: %d mismatches outside tie bands, first at %s (gpu %s, ref %s)" % (
        what, bad.sum(), np.argwhere(bad)[:3].tolist(), g[bad][:3], r[bad][:3])
    assert np.all(np.abs(g[mism].astype(np.int64) - r[mism].astype(np.int64)) <= 1), what
    assert mism.sum() <= TIE_FRACTION * mism.size, "%s: %d tie mismatches" % (what, mism.sum())
    return int(mism.sum())


def e2m1_rank(codes):
    """Signed position of an E2M1 code on the value axis (-7..7)."""
    c = np.asarray(codes, dtype=np.int64)
    mag = c & 7
    return np.where(c & 8, -mag, mag)


def check_int4_quant(codes_gpu, scales_gpu, xr):
    """codes_gpu uint8 [M, K/2], scales_gpu fp32 [M] against the oracle on rotated fp64 xr."""
    q, s, tie = quant.int4_sym_rows(xr)
    sg = np.asarray(scales_gpu, dtype=np.float64)
    so = s.astype(np.float64)
    assert np.all(np.abs(sg - so) <= SCALE_RTOL * so + 1e-38), np.max(np.abs(sg - so) / np.maximum(so, 1e-38))
    qg = quant.unpack_nibbles(codes_gpu, signed=True)
    return check_codes(qg, q, tie, what="int4 codes")


def check_int_quant(codes_gpu, scales_gpu, xr, bits):
    """codes_gpu int8 [M, K] (one 6- or 8-bit code per byte), scales_gpu fp32 [M]
    against the oracle on rotated fp64 xr."""
    q, s, tie = quant.int_sym_rows(xr, bits)
    sg = np.asarray(scales_gpu, dtype=np.float64)
    so = s.astype(np.float64)
    assert np.all(np.abs(sg - so) <= SCALE_RTOL * so + 1e-38), np.max(np.abs(sg - so) / np.maximum(so, 1e-38))
    return check_codes(np.asarray(codes_gpu, dtype=np.int64), q, tie, what="int%d codes" % bits)


def check_nvfp4_quant(codes_gpu, sc_gpu, g_gpu, xr, g_ref=None):
    g_o = quant.nvfp4_global_scale(xr) if g_ref is None else np.float32(g_ref)
    if g_ref is None:
        assert abs(float(g_gpu) - float(g_o)) <= SCALE_RTOL * float(g_o), (float(g_gpu), float(g_o))
    e, sc, tie_e, tie_s = quant.nvfp4_rows(xr, g_o)
    scg = np.asarray(sc_gpu, dtype=np.int64)
    n_s = check_codes(scg, sc, tie_s, what="e4m3 scales")
    bad_blk = (scg != sc)
    excused = np.repeat(bad_blk, 16, axis=1)
    eg = quant.unpack_nibbles(codes_gpu, signed=False)
    n_e = check_codes(eg, e, tie_e, rank=e2m1_rank, excused=excused, what="e2m1 codes")
    check_tie_budget(n_s, sc.size, int(excused.sum()) + n_e, e.size, "nvfp4")
    return n_s, n_e


def check_mxfp4_quant(codes_gpu, sc_gpu, xr):
    """MXFP4 parity: E8M0 scales identical except at oracle-flagged
    power-of-two ties (by one exponent step), whose blocks are then excused
    from the code comparison; E2M1 codes identical modulo flagged ties."""
    e, sc, tie_e, tie_s = quant.mxfp4_rows(xr)
    scg = np.asarray(sc_gpu, dtype=np.int64)
    bad = scg != sc
    assert not (bad & ~tie_s).any(), "E8M0 scale mismatch outside tie bands"
    assert np.all(np.abs(scg - sc) <= 1)
    excused = np.repeat(bad, 32, axis=1)
    eg = quant.unpack_nibbles(codes_gpu, signed=False)
    n_e = check_codes(eg, e, tie_e, rank=e2m1_rank, excused=excused, what="e2m1 codes")
    check_tie_budget(int(bad.sum()), bad.size, int(excused.sum()) + n_e, e.size, "mxfp4")
    return int(bad.sum()), n_e


def check_tie_budget(n_scales, total_scales, n_codes, total_codes, what):
    """Rounding-boundary ties may affect at most TIE_FRACTION of the
    elements: of the scale (or scale/zero) elements, and of the code elements,
    where n_codes counts the code mismatches at ties plus every code of a
    block or vector excused by a scale tie."""
    assert n_scales <= TIE_FRACTION * total_scales, "%s: %d of %d scales at ties" % (what, n_scales, total_scales)
    assert n_codes <= TIE_FRACTION * total_codes, "%s: %d of %d codes at or excused by ties" % (
        what, n_codes, total_codes)


def mxfp4_tie_bounds(e, sc, tie_e, tie_s):
    """An E2M1 tie moves a value by at most one grid step (<= 2) times the
    block scale; an E8M0 tie doubles or halves the block scale, moving each
    value by at most its magnitude plus a grid step at the larger scale."""
    xhat = quant.mxfp4_dequant(e, sc)
    sval = np.repeat(formats.e8m0_values(sc), 32, axis=1)
    d = tie_e * 2.0 * sval
    blk = np.repeat(tie_s, 32, axis=1)
    d = d + blk * (np.abs(xhat) + 4.0 * sval)
    return xhat, d


def _fp16_ulp(v):
    h = np.asarray(v, dtype=np.float64).astype(np.float16)
    return np.abs(np.nextafter(h, np.float16(np.inf)).astype(np.float64) - h.astype(np.float64))


def check_kv4(codes_gpu, scale_gpu, zero_gpu, xr):
    """KV4 parity.  fp16 scale / zero decisions may differ only at oracle-flagged
    ties and by one fp16 step; such a vector is excused from the code
    comparison and counted separately (returned), the 1e-4 bound applying to
    the code elements of the other vectors."""
    q, s_h, z_h, tie, tie_sz = quant.kv4_vectors(xr)
    sg = np.asarray(scale_gpu, dtype=np.float64)
    zg = np.asarray(zero_gpu, dtype=np.float64)
    bad_sz = (sg != s_h) | (zg != z_h)
    assert not (bad_sz & ~tie_sz).any(), "fp16 scale/zero mismatch outside tie bands"
    assert np.all(np.abs(sg - s_h) <= _fp16_ulp(s_h) + 1e-30)
    assert np.all(np.abs(zg - z_h) <= np.maximum(_fp16_ulp(z_h), _fp16_ulp(zg)) + 1e-30)
    qg = quant.unpack_nibbles(codes_gpu, signed=False)
    excused = np.repeat(bad_sz[..., None], xr.shape[-1], axis=-1)
    n_codes = check_codes(qg, q, tie, excused=excused, what="kv4 codes")
    n_sz = int((sg != s_h).sum() + (zg != z_h).sum())
    check_tie_budget(n_sz, 2 * bad_sz.size, int(excused.sum()) + n_codes, q.size, "kv4")
    return n_codes, int(bad_sz.sum())


def check_y(y_gpu, y_ref, tol=Y_TOL):
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    err = np.linalg.norm(y_gpu - y_ref) / max(np.linalg.norm(y_ref), 1e-300)
    assert err <= tol, err
    return err


def check_y_with_ties(y_gpu, y_ref, xhat, dx, what_, dw, tol=Y_TOL):
    """Y parity that accounts for legitimate tie decisions upstream.

    xhat / what_ are the oracle's dequantized operands, dx / dw non-negative
    per-element bounds on how far a tie decision (flagged by the oracle) may
    move them.  The part of |Y_gpu - Y_ref| beyond the induced bound
    dx.(|what|+dw)^T + |xhat|.dw^T must be within tol (relative Frobenius).
    Everything here is computed from oracle data only.
    """
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    bound = dx @ (np.abs(what_) + dw).T + np.abs(xhat) @ dw.T
    excess = np.maximum(np.abs(y_gpu - y_ref) - bound, 0.0)
    err = np.linalg.norm(excess) / max(np.linalg.norm(y_ref), 1e-300)
    assert err <= tol, err
    return err, float(np.linalg.norm(y_gpu - y_ref) / max(np.linalg.norm(y_ref), 1e-300))


def int4_tie_bounds(q, s, tie):
    s64 = np.asarray(s, dtype=np.float64)[:, None]
    return q * s64, tie * s64


def nvfp4_tie_bounds(e, sc, g, tie_e, tie_s):
    """An E2M1 tie moves a value by at most one grid step (<= 2) times S*g; an
    E4M3 scale tie moves the block scale by one step (<= 1/8 relative for normal
    scales, one subnormal step below) and may move every code of the block by a
    step as well."""
    xhat = quant.nvfp4_dequant(e, sc, g)
    rows, k = xhat.shape
    sval = formats.e4m3_values(sc)
    sg = np.repeat(sval * np.float64(g), 16, axis=1)
    d = tie_e * 2.0 * sg
    blk = np.repeat(tie_s, 16, axis=1)
    d = d + blk * (np.abs(xhat) * 0.25 + 2.0 * sg + 2.0 ** -9 * 6.0 * np.float64(g))
    return xhat, d


def check_bf16_y(y_gpu_bf16, y_ref, abs_terms, k):
    """bf16 Y: within one bf16 step of the oracle's Y rounded to bf16, plus the
    fp32 accumulation bound gamma_K * sum_k |x_k w_k| (abs_terms) of the GPU's
    own sum (which matters where terms cancel and Y is near zero)."""
    got = np.asarray(y_gpu_bf16, dtype=np.float64)
    rb = bf16_round(y_ref)
    gamma = k * 2.0 ** -24 / (1 - k * 2.0 ** -24)
    tol = np.abs(rb) * 2.0 ** -7 + gamma * abs_terms * 2.0 + 1e-30
    bad = np.abs(got - rb) > tol
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError("%d bf16 elements off, e.g. %s" % (bad.sum(), [
            (tuple(i), float(got[tuple(i)]), float(y_ref[tuple(i)]), float(tol[tuple(i)])) for i in idx]))


def bf16_round(v):
    return torch.from_numpy(np.asarray(v, dtype=np.float64)).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


__all__ = ["formats"]
