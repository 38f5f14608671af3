"""Oracle: the W4A4 matrix product, from the dequantized definition.

Test infrastructure only (see ``oracle/__init__.py``).

"Rotations for 4-Bit Activations: QuaRot, SpinQuant, and Friends", section
"A rotation changes nothing, and that is the point": Y = X.W^T =
(X.Q).(W.Q)^T, so the layer is computed as Q(X.Q) . Q(W.Q)^T from the
quantized operands.

* INT4: acc[m, n] = sum_k qx[m, k] qw[n, k] exactly (integers), then
  Y = acc * s_x[m] * s_w[n].  The same with 6- or 8-bit codes on either side
  (W4A8, W6A6, W8A8: "QuaRot (rotation-based outlier removal, W4A4KV4)",
  field "Bits"; "SpinQuant (learned rotations + W4A4KV4)", field
  "Activation scheme").
* NVFP4: Y = sum_k xhat[m, k] what[n, k] with xhat = e * S_b * g (exact fp64
  dequantized values).

The integer sum is formed by a float64 matrix product of integer-valued
arrays, which is exact here because every product is at most 64 (INT4) or
128 * 128 (8-bit codes) in magnitude and every partial sum stays far below
2^53.
"""

import numpy as np

from . import quant


def int4_acc(qx, qw):
    """Exact integer accumulators acc[m, n] = sum_k qx[m,k]*qw[n,k] (int64)."""
    qx = np.asarray(qx, dtype=np.int64)
    qw = np.asarray(qw, dtype=np.int64)
    k = qx.shape[1]
    if k * 64 >= 2 ** 53:
        raise ValueError("K too large for an exact float64 sum")
    acc = qx.astype(np.float64) @ qw.astype(np.float64).T
    return np.rint(acc).astype(np.int64)


def int_acc(qx, qw):
    """Exact integer accumulators for signed codes of any width up to 8 bits
    (W4A4, W4A8, W6A6, W8A8): acc[m, n] = sum_k qx[m,k]*qw[n,k] (int64)."""
    qx = np.asarray(qx, dtype=np.int64)
    qw = np.asarray(qw, dtype=np.int64)
    k = qx.shape[1]
    if k * 128 * 128 >= 2 ** 53:
        raise ValueError("K too large for an exact float64 sum")
    acc = qx.astype(np.float64) @ qw.astype(np.float64).T
    return np.rint(acc).astype(np.int64)


def int4_y(acc, sx, sw):
    """Y = acc * s_x[m] * s_w[n] in fp64 (scales are fp32 values)."""
    return (np.asarray(acc, dtype=np.float64)
            * np.asarray(sx, dtype=np.float32).astype(np.float64)[:, None]
            * np.asarray(sw, dtype=np.float32).astype(np.float64)[None, :])


def nvfp4_y(ex, sx, gx, ew, sw, gw):
    """Y = deq(X) . deq(W)^T in fp64 from NVFP4 codes and scales."""
    xh = quant.nvfp4_dequant(ex, sx, gx)
    wh = quant.nvfp4_dequant(ew, sw, gw)
    return xh @ wh.T


def mxfp4_y(ex, sx, ew, sw):
    """Y = deq(X) . deq(W)^T in fp64 from MXFP4 codes and E8M0 scales."""
    xh = quant.mxfp4_dequant(ex, sx)
    wh = quant.mxfp4_dequant(ew, sw)
    return xh @ wh.T
