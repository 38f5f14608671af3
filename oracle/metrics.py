"""Oracle: the three measures the article uses, in fp64.

Test infrastructure only (see ``oracle/__init__.py``).

"Rotations for 4-Bit Activations: QuaRot, SpinQuant, and Friends":

* section "A rotation changes nothing, and that is the point": the ratio of the
  largest value to the median channel's maximum, and the kurtosis (3 for a
  Gaussian; hundreds to thousands when a few channels dominate);
* section "What it buys in 4 bits, and what it doesn't": the relative error of
  the quantized product ||X.W^T - Q(X).Q(W)^T|| / ||X.W^T||.

Readings: kurtosis is Pearson's (non-excess) E[(x - mu)^4] / sigma^4 over all
entries; the ratio takes a_c = max over tokens of |x[:, c]| per channel c and
returns max_c a_c / median_c a_c; the norm is Frobenius.

Parity unpinned for the article's exact percentages and ratios: those were
measured on real Qwen3-8B layer inputs that are not available here, so the
synthetic stand-ins can only reproduce their direction (checked as
inequalities by the tests).
"""

import numpy as np


def amax_median_ratio(x):
    a = np.abs(np.asarray(x, dtype=np.float64)).max(axis=0)
    return float(a.max() / np.median(a))


def kurtosis(x):
    x = np.asarray(x, dtype=np.float64).reshape(-1)
    mu = x.mean()
    d = x - mu
    var = np.mean(d * d)
    return float(np.mean(d ** 4) / (var * var))


def rel_product_error(y_ref, y_q):
    y_ref = np.asarray(y_ref, dtype=np.float64)
    y_q = np.asarray(y_q, dtype=np.float64)
    return float(np.linalg.norm(y_ref - y_q) / np.linalg.norm(y_ref))
