"""Oracle: the randomized (block) Hadamard rotation, as a dense fp64 product.

Test infrastructure only (see ``oracle/__init__.py``).

Follows "Rotations for 4-Bit Activations: QuaRot, SpinQuant, and Friends",
section "A rotation changes nothing, and that is the point": Q is a Hadamard
matrix scaled by 1/sqrt(n), so every entry is +-1/sqrt(n); and section
"Gotchas" / "The recipe": the rotation is applied in 128-wide blocks
(block-diagonal Q) or at full width.  The random +-1 sign diagonal is the
"randomized Hadamard" of the QuaRot page ("Activation scheme") and of the
SpinQuant page's notes ("QuaRot uses a randomized Hadamard").

Reading taken where the pages are silent: Q = diag(s) . H_B / sqrt(B) per block
(flip the signs of the input channels, then transform), H_B the Sylvester
(natural-order) Hadamard, one independent sign per channel.  The same Q is
applied to X and to W, so (X.Q)(W.Q)^T = X.W^T.
"""

import functools

import numpy as np


def sylvester(n):
    """Dense Sylvester Hadamard H_n (n a power of two), fp64, entries +-1.

    Closed form H[i, j] = (-1)^popcount(i & j).  The matrix depends on n only;
    it is built once per n and returned read-only.
    """
    if n < 1 or (n & (n - 1)) != 0:
        raise ValueError("Hadamard order must be a power of two, got %d" % n)
    return _sylvester_built(n)


@functools.lru_cache(maxsize=16)
def _sylvester_built(n):
    idx = np.arange(n, dtype=np.int64)
    anded = idx[:, None] & idx[None, :]
    parity = np.zeros_like(anded)
    while np.any(anded):
        parity ^= anded & 1
        anded >>= 1
    h = np.where(parity == 0, 1.0, -1.0)
    h.setflags(write=False)
    return h


def rotation_block_matrix(signs_blk):
    """The B x B block diag(s) . H_B / sqrt(B) for one block of signs."""
    b = len(signs_blk)
    return (np.asarray(signs_blk, dtype=np.float64)[:, None] * sylvester(b)) / np.sqrt(b)


def rotate(x, signs, block):
    """X.Q for X [rows, K] (fp64), Q = blockdiag_{K/B}(diag(s_blk) H_B / sqrt(B)).

    ``block`` = 128 for 128-wide blocks, or 0 for a full-width rotation
    (B = K, K a power of two).  Returns fp64 [rows, K].
    """
    x = np.asarray(x, dtype=np.float64)
    k = x.shape[-1]
    b = k if block == 0 else block
    if k % b != 0:
        raise ValueError("K=%d is not a multiple of the block %d" % (k, b))
    signs = np.asarray(signs)
    if signs.shape != (k,):
        raise ValueError("need one sign per channel")
    out = np.empty_like(x)
    for j in range(k // b):
        sl = slice(j * b, (j + 1) * b)
        out[..., sl] = x[..., sl] @ rotation_block_matrix(signs[sl])
    return out


def rotation_matrix(signs, block):
    """The dense K x K Q (small K only; used by the invariance checks)."""
    k = len(signs)
    b = k if block == 0 else block
    q = np.zeros((k, k))
    for j in range(k // b):
        sl = slice(j * b, (j + 1) * b)
        q[sl, sl] = rotation_block_matrix(np.asarray(signs)[sl])
    return q
