"""Pins for the oracle's rotation (CPU only).

Each check fixes the oracle against something other than itself: the
textbook doubling construction, the orthogonality closed form H.H^T = nI, an
independent butterfly transform, the article's one-hot outlier example and the
computational invariance of "Rotations for 4-Bit Activations: QuaRot,
SpinQuant, and Friends", section "A rotation changes nothing, and that is the
point".
"""

import numpy as np
import pytest

from oracle import hadamard


def _doubling(n):
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def _butterfly(x, signs, block):
    """In-place fast Walsh-Hadamard transform by butterflies (not a matmul)."""
    y = np.array(x, dtype=np.float64) * signs
    n = y.shape[-1]
    b = n if block == 0 else block
    for base in range(0, n, b):
        h = 1
        while h < b:
            for i in range(base, base + b, 2 * h):
                for j in range(i, i + h):
                    a, c = y[..., j].copy(), y[..., j + h].copy()
                    y[..., j], y[..., j + h] = a + c, a - c
            h *= 2
        y[..., base:base + b] /= np.sqrt(b)
    return y


def test_h4_matches_golden(golden):
    rows = [list(map(float, r.split())) for r in golden("hadamard_h4.txt")]
    assert np.array_equal(hadamard.sylvester(4), np.array(rows))


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_sylvester_equals_doubling(n):
    assert np.array_equal(hadamard.sylvester(n), _doubling(n))


@pytest.mark.parametrize("n", [1 << p for p in range(13)])
def test_orthogonality_closed_form(n):
    h = hadamard.sylvester(n)
    assert np.array_equal(h @ h.T, n * np.eye(n))
    assert set(np.unique(h)) <= {-1.0, 1.0}


def test_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        hadamard.sylvester(12)


@pytest.mark.parametrize("n,block", [(2, 0), (4, 0), (8, 0), (16, 0), (16, 4), (16, 8), (32, 16), (12, 4),
                                     (64, 32), (128, 16), (128, 32)])
def test_rotate_matches_butterfly(n, block):
    rng = np.random.default_rng(7 + n + block)
    x = rng.standard_normal((5, n))
    s = rng.choice([-1, 1], size=n)
    assert np.allclose(hadamard.rotate(x, s, block), _butterfly(x, s, block), rtol=0, atol=1e-13)


def test_onehot_outlier_golden(golden):
    vals = list(map(float, golden("onehot_outlier.txt")[0].split()))
    n, ch, m = int(vals[0]), int(vals[1]), vals[2]
    expect = np.array(vals[3:])
    x = np.zeros((1, n))
    x[0, ch] = m
    got = hadamard.rotate(x, np.ones(n, dtype=np.int8), 0)
    assert np.array_equal(got[0], expect)
    assert np.all(np.abs(got) == m / np.sqrt(n))


@pytest.mark.parametrize("k,block", [(512, 128), (256, 0), (384, 128), (256, 16), (256, 32)])
def test_onehot_spreads_to_block(k, block):
    """Each one-hot input maps to a row of Q: +-1/sqrt(B) inside its block, 0 outside."""
    rng = np.random.default_rng(3)
    s = rng.choice([-1, 1], size=k)
    b = k if block == 0 else block
    eye = np.eye(k)
    r = hadamard.rotate(eye, s, block)
    for j in range(0, k, 37):
        blk = j // b
        inside = r[j, blk * b:(blk + 1) * b]
        assert np.allclose(np.abs(inside), 1 / np.sqrt(b), atol=1e-15)
        out = np.delete(r[j], np.s_[blk * b:(blk + 1) * b])
        assert np.all(out == 0)


@pytest.mark.parametrize("k,block", [(512, 128), (1024, 0), (768, 128)])
def test_invariance_exact_fp64(k, block):
    """(X.Q)(W.Q)^T == X.W^T to fp64 rounding (computational invariance)."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((32, k))
    x[:, 5] *= 50
    w = 0.02 * rng.standard_normal((48, k))
    s = rng.choice([-1, 1], size=k)
    y = x @ w.T
    yr = hadamard.rotate(x, s, block) @ hadamard.rotate(w, s, block).T
    assert np.linalg.norm(y - yr) / np.linalg.norm(y) <= 1e-12


def test_rotation_is_orthogonal_and_norm_preserving():
    rng = np.random.default_rng(5)
    s = rng.choice([-1, 1], size=256)
    q = hadamard.rotation_matrix(s, 128)
    assert np.allclose(q @ q.T, np.eye(256), atol=1e-14)
    x = rng.standard_normal((9, 256))
    assert np.allclose(np.linalg.norm(hadamard.rotate(x, s, 128), axis=1), np.linalg.norm(x, axis=1))


def test_sign_flip_changes_result():
    """A wrong sign vector must give a different rotation (guards a dropped D)."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 128))
    s = rng.choice([-1, 1], size=128)
    assert not np.allclose(hadamard.rotate(x, s, 128), hadamard.rotate(x, np.ones(128), 128))


def test_block_of_one_is_the_sign_diagonal():
    """block = 1 (the unrotated arm): H_1 = [1], so Q = diag(s) and X.Q flips
    the signs of the channels and nothing else."""
    rng = np.random.default_rng(31)
    x = rng.standard_normal((5, 64))
    s = rng.choice([-1, 1], size=64)
    assert np.array_equal(hadamard.rotate(x, s, 1), x * s)
    assert np.array_equal(hadamard.rotate(x, np.ones(64, dtype=np.int64), 1), x)
