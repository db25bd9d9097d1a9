"""Pins of the block Hadamard rotation oracle (CPU): what the mathematics fixes about R = H S / 32.

Source: "Ternary Bonsai 2 27B ..." (discuss.pytorch.kr), section "블록 단위 하다마드 회전"
(R = H_n S / sqrt(n), n = 1024; f(x) = W(Rx))."""
import math

import numpy as np
import pytest

import oracle as O

N = O.ROTATE_BLOCK


def _signs(seed):
    return np.where(np.random.default_rng(seed).random(N) < 0.5, -1, 1).astype(np.int8)


def test_hadamard_entries_are_popcount_parity():
    # Sylvester order: H[i][j] = (-1)^popcount(i & j), computed here without the recursion
    h = O.hadamard(N)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    bits = np.bitwise_and(i, j)
    pc = np.zeros_like(bits)
    for b in range(10):
        pc += (bits >> b) & 1
    assert np.array_equal(h, np.where(pc % 2 == 0, 1.0, -1.0))


def test_hadamard_small_matrix_literal():
    assert np.array_equal(O.hadamard(4), np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], float))


def test_hadamard_orthogonal():
    h = O.hadamard(N)
    assert np.array_equal(h @ h.T, N * np.eye(N))


def test_rotation_is_orthogonal_and_invertible():
    s = _signs(1)
    x = np.random.default_rng(2).standard_normal((3, 2 * N))
    y = O.rotate(x, s)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    # R^T = S H / 32 undoes R
    d = O.sign_diagonal(s)
    back = (y.reshape(3, 2, N) @ O.hadamard(N).T / 32.0) * d
    assert np.allclose(back.reshape(3, 2 * N), x, rtol=0, atol=1e-12)


def test_rotation_of_basis_vectors_is_signed_column():
    # R e_j = s_j H[:, j] / 32 (the sign multiplies the input, before H)
    s = _signs(3)
    h = O.hadamard(N)
    for j in (0, 1, 7, 513, 1023):
        e = np.zeros(N)
        e[j] = 1.0
        assert np.array_equal(O.rotate(e, s), s[j] * h[:, j] / 32.0)


def test_rotation_of_constant_block():
    # all signs +1: H 1 = N e_0, so R (c 1) = 32 c e_0
    y = O.rotate(np.full(N, 3.0), np.ones(N, dtype=np.int8))
    want = np.zeros(N)
    want[0] = 32.0 * 3.0
    assert np.array_equal(y, want)


def test_blocks_are_independent():
    s = _signs(4)
    a, b = np.random.default_rng(5).standard_normal((2, N))
    both = O.rotate(np.concatenate([a, b]), s)
    assert np.allclose(both, np.concatenate([O.rotate(a, s), O.rotate(b, s)]), rtol=0, atol=1e-12)


def test_k_must_be_block_multiple():
    with pytest.raises(ValueError):
        O.rotate(np.zeros(1000), np.ones(N))
    with pytest.raises(ValueError):
        O.rotate(np.zeros(N), np.ones(10))


def test_planted_mistakes_are_caught():
    s = _signs(6)
    h = O.hadamard(N)
    x = np.random.default_rng(7).standard_normal(N)
    y = O.rotate(x, s)
    d = O.sign_diagonal(s)
    assert not np.allclose(y, d * (h @ x) / 32.0)               # S applied after H
    assert not np.allclose(y, h @ (d * x))                      # scale 1/sqrt(n) dropped
    seq = h[np.argsort([np.count_nonzero(np.diff(r)) for r in h], kind="stable")]
    assert not np.allclose(y, seq @ (d * x) / 32.0)              # sequency (Walsh) row order
    assert math.isclose(np.linalg.norm(y), np.linalg.norm(x), rel_tol=1e-12)
