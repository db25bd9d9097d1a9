"""CPU oracle for the activation-side block Hadamard rotation (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference legs import this module.
It shares no code with the CUDA path.

Source: "Ternary Bonsai 2 27B, 5.93GB로 줄이고도 FP16 성능의 98.2%를 지킨 삼진 모델"
(discuss.pytorch.kr), section "블록 단위 하다마드 회전": the stored ternary weights live in a rotated
basis, R = (1/sqrt(n)) H_n S with n = 1024, H_n the Walsh-Hadamard matrix and S a fixed diagonal of
+-1 signs, and each layer computes f(x) = W (R x); section "처리량": at run time every projection is
preceded by the sign flip and a block fast Walsh-Hadamard transform of the activations.

Readings of points the page leaves open:
  R9   H_n is the Sylvester (natural-order) Walsh-Hadamard matrix, H[i][j] = (-1)^popcount(i & j),
       built here by the recursion H_2m = [[H_m, H_m], [H_m, -H_m]].
  R10  S is given by the caller as n signs (negative entry = -1, anything else = +1), the same S for
       every block; R acts on each consecutive n-element block of x independently (K % 1024 == 0).
  R11  The rotated activations are fp16 like x; the transform itself is exact in fp64 here.
Parity of the pages' own transform kernels is unpinned (the pages print no kernel or example).
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 1024


def hadamard(n: int) -> np.ndarray:
    """Sylvester Walsh-Hadamard matrix H_n (n a power of two) as float64, by the doubling recursion."""
    if n < 1 or n & (n - 1):
        raise ValueError("n must be a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def sign_diagonal(signs: np.ndarray) -> np.ndarray:
    """The diagonal of S: -1 where the caller's sign is negative, +1 elsewhere (R10)."""
    s = np.asarray(signs)
    if s.shape != (BLOCK,):
        raise ValueError("signs must have 1024 entries")
    return np.where(s < 0, -1.0, 1.0)


def rotate(x: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """y = R x per 1024-block of every row of x ([batch][k] or [k]), R = H S / sqrt(1024), in fp64."""
    x = np.asarray(x, dtype=np.float64)
    squeeze = x.ndim == 1
    x2 = x.reshape(1, -1) if squeeze else x
    b, k = x2.shape
    if k % BLOCK:
        raise ValueError("k must be a multiple of 1024")
    r = hadamard(BLOCK) * sign_diagonal(signs)[None, :] / math.sqrt(BLOCK)  # R = H S / sqrt(n)
    blocks = x2.reshape(b, k // BLOCK, BLOCK)
    y = blocks @ r.T  # each block: R x_blk
    y = y.reshape(b, k)
    return y[0] if squeeze else y


def rotate_tolerance(x: np.ndarray, y_ref: np.ndarray) -> np.ndarray:
    """Bound for an fp32 transform rounded once to fp16: 2^-11 |y| for the final rounding plus
    2^-18 * (1/32) sum_j |x_j| over the block (ten fp32 butterfly stages, with a wide margin)."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    b = x.reshape(-1, x.shape[-1] // BLOCK, BLOCK).sum(axis=2) / 32.0
    mass = np.repeat(b, BLOCK, axis=1).reshape(np.shape(y_ref))
    return 2.0 ** -11 * np.abs(y_ref) + 2.0 ** -18 * mass + 1e-7
