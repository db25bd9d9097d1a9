"""Shared helpers for the GPU parity tests: seeded workloads, oracle packing in row chunks, and
the tolerance check. Inputs come from gemm_tern_gemv_b200.synth; expected values from oracle/."""
from __future__ import annotations

import numpy as np

import oracle as O
from gemm_tern_gemv_b200 import synth

CHUNK_ROWS = 4096


def pack_rows(t: np.ndarray, layout: int) -> np.ndarray:
    """Oracle packing of t [n][k], one row chunk at a time (bounded host memory)."""
    n, k = t.shape
    out = np.empty((n, O.row_bytes(layout, k)), dtype=np.uint8)
    for r in range(0, n, CHUNK_ROWS):
        out[r : r + CHUNK_ROWS] = O.pack(t[r : r + CHUNK_ROWS], layout)
    return out


def ternarize_rows(w: np.ndarray, s: np.ndarray) -> np.ndarray:
    n, k = w.shape
    out = np.empty((n, k), dtype=np.int8)
    for r in range(0, n, CHUNK_ROWS):
        out[r : r + CHUNK_ROWS] = O.ternarize(w[r : r + CHUNK_ROWS], s[r : r + CHUNK_ROWS])
    return out


def workload(layout: int, n: int, k: int, batch: int, seed: int, p_zero: float = 0.4):
    """(codes uint8 [n][row_bytes], scales fp16 [n][k/128], x fp16 [batch][k])."""
    if layout == O.Q1_0_G128:
        t = synth.binary_codes(n, k, seed)
    else:
        t = synth.ternary_codes(n, k, seed, p_zero=p_zero)
    s = synth.group_scales(n, k // 128, seed)
    x = synth.activations(batch, k, seed)
    return pack_rows(t, layout), s, x


def sample_rows(n: int, count: int, seed: int) -> np.ndarray:
    """Sorted sample of rows that always includes the first and last 16 rows (ragged tails)."""
    if n <= count:
        return np.arange(n)
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(n, size=count, replace=False).tolist())
    pick.update(range(16))
    pick.update(range(n - 16, n))
    return np.array(sorted(pick))


def check_product(y_gpu: np.ndarray, y_ref: np.ndarray, a: np.ndarray, what: str) -> float:
    """Asserts |y - y_ref| <= 2e-3 * A + 1e-5 elementwise; returns the worst error/tolerance ratio."""
    y = np.asarray(y_gpu, dtype=np.float64)
    assert y.shape == y_ref.shape, (what, y.shape, y_ref.shape)
    assert np.isfinite(y).all(), what
    tol = O.tolerance(a)
    ratio = np.abs(y - y_ref) / tol
    worst = float(ratio.max()) if ratio.size else 0.0
    if worst > 1.0:
        i = np.unravel_index(int(ratio.argmax()), ratio.shape)
        raise AssertionError(f"{what}: |y-y_ref|/tol = {worst:.3g} at {i}: y={y[i]!r} ref={y_ref[i]!r} A={a[i]!r}")
    return worst
