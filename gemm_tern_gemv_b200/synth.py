"""Seeded synthetic inputs for the ternary products: codes, group scales, activations, latents.

This module only draws random numbers with the workload's distributions. It holds none of the
product, packing or ternarisation arithmetic, so the CUDA path and the CPU oracle can both take
their inputs from here without sharing any of the method's code.

Distributions (the workloads of the ternary Bonsai pages: 8B- and 27B-class layers):
  * ternary codes t, iid: P(t=0)=0.4, P(t=+1)=P(t=-1)=0.3, drawn as u~U[0,1):
    t=-1 if u<0.3, t=0 if u<0.7, else t=+1;
  * group scales: fp16(|N(0,1)| * 0.02), round to nearest;
  * activations: fp16(N(0,1));
  * pack latents: w = fp16(s*t + 0.3*s*N(0,1)), s being the weight's group scale.

The generator is numpy's counter-based Philox, keyed by (seed, stream), so every tensor of a
workload has its own independent, reproducible stream.
"""
from __future__ import annotations

import numpy as np

GROUP = 128

# stream ids: one independent Philox stream per tensor kind
_S_CODES, _S_SCALES, _S_ACT, _S_NOISE = 1, 2, 3, 4

_CHUNK = 1 << 22  # values drawn per chunk, bounds host memory for the 622M-weight LM head


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([int(seed), int(stream)])))


def ternary_codes(n: int, k: int, seed: int, p_zero: float = 0.4) -> np.ndarray:
    """int8 [n][k] of t in {-1,0,+1}, P(0)=p_zero, P(+1)=P(-1)=(1-p_zero)/2."""
    rng = _rng(seed, _S_CODES)
    lo = (1.0 - p_zero) / 2.0
    hi = lo + p_zero
    out = np.empty(n * k, dtype=np.int8)
    for s in range(0, n * k, _CHUNK):
        e = min(n * k, s + _CHUNK)
        u = rng.random(e - s)
        t = np.ones(e - s, dtype=np.int8)
        t[u < hi] = 0
        t[u < lo] = -1
        out[s:e] = t
    return out.reshape(n, k)


def binary_codes(n: int, k: int, seed: int) -> np.ndarray:
    """int8 [n][k] of t in {-1,+1} with P(+1) = P(-1) = 1/2 (the binary layout's codes)."""
    return ternary_codes(n, k, seed, p_zero=0.0)


def codes_for(layout: int, n: int, k: int, seed: int) -> np.ndarray:
    """Codes of the distribution a layout holds: binary for layout 3 (Q1_0_g128), else ternary."""
    return binary_codes(n, k, seed) if layout == 3 else ternary_codes(n, k, seed)


def group_scales(n: int, groups: int, seed: int, sigma: float = 0.02) -> np.ndarray:
    """float16 [n][groups] = fp16(|N(0,1)|*sigma)."""
    rng = _rng(seed, _S_SCALES)
    return (np.abs(rng.standard_normal((n, groups))) * sigma).astype(np.float16)


def activations(b: int, k: int, seed: int) -> np.ndarray:
    """float16 [b][k] = fp16(N(0,1))."""
    rng = _rng(seed, _S_ACT)
    return rng.standard_normal((b, k)).astype(np.float16)


def latents(t: np.ndarray, scales: np.ndarray, seed: int, noise: float = 0.3) -> np.ndarray:
    """float16 [n][k] = fp16(s*t + noise*s*N(0,1)) with s the group scale of each weight.

    This is the synthetic recipe for drifted QAT latents around a ternary checkpoint; it is an
    input construction only (nothing here decides a code).
    """
    n, k = t.shape
    rng = _rng(seed, _S_NOISE)
    s = np.repeat(scales.astype(np.float64), GROUP, axis=1)[:, :k]
    z = rng.standard_normal((n, k))
    return (s * (t.astype(np.float64) + noise * z)).astype(np.float16)


def seed_for(config: int, matrix: int) -> int:
    """Seed of matrix `matrix` in workload `config` (the 1024x1024 GEMV uses seed 0)."""
    return 0 if config == 1 else 100 * config + matrix
