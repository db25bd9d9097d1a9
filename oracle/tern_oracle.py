"""CPU oracle for ternary group-scaled weights: layouts, pack/unpack, ternarize, GEMV/GEMM.

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, obviously-correct statement of what the
CUDA library computes. It shares no code with the CUDA path and must only be imported by tests/,
__graft_entry__.smoke() and bench.py's CPU-baseline / reference legs. Every value here is fp64 (or
exact integers) and written in the order the definition states; a library matmul serves as the
dot-product step.

Sources (the ternary Bonsai web pages; section names as printed there):
  [Metal-8B]   "Metal 환경에서 삼진 모델(Ternary Model)인 Bonsai 8B를 파인튜닝(Fine-tuning)"
               (molayo1419.me), paragraph "그것을 파인튜닝(Fine-tuning)하는 방법": a weight is
               code * scale, one fp16 scale per 128 weights; ternarize per group on every forward;
               re-pack to 2-bit after re-ternarizing; the 2-bit re-encode is lossless.
  [velog-27B]  "Bonsai 27B와 1비트가 살아남는 법" (velog.io), section "포맷의 정체":
               w_i = s_g * t_i, 128 weights share one FP16 scale s_g.
  [Bonsai2]    "Ternary Bonsai 2 27B, 5.93GB로 줄이고도 FP16 성능의 98.2%를 지킨 삼진 모델"
               (discuss.pytorch.kr), section "그룹 단위 스케일을 공유하는 삼진 형식" (eqs.
               w_i = s_g t_i and b_eff ~ log2(3) + 16/128 ~ 1.71), section "두 가지 패킹:
               PTQ1_0과 PQ2_0" (packing table; a scale-only container is 34 bytes per 128 weights
               = 2.125 bits/weight), section "하이브리드 어텐션을 위한 저비트 커널" (kernels
               consume packed weights and fuse unpack + group scale into the product).

Readings of points the pages leave open (each is stated where it is used):
  R1  Q2_0_g128 bit layout: the code is t as a 2-bit two's-complement integer (0b00 = 0,
      0b01 = +1, 0b11 = -1; 0b10 is invalid); weight k of a row sits in byte k/4, bits
      2*(k%4)..2*(k%4)+1 (little-endian in k); scales are a separate fp16 array s[n][k/128]. Rows
      are K/4 bytes (always a multiple of 16 because K % 128 == 0).
  R2  Dense base-3 layout (T3_5PB_g128, 5 trits per byte): byte j of a row holds
      sum_{i<5} c_{5j+i} * 3^i with c = t + 1 (a byte > 242 is invalid); the row is a continuous
      trit stream, trits past K are c = 1 (t = 0), and the row is padded with bytes of value 121
      (five c = 1 trits) up to a multiple of 16 bytes.
  R3  Ternarize: t = round(clamp(w/s, -1, 1)) with w/s exact (fp64 quotient of two fp16 values)
      and round-half-to-even, so exact ties |w/s| = 1/2 give 0; s == 0, s NaN or w NaN give 0.
  R12 Binary layout (Q1_0_g128, weights in {-1, +1}, one fp16 scale per 128; [velog-27B] section
      "ternary와 binary가 뭔가": binary 1.125 bits per weight; [Metal-8B] opening paragraph "이
      모델들이란 무엇인가": binary weights share one fp16 scale per 128): weight k of a row is bit
      k % 8 of byte k / 8, 1 = +1 and 0 = -1; every bit pattern is valid; rows are K/8 bytes
      (a multiple of 16). Binarize: t = -1 exactly when w * s < 0 (zero and NaN give +1).
  R4  Products take x as given (any rotation of x is the caller's step) and are compared with
      |y - y_ref| <= 2e-3 * sum_k |w_k x_k| + 1e-5.
"""
from __future__ import annotations

import math

import numpy as np

GROUP = 128
Q2_0_G128 = 1
T3_5PB_G128 = 2
Q1_0_G128 = 3
LAYOUTS = (Q2_0_G128, T3_5PB_G128, Q1_0_G128)

T3_PAD_BYTE = 121  # 1 + 3 + 9 + 27 + 81: five trits with c = 1 (t = 0)
_POW3 = (1, 3, 9, 27, 81)

REL_TOL = 2e-3
ABS_TOL = 1e-5


class InvalidCode(ValueError):
    pass


# ----------------------------------------------------------------------------------------------
# layout size arithmetic  ([Bonsai2] "두 가지 패킹"; [Bonsai2] eq. b_eff)
# ----------------------------------------------------------------------------------------------
def _check(layout: int, k: int) -> None:
    if layout not in LAYOUTS:
        raise ValueError(f"unknown layout id {layout}")
    if k <= 0 or k % GROUP:
        raise ValueError(f"K must be a positive multiple of {GROUP}, got {k}")


def code_bytes(layout: int, k: int) -> int:
    """Bytes that carry the K codes of one row, before the 16-byte row padding (R1, R2)."""
    _check(layout, k)
    if layout == Q1_0_G128:
        return k // 8  # R12: one bit per weight
    return k // 4 if layout == Q2_0_G128 else -(-k // 5)


def row_bytes(layout: int, k: int) -> int:
    """Minimum row stride of the packed codes: code_bytes rounded up to 16 bytes."""
    return -(-code_bytes(layout, k) // 16) * 16


def packed_bytes(layout: int, n: int, k: int) -> int:
    return n * row_bytes(layout, k)


def bits_per_weight(layout: int, k: int) -> float:
    """Stored bits per weight: padded code row plus one 16-bit scale per 128 weights."""
    return (row_bytes(layout, k) * 8 + (k // GROUP) * 16) / k


def information_bound_bits() -> float:
    """[Bonsai2] eq. b_eff: log2(3) bits per trit plus a 16-bit scale shared by 128 weights."""
    return math.log2(3.0) + 16.0 / GROUP


# ----------------------------------------------------------------------------------------------
# pack / unpack  ([Metal-8B]: lossless re-encode; readings R1, R2)
# ----------------------------------------------------------------------------------------------
def pack(t: np.ndarray, layout: int) -> np.ndarray:
    """Pack int8 codes t [n][k] in {-1,0,1} into uint8 [n][row_bytes(layout, k)]."""
    t = np.asarray(t)
    n, k = t.shape
    _check(layout, k)
    if t.size and (t.min() < -1 or t.max() > 1):
        raise ValueError("codes must be in {-1, 0, +1}")
    out = np.zeros((n, row_bytes(layout, k)), dtype=np.uint8)
    if layout == Q1_0_G128:
        if t.size and (t == 0).any():
            raise ValueError("binary codes must be in {-1, +1}")
        bit = (t > 0).astype(np.int64).reshape(n, k // 8, 8)  # R12: bit k % 8 of byte k / 8
        out[:, : k // 8] = sum(bit[:, :, i] << i for i in range(8)).astype(np.uint8)
    elif layout == Q2_0_G128:
        c = t.astype(np.int64) & 3  # R1: 2-bit two's complement
        c4 = c.reshape(n, k // 4, 4)
        byte = c4[:, :, 0] + (c4[:, :, 1] << 2) + (c4[:, :, 2] << 4) + (c4[:, :, 3] << 6)
        out[:, : k // 4] = byte.astype(np.uint8)
    else:
        nb = code_bytes(layout, k)
        cp = np.ones((n, nb * 5), dtype=np.int64)  # trits past K are c = 1
        cp[:, :k] = t.astype(np.int64) + 1         # R2: c = t + 1
        c5 = cp.reshape(n, nb, 5)
        byte = sum(c5[:, :, i] * _POW3[i] for i in range(5))
        out[:, :nb] = byte.astype(np.uint8)
        out[:, nb:] = T3_PAD_BYTE
    return out


def unpack(codes: np.ndarray, layout: int, k: int, rows=None, check: bool = True) -> np.ndarray:
    """Unpack uint8 codes [n][stride] (stride >= row_bytes) to int8 t [len(rows)][k].

    With check=True an invalid code (Q2 field == 0b10, T3 byte > 242 among the bytes that hold the
    K codes) raises InvalidCode.
    """
    codes = np.asarray(codes, dtype=np.uint8)
    _check(layout, k)
    if rows is not None:
        codes = codes[np.asarray(rows)]
    n = codes.shape[0]
    kk = np.arange(k)
    if layout == Q1_0_G128:
        bit = (codes[:, kk // 8].astype(np.int64) >> (kk % 8)) & 1
        bad = np.zeros(bit.shape, dtype=bool)
        t = 2 * bit - 1
    elif layout == Q2_0_G128:
        byte = codes[:, kk // 4].astype(np.int64)
        f = (byte >> (2 * (kk % 4))) & 3
        bad = f == 2
        t = np.where(f == 3, -1, f)  # two's complement: 3 -> -1
    else:
        byte = codes[:, kk // 5].astype(np.int64)
        c = (byte // np.array(_POW3)[kk % 5]) % 3
        bad = byte > 242
        t = c - 1
    if check and bad.any():
        r, col = np.argwhere(bad)[0]
        raise InvalidCode(f"invalid code at row {r}, k {col}")
    t = t.astype(np.int8)
    if n == 0:
        t = t.reshape(0, k)
    return t


def count_invalid(codes: np.ndarray, layout: int, n: int, k: int) -> int:
    """Number of weights (row, k < K) whose code is invalid."""
    codes = np.asarray(codes, dtype=np.uint8)[:n]
    kk = np.arange(k)
    if layout == Q1_0_G128:
        return 0  # every bit is a valid code
    if layout == Q2_0_G128:
        f = (codes[:, kk // 4].astype(np.int64) >> (2 * (kk % 4))) & 3
        return int((f == 2).sum())
    return int((codes[:, kk // 5] > 242).sum())


def binarize(w: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """R12: t = -1 where w * s < 0 (w and its group's scale of strictly opposite signs), else +1."""
    w = np.asarray(w, dtype=np.float16).astype(np.float64)
    n, k = w.shape
    s = np.repeat(np.asarray(scales, dtype=np.float16)[:, : k // GROUP].astype(np.float64), GROUP, axis=1)
    neg = ((w < 0) & (s > 0)) | ((w > 0) & (s < 0))
    return np.where(neg, -1, 1).astype(np.int8)


def count_flips(old_codes: np.ndarray, new_codes: np.ndarray, layout: int, k: int) -> int:
    """Weights (row, k < K) whose code field differs between two packings of one matrix: the
    2-bit field (Q2) or the base-3 digit (T3), read straight from the bytes as the layout defines
    them (the QAT flip count of [Metal-8B]; for valid codes this is the number of changed t)."""
    old = np.asarray(old_codes, dtype=np.uint8)
    new = np.asarray(new_codes, dtype=np.uint8)
    _check(layout, k)
    kk = np.arange(k)
    if layout == Q1_0_G128:
        f_old = (old[:, kk // 8] >> (kk % 8)) & 1
        f_new = (new[:, kk // 8] >> (kk % 8)) & 1
    elif layout == Q2_0_G128:
        f_old = (old[:, kk // 4] >> (2 * (kk % 4))) & 3
        f_new = (new[:, kk // 4] >> (2 * (kk % 4))) & 3
    else:
        p = np.array(_POW3)[kk % 5]
        f_old = (old[:, kk // 5].astype(np.int64) // p) % 3
        f_new = (new[:, kk // 5].astype(np.int64) // p) % 3
    return int((f_old != f_new).sum())


def dequantize(t: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """fp64 w[n][k] = s[n][k/128] * t[n][k]  ([velog-27B] "포맷의 정체"; [Bonsai2] eq. w_i)."""
    n, k = t.shape
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)[:, : k // GROUP]
    return np.repeat(s, GROUP, axis=1) * t.astype(np.float64)


# ----------------------------------------------------------------------------------------------
# ternarize  ([Metal-8B]: per-group ternarization of latents, then re-pack; reading R3)
# ----------------------------------------------------------------------------------------------
def ternarize(w: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """int8 t[n][k] = round_half_even(clamp(w / s, -1, 1)) per weight with its group's scale."""
    w = np.asarray(w, dtype=np.float16)
    n, k = w.shape
    s = np.repeat(np.asarray(scales, dtype=np.float16).astype(np.float64)[:, : k // GROUP], GROUP, axis=1)
    wd = w.astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = wd / s
    dead = (s == 0) | np.isnan(s) | np.isnan(wd) | np.isnan(q)
    q = np.where(dead, 0.0, q)
    t = np.rint(np.clip(q, -1.0, 1.0))  # np.rint rounds half to even
    return t.astype(np.int8)


# ----------------------------------------------------------------------------------------------
# products  ([Bonsai2] "하이브리드 어텐션을 위한 저비트 커널": y = W x with W = s * t)
# ----------------------------------------------------------------------------------------------
def gemv(codes, scales, x, layout: int, k: int, rows=None):
    """y_ref[b][n] = sum_k w[n][k] * x[b][k] in fp64 and A[b][n] = sum_k |w[n][k] * x[b][k]|.

    codes: uint8 [N][stride]; scales: fp16 [N][>=K/128]; x: fp16 [B][K]. `rows` restricts the
    output to a subset of rows (sampled checks at full size).
    """
    sc = np.asarray(scales, dtype=np.float16)
    if rows is not None:
        sc = sc[np.asarray(rows)]
    t = unpack(codes, layout, k, rows=rows)
    w = dequantize(t, sc)
    xd = np.asarray(x, dtype=np.float16).astype(np.float64)
    y = xd @ w.T
    a = np.abs(xd) @ np.abs(w).T
    return y, a


def gemv_t(codes, scales, dy, layout: int, k: int, cols=None):
    """dx_ref[b][k] = sum_n w[n][k] * dy[b][n] in fp64 (the transposed product W^T dy of the STE
    backward, [Metal-8B]) and A[b][k] = sum_n |w[n][k] * dy[b][n]|; `cols` selects output columns.

    codes: uint8 [N][stride]; scales: fp16 [N][>=K/128]; dy: fp16 [B][N].
    """
    t = unpack(codes, layout, k)
    w = dequantize(t, np.asarray(scales, dtype=np.float16))
    if cols is not None:
        w = w[:, np.asarray(cols)]
    dyd = np.asarray(dy, dtype=np.float16).astype(np.float64)
    return dyd @ w, np.abs(dyd) @ np.abs(w)


def gemm(codes, scales, X, layout: int, k: int, rows=None):
    """Y_ref[m][n] = sum_k X[m][k] * s[n][k/128] * t[n][k] (fp64) and the matching A.

    The prefill product is the same contraction as the GEMV with M tokens in place of the batch;
    `rows` selects token rows m of the output.
    """
    Xd = np.asarray(X, dtype=np.float16)
    if rows is not None:
        Xd = Xd[np.asarray(rows)]
    return gemv(codes, scales, Xd, layout, k)


def tolerance(a: np.ndarray) -> np.ndarray:
    """Allowed |y - y_ref| for a product whose sum of |w x| is a (reading R4)."""
    return REL_TOL * np.asarray(a) + ABS_TOL


def within_tolerance(y, y_ref, a) -> np.ndarray:
    y = np.asarray(y, dtype=np.float64)
    return np.abs(y - y_ref) <= tolerance(a)
