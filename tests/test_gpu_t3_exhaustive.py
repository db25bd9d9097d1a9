"""Every ordered pair of valid base-3 bytes, in both 16-bit lanes of a 32-bit word, through every
product kernel that decodes the dense layout in registers.

The base-3 decoders work on two bytes at a time: bytes (0, 2) and (1, 3) of a word share a 32-bit
register as 16-bit lanes, and a carry from one lane to the other could corrupt a neighbour only for
particular byte pairs. Here word w of the matrix holds the pair number w in lanes (0, 2) and a shifted
pair in lanes (1, 3), so each of the 243^2 pairs occurs in both lanes ("Ternary Bonsai 2 27B ..."
discuss.pytorch.kr, section "두 가지 패킹: PTQ1_0과 PQ2_0": the dense trit packing). Scales are 1
and activations small integers, so every result is an exact integer and is compared for equality:
  * the int8-plane GEMV (K = 5120, a whole number of 32-byte units), batches 1 and 2;
  * the register GEMV (K = 4992, not a whole number of units), batches 1 and 2;
  * the transposed product W^T dy.
"""
import numpy as np
import pytest

import oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402

PAIRS = 243 * 243


def _codes(n, k, seed):
    """uint8 [n][row_bytes]: data words cycle through every byte pair in both lanes."""
    rb = T.row_bytes(T.T3_5PB_G128, k)
    full = k // 5  # bytes whose five trits are all below K
    words_per_row = full // 4
    assert n * words_per_row >= PAIRS
    rng = np.random.default_rng(seed)
    codes = np.full((n, rb), 121, dtype=np.uint8)  # 121: five trits c = 1 (t = 0)
    w = np.arange(n * words_per_row)
    off = int(rng.integers(0, PAIRS))
    a = w % PAIRS
    b = (w + off) % PAIRS
    words = np.stack([a % 243, b % 243, a // 243, b // 243], axis=1).astype(np.uint8)  # bytes 0..3
    codes[:, : 4 * words_per_row] = words.reshape(n, 4 * words_per_row)
    # bytes between the last whole word and K: random valid bytes; a byte straddling K keeps its
    # trits past K at c = 1
    for j in range(4 * words_per_row, rb):
        lo = 5 * j
        if lo + 5 <= k:
            codes[:, j] = rng.integers(0, 243, size=n)
        elif lo < k:
            m = k - lo
            d = rng.integers(0, 3, size=(n, m))
            codes[:, j] = (d * (3 ** np.arange(m))).sum(axis=1) + sum(3**i for i in range(m, 5))
    return codes


def _small_ints(shape, seed, density=0.125):
    # +-1 / +-2 on a sparse support: |result| stays far below 2048, exact in fp16
    rng = np.random.default_rng(seed)
    v = rng.choice([-2, -1, 1, 2], size=shape) * (rng.random(shape) < density)
    return v.astype(np.float16)


@pytest.mark.parametrize("k", [5120, 4992])
@pytest.mark.parametrize("batch", [1, 2])
def test_gemv_every_byte_pair_exact(k, batch):
    n = 256
    codes = _codes(n, k, seed=k + batch)
    s = np.ones((n, k // 128), dtype=np.float16)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), T.T3_5PB_G128, k)
    # eight activation patterns whose supports cover every k (k mod 8), so every trit is exercised
    rng = np.random.default_rng(k)
    for part in range(8):
        x = np.zeros((batch, k), dtype=np.float16)
        sel = (np.arange(k) % 8) == part
        x[:, sel] = rng.choice([-2, -1, 1, 2], size=(batch, int(sel.sum()))).astype(np.float16)
        y = T.gemv(W, torch.from_numpy(x).cuda())
        torch.cuda.synchronize()
        y_ref, _ = O.gemv(codes, s, x, T.T3_5PB_G128, k)
        assert np.abs(y_ref).max() < 2048
        assert np.array_equal(y.cpu().numpy().astype(np.float64), y_ref), (k, batch, part)


def test_gemv_t_every_byte_pair_exact():
    n, k, batch = 256, 5120, 2
    codes = _codes(n, k, seed=7)
    s = np.ones((n, k // 128), dtype=np.float16)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), T.T3_5PB_G128, k)
    dy = _small_ints((batch, n), seed=8, density=1.0)
    dx = T.gemv_t(W, torch.from_numpy(dy).cuda())
    torch.cuda.synchronize()
    ref = O.gemv_t(codes, s, dy, T.T3_5PB_G128, k)
    ref = ref[0] if isinstance(ref, tuple) else ref
    assert np.abs(ref).max() < 2048
    assert np.array_equal(dx.cpu().numpy().astype(np.float64), ref)


def test_the_matrices_hold_every_pair_in_both_lanes():
    # the construction itself, checked on the CPU side of the test: both lane pairs see all 243^2
    for k in (5120, 4992):
        codes = _codes(256, k, seed=k + 1)
        words = codes[:, : 4 * ((k // 5) // 4)].reshape(-1, 4).astype(np.int64)
        assert len(np.unique(words[:, 0] + 243 * words[:, 2])) == PAIRS
        assert len(np.unique(words[:, 1] + 243 * words[:, 3])) == PAIRS
        O.unpack(codes, T.T3_5PB_G128, k)  # every byte valid, padding trits included
