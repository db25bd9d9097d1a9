"""Pins for the CPU oracle: page-printed numbers, exhaustive byte tables, round trips, closed forms,
brute force on tiny inputs, and planted mistakes that the pins must catch.

None of these compares the oracle with itself: every expected value comes from the pages, from a
hand derivation stored under tests/golden/, from exact integer / exactly-rounded arithmetic
written independently here, or from a closed form.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from gemm_tern_gemv_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
CONFIG_K = (1024, 4096, 5120, 12288, 17408)


def _golden_bits():
    vals = {}
    with open(os.path.join(GOLDEN, "bits_per_weight.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                name, v, tol = line.split()[:3]
                vals[name] = (float(v), float(tol))
    return vals


def _golden_hand():
    cases = []
    with open(os.path.join(GOLDEN, "hand_packed.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            lhs, rhs = line.split("->")
            parts = lhs.split()
            layout = {"Q2": O.Q2_0_G128, "T3": O.T3_5PB_G128, "Q1": O.Q1_0_G128}[parts[0]]
            t = [int(v) for v in parts[1:]]
            b = [int(v, 16) for v in rhs.split()]
            cases.append((layout, t, b))
    return cases


# ---------------------------------------------------------------- layout arithmetic vs the pages
def test_bits_per_weight_against_pages():
    g = _golden_bits()
    # Q2_0_g128: 128 weights -> 32 code bytes + 2 scale bytes = the page's 34-byte container
    assert O.row_bytes(O.Q2_0_G128, 128) + 2 == 34
    for k in CONFIG_K:
        assert O.bits_per_weight(O.Q2_0_G128, k) == g["q2_container_bits"][0]
    # the MLX container adds a 2-byte bias per group: 36 bytes -> 2.25 bits/weight
    assert (O.row_bytes(O.Q2_0_G128, 128) + 2 + 2) * 8 / 128 == g["mlx_container_bits"][0]
    bound, tol = g["ternary_bound_bits"]
    assert abs(O.information_bound_bits() - bound) <= tol
    assert O.bits_per_weight(O.T3_5PB_G128, 5120) == g["base3_bits_k5120"][0]
    for k in CONFIG_K:
        b = O.bits_per_weight(O.T3_5PB_G128, k)
        assert O.information_bound_bits() < b <= g["ptq1_0_bits_upper"][0]


def test_row_bytes_closed_forms():
    for k in range(128, 20000, 128):
        assert O.row_bytes(O.Q2_0_G128, k) == k // 4
        rb = O.row_bytes(O.T3_5PB_G128, k)
        assert rb % 16 == 0 and rb * 5 >= k and (rb - 16) * 5 < k
        assert O.row_bytes(O.Q1_0_G128, k) == k // 8
    with pytest.raises(ValueError):
        O.row_bytes(O.Q2_0_G128, 100)
    with pytest.raises(ValueError):
        O.row_bytes(4, 128)


# ---------------------------------------------------------------- exhaustive byte tables
def test_q2_byte_table_exhaustive():
    codes = np.zeros((256, 32), dtype=np.uint8)
    codes[:, 0] = np.arange(256)
    valid = 0
    for byte in range(256):
        fields = [(byte >> (2 * i)) & 3 for i in range(4)]
        if 2 in fields:
            with pytest.raises(O.InvalidCode):
                O.unpack(codes[byte : byte + 1], O.Q2_0_G128, 128)
            continue
        valid += 1
        t = O.unpack(codes[byte : byte + 1], O.Q2_0_G128, 128)
        # a 2-bit two's-complement field: 0b11 is -1
        assert list(t[0, :4]) == [f - 4 if f >= 2 else f for f in fields]
        assert O.pack(t, O.Q2_0_G128)[0, 0] == byte
    assert valid == 3**4


def test_q2_count_invalid_is_the_number_of_0b10_fields():
    # every byte value in the first byte of its row; the count must equal the number of 2-bit fields
    # equal to 0b10 (the one invalid code), counted here bit by bit, independently of the oracle
    codes = np.zeros((256, 32), dtype=np.uint8)
    codes[:, 0] = np.arange(256)
    expected = 0
    for byte in range(256):
        for i in range(4):
            hi, lo = (byte >> (2 * i + 1)) & 1, (byte >> (2 * i)) & 1
            expected += int(hi == 1 and lo == 0)
    assert expected == 4 * 64  # each field position holds 0b10 in a quarter of the 256 bytes
    assert O.count_invalid(codes, O.Q2_0_G128, 256, 128) == expected
    # per row, including bytes past the first and rows with several invalid fields
    for byte in (0x02, 0x08, 0x20, 0x80, 0xAA, 0x55, 0xFF, 0x00):
        row = np.full((1, 32), byte, dtype=np.uint8)
        per_byte = sum(((byte >> (2 * i)) & 3) == 2 for i in range(4))
        assert O.count_invalid(row, O.Q2_0_G128, 1, 128) == 32 * per_byte


def test_t3_byte_table_exhaustive():
    codes = np.full((256, 32), O.T3_PAD_BYTE, dtype=np.uint8)
    codes[:, 0] = np.arange(256)
    for byte in range(256):
        if byte > 242:
            with pytest.raises(O.InvalidCode):
                O.unpack(codes[byte : byte + 1], O.T3_5PB_G128, 128)
            continue
        t = O.unpack(codes[byte : byte + 1], O.T3_5PB_G128, 128)
        digits = [int(v) + 1 for v in t[0, :5]]
        assert all(0 <= d <= 2 for d in digits)
        assert sum(d * 3**i for i, d in enumerate(digits)) == byte  # base-3 identity
        assert O.pack(t, O.T3_5PB_G128)[0, 0] == byte
    # an invalid byte makes all five of its weights invalid
    assert O.count_invalid(codes, O.T3_5PB_G128, 256, 128) == 5 * (256 - 243)


def test_hand_packed_golden():
    seen = set()
    for layout, t, expect in _golden_hand():
        seen.add(layout)
        # the rest of the row is t = 0 (t = -1 for the binary layout, which has no zero)
        row = np.full((1, 128), -1 if layout == O.Q1_0_G128 else 0, dtype=np.int8)
        row[0, : len(t)] = t
        p = O.pack(row, layout)
        assert list(p[0, : len(expect)]) == expect, (layout, t)
        assert list(O.unpack(p, layout, 128)[0]) == list(row[0])
    assert seen == set(O.LAYOUTS)


def test_t3_padding_bytes():
    k = 4096  # 4096 trits -> 820 bytes, row padded to 832 with 121s; trits 4096..4099 are c=1
    t = synth.ternary_codes(3, k, seed=7)
    p = O.pack(t, O.T3_5PB_G128)
    assert p.shape == (3, 832)
    assert (p[:, 820:] == O.T3_PAD_BYTE).all()
    last = p[:, 819].astype(int)
    # byte 819 holds k = 4095 (digit 0) and four padding trits (c = 1)
    assert ((last - (t[:, 4095] + 1)) == 3 + 9 + 27 + 81).all()


# ---------------------------------------------------------------- round trips (lossless re-encode)
@pytest.mark.parametrize("layout", O.LAYOUTS)
@pytest.mark.parametrize("k", [128, 256, 384, 640, 1024, 1152, 4096, 5120])
def test_round_trip(layout, k):
    t = synth.codes_for(layout, 17, k, seed=k + layout)
    p = O.pack(t, layout)
    assert p.shape == (17, O.row_bytes(layout, k))
    assert np.array_equal(O.unpack(p, layout, k), t)
    assert np.array_equal(O.pack(O.unpack(p, layout, k), layout), p)


def test_unpack_row_subset_and_stride():
    k = 1024
    t = synth.ternary_codes(9, k, seed=3)
    p = O.pack(t, O.T3_5PB_G128)
    wide = np.zeros((9, p.shape[1] + 48), dtype=np.uint8)  # caller stride > row bytes
    wide[:, : p.shape[1]] = p
    assert np.array_equal(O.unpack(wide, O.T3_5PB_G128, k, rows=[8, 1, 4]), t[[8, 1, 4]])


# ---------------------------------------------------------------- ternarize
def test_ternarize_is_lossless_on_scaled_codes():
    n, k = 64, 1024
    t = synth.ternary_codes(n, k, seed=11)
    s = synth.group_scales(n, k // 128, seed=11)
    s[s == 0] = np.float16(0.01)
    w = (np.repeat(s.astype(np.float64), 128, axis=1) * t).astype(np.float16)  # exact: s*t
    assert np.array_equal(O.ternarize(w, s), t)


def test_ternarize_ties_and_specials():
    s = np.float16(0.015625 * 1.5)  # 0.0234375, exactly representable
    half = np.float16(float(s) / 2)  # exact half
    assert float(half) * 2 == float(s)
    up = np.nextafter(half, np.float16(1))
    down = np.nextafter(half, np.float16(0))
    vals = [half, -half, up, -up, down, -down, np.float16(0), np.float16(-0.0),
            np.float16(np.inf), np.float16(-np.inf), np.float16(np.nan), s, -s, s * 3]
    expect = [0, 0, 1, -1, 0, 0, 0, 0, 1, -1, 0, 1, -1, 1]
    w = np.zeros((1, 128), dtype=np.float16)
    w[0, : len(vals)] = vals
    sc = np.full((1, 1), s, dtype=np.float16)
    assert list(O.ternarize(w, sc)[0, : len(vals)]) == expect
    # negative scale flips the sign; zero / NaN scale kills the group; inf scale gives 0
    for sv, want in ((-s, [0, 0, -1, 1]), (np.float16(0), [0, 0, 0, 0]),
                     (np.float16(np.nan), [0, 0, 0, 0]), (np.float16(np.inf), [0, 0, 0, 0])):
        sc = np.full((1, 1), sv, dtype=np.float16)
        assert list(O.ternarize(w, sc)[0, :4]) == want, sv


def test_ternarize_flip_rate_matches_noise_model():
    # w/s = t + 0.3 z. A t = 0 code flips when |0.3 z| > 1/2, i.e. |z| > 5/3; a t = +-1 code flips
    # when t*(t + 0.3 z) <= 1/2, i.e. z beyond 5/3 toward zero. Hence
    # P(flip) = 0.4 * 2*Phi(-5/3) + 0.6 * Phi(-5/3) = 6.69 %.
    n, k = 512, 4096
    t = synth.ternary_codes(n, k, seed=5)
    s = synth.group_scales(n, k // 128, seed=5)
    w = synth.latents(t, s, seed=5)
    live = np.repeat(s, 128, axis=1) != 0
    got = (O.ternarize(w, s) != t)[live].mean()
    phi = 0.5 * math.erfc((5.0 / 3.0) / math.sqrt(2.0))
    want = 0.4 * 2 * phi + 0.6 * phi
    assert abs(want - 0.0669) < 5e-4
    assert abs(got - want) < 2e-3, (got, want)


# ---------------------------------------------------------------- products
def _brute(t, s, x):
    """Exact sum_k s[n][k/128] t[n][k] x[b][k] with Fractions (fp16 values are exact rationals)."""
    n, k = t.shape
    y = np.zeros((x.shape[0], n), dtype=object)
    for b in range(x.shape[0]):
        for r in range(n):
            acc = Fraction(0)
            for kk in range(k):
                tv = int(t[r, kk])
                if tv:
                    acc += tv * Fraction(float(s[r, kk // 128])) * Fraction(float(x[b, kk]))
            y[b, r] = acc
    return y


@pytest.mark.parametrize("layout", O.LAYOUTS)
def test_gemv_integer_bruteforce(layout):
    rng = np.random.default_rng(1)
    for n, k, b in ((1, 128, 1), (7, 256, 3), (33, 384, 2), (5, 640, 9)):
        t = synth.codes_for(layout, n, k, seed=n * k)
        s = np.ones((n, k // 128), dtype=np.float16)
        x = rng.integers(-2, 3, size=(b, k)).astype(np.float16)
        y, a = O.gemv(O.pack(t, layout), s, x, layout, k)
        ex = _brute(t, s, x)
        assert np.array_equal(y, ex.astype(np.float64))
        assert np.array_equal(a, np.abs(x.astype(np.float64)) @ np.abs(t.astype(np.float64)).T)


@pytest.mark.parametrize("layout", O.LAYOUTS)
def test_gemv_exact_rational(layout):
    n, k, b = 6, 384, 2
    t = synth.codes_for(layout, n, k, seed=21)
    s = synth.group_scales(n, k // 128, seed=21)
    x = synth.activations(b, k, seed=21)
    y, a = O.gemv(O.pack(t, layout), s, x, layout, k)
    ex = _brute(t, s, x)
    for bi in range(b):
        for r in range(n):
            e = float(ex[bi, r])
            assert abs(y[bi, r] - e) <= 1e-12 * max(1.0, float(a[bi, r]))


def test_gemv_closed_forms():
    k = 512
    x = synth.activations(2, k, seed=2)
    xd = x.astype(np.float64)
    s = synth.group_scales(3, k // 128, seed=2)
    # all codes 0 -> y = 0 and A = 0
    t0 = np.zeros((3, k), dtype=np.int8)
    y, a = O.gemv(O.pack(t0, O.Q2_0_G128), s, x, O.Q2_0_G128, k)
    assert not y.any() and not a.any()
    # all codes +1 -> y = sum_g s_g * sum_{k in g} x_k
    t1 = np.ones((3, k), dtype=np.int8)
    y, _ = O.gemv(O.pack(t1, O.T3_5PB_G128), s, x, O.T3_5PB_G128, k)
    gs = xd.reshape(2, k // 128, 128).sum(axis=2)
    assert np.allclose(y, gs @ s.astype(np.float64).T, rtol=1e-12, atol=0)
    # one group: y = s * (sum_{t=+1} x - sum_{t=-1} x)
    t = synth.ternary_codes(1, 128, seed=9)
    sc = np.array([[0.03125]], dtype=np.float16)
    y, _ = O.gemv(O.pack(t, O.Q2_0_G128), sc, x[:, :128], O.Q2_0_G128, 128)
    want = 0.03125 * (xd[:, :128][:, t[0] == 1].sum(axis=1) - xd[:, :128][:, t[0] == -1].sum(axis=1))
    assert np.allclose(y[:, 0], want, rtol=1e-12, atol=1e-15)


def test_gemm_rows_select_tokens():
    k, n, m = 256, 9, 5
    t = synth.ternary_codes(n, k, seed=4)
    s = synth.group_scales(n, k // 128, seed=4)
    X = synth.activations(m, k, seed=4)
    p = O.pack(t, O.Q2_0_G128)
    Y, _ = O.gemm(p, s, X, O.Q2_0_G128, k)
    Y2, _ = O.gemm(p, s, X, O.Q2_0_G128, k, rows=[3, 0])
    assert np.array_equal(Y2, Y[[3, 0]])
    ex = _brute(t, s, X[[3]])
    assert abs(Y[3, 4] - float(ex[0, 4])) < 1e-12


def test_tolerance_formula():
    assert O.tolerance(0.0) == 1e-5
    assert abs(O.tolerance(100.0) - 0.20001) < 1e-12


# ---------------------------------------------------------------- planted mistakes must be caught
def _q2_pack_msb_first(t, layout):
    """Plausible mistake: first weight in the high bits of the byte."""
    n, k = t.shape
    c = (t.astype(np.int64) & 3).reshape(n, k // 4, 4)
    out = np.zeros((n, k // 4), dtype=np.uint8)
    for i in range(4):
        out |= (c[:, :, i] << (6 - 2 * i)).astype(np.uint8)
    return out


def _q2_pack_offset(t, layout):
    """Plausible mistake: offset-binary codes c = t + 1 instead of two's complement."""
    n, k = t.shape
    c = (t.astype(np.int64) + 1).reshape(n, k // 4, 4)
    return sum(c[:, :, i] << (2 * i) for i in range(4)).astype(np.uint8)


def _t3_pack_reversed_digits(t, layout):
    """Plausible mistake: digit 0 as the most significant trit."""
    n, k = t.shape
    c = np.ones((n, -(-k // 5) * 5), dtype=np.int64)
    c[:, :k] = t + 1
    c = c.reshape(n, -1, 5)
    return sum(c[:, :, i] * 3 ** (4 - i) for i in range(5)).astype(np.uint8)


def _ternarize_half_away(w, s):
    """Plausible mistake: round half away from zero (C round())."""
    q = w.astype(np.float64) / np.repeat(s.astype(np.float64), 128, axis=1)
    return (np.sign(q) * np.floor(np.abs(np.clip(q, -1, 1)) + 0.5)).astype(np.int8)


def _gemv_scale_dropped(codes, scales, x, layout, k):
    t = O.unpack(codes, layout, k)
    return x.astype(np.float64) @ t.astype(np.float64).T


def _gemv_scale_wrong_group(codes, scales, x, layout, k):
    t = O.unpack(codes, layout, k)
    s = np.asarray(scales, np.float64)[:, ::-1]  # groups reversed
    w = np.repeat(s, 128, axis=1) * t
    return x.astype(np.float64) @ w.T


def test_planted_mistakes_are_caught():
    cases = _golden_hand()
    q2 = [(t, b) for (l, t, b) in cases if l == O.Q2_0_G128]
    t3 = [(t, b) for (l, t, b) in cases if l == O.T3_5PB_G128]

    def hand_ok(packer, rows):
        for t, expect in rows:
            r = np.zeros((1, 128), dtype=np.int8)
            r[0, : len(t)] = t
            if list(packer(r, None)[0, : len(expect)]) != expect:
                return False
        return True

    assert hand_ok(lambda r, _: O.pack(r, O.Q2_0_G128), q2)
    assert not hand_ok(_q2_pack_msb_first, q2)
    assert not hand_ok(_q2_pack_offset, q2)
    assert hand_ok(lambda r, _: O.pack(r, O.T3_5PB_G128), t3)
    assert not hand_ok(_t3_pack_reversed_digits, t3)

    s = np.full((1, 1), 0.0234375, dtype=np.float16)
    w = np.zeros((1, 128), dtype=np.float16)
    w[0, 0] = np.float16(0.0234375 / 2)
    assert O.ternarize(w, s)[0, 0] == 0
    assert _ternarize_half_away(w, s)[0, 0] != 0

    n, k = 4, 384
    t = synth.ternary_codes(n, k, seed=8)
    sc = synth.group_scales(n, k // 128, seed=8)
    x = synth.activations(1, k, seed=8)
    ex = _brute(t, sc, x).astype(np.float64)
    p = O.pack(t, O.Q2_0_G128)
    assert np.allclose(O.gemv(p, sc, x, O.Q2_0_G128, k)[0], ex, rtol=1e-12, atol=0)
    assert not np.allclose(_gemv_scale_dropped(p, sc, x, O.Q2_0_G128, k), ex, rtol=1e-3)
    assert not np.allclose(_gemv_scale_wrong_group(p, sc, x, O.Q2_0_G128, k), ex, rtol=1e-3)


@pytest.mark.parametrize("layout", O.LAYOUTS)
def test_count_flips_pins(layout):
    k = 640
    t1 = synth.codes_for(layout, 40, k, seed=11)
    p1 = O.pack(t1, layout)
    assert O.count_flips(p1, p1, layout, k) == 0
    # any set of changed weights: the count is the number of changed t (unpack is an independent read)
    t2 = t1.copy()
    rng = np.random.default_rng(12)
    for _ in range(37):
        r, c = rng.integers(0, 40), rng.integers(0, k)
        t2[r, c] = -t2[r, c] if layout == O.Q1_0_G128 else (t2[r, c] + 2) % 3 - 1  # -1 -> 0 -> 1 -> -1
    p2 = O.pack(t2, layout)
    assert O.count_flips(p1, p2, layout, k) == int((O.unpack(p1, layout, k) != O.unpack(p2, layout, k)).sum())
    assert O.count_flips(p1, p2, layout, k) == int((t1 != t2).sum())
    assert O.count_flips(p1, p2, layout, k) == O.count_flips(p2, p1, layout, k)


def test_count_flips_ignores_base3_padding():
    k = 128  # 26 bytes of trits (128 = 25*5 + 3), byte 25 holds 2 padding trits
    t = synth.ternary_codes(3, k, seed=13)
    p = O.pack(t, O.T3_5PB_G128)
    q = p.copy()
    q[:, 25] = (q[:, 25] % 27) + 27 * 2  # change only the digits of the padding trits (k = 128, 129)
    assert O.count_flips(p, q, O.T3_5PB_G128, k) == 0
    q[:, 30] = 0  # a byte past the data
    assert O.count_flips(p, q, O.T3_5PB_G128, k) == 0


@pytest.mark.parametrize("layout", [O.Q2_0_G128, O.T3_5PB_G128])
def test_transposed_product_is_the_adjoint(layout):
    # <dx, x> = <dy, W x> for every x, dy: W^T is the adjoint of the forward product (checked with the
    # forward oracle), and integer inputs give exact integers
    n, k = 37, 640
    t = synth.ternary_codes(n, k, seed=21)
    codes = O.pack(t, layout)
    s = synth.group_scales(n, k // 128, seed=21)
    rng = np.random.default_rng(22)
    x = rng.integers(-3, 4, size=(1, k)).astype(np.float16)
    dy = rng.integers(-3, 4, size=(2, n)).astype(np.float16)
    dx, _ = O.gemv_t(codes, s, dy, layout, k)
    y, _ = O.gemv(codes, s, x, layout, k)
    for b in range(2):
        assert math.isclose(float(dx[b] @ x[0].astype(np.float64)), float(y[0] @ dy[b].astype(np.float64)),
                            rel_tol=1e-12, abs_tol=1e-9)
    ones = np.ones((n, k // 128), dtype=np.float16)
    dxi, _ = O.gemv_t(codes, ones, dy, layout, k)
    assert np.array_equal(dxi, dy.astype(np.int64) @ t.astype(np.int64))



# ---------------------------------------------------------------- binary layout (R12)
def test_q1_bits_per_weight_is_the_pages_figure():
    # [velog-27B] "ternary와 binary가 뭔가": binary with a group scale is 1.125 bits per weight
    for k in (128, 1024, 4096, 5120, 17408):
        assert O.bits_per_weight(O.Q1_0_G128, k) == 1.125


def test_q1_byte_table_exhaustive():
    # every byte value is valid and its 8 weights are its bits, LSB first, 1 -> +1, 0 -> -1
    codes = np.arange(256, dtype=np.uint8).reshape(256, 1).repeat(16, axis=1)
    t = O.unpack(codes, O.Q1_0_G128, 128)
    for v in range(256):
        want = [1 if (v >> i) & 1 else -1 for i in range(8)]
        assert t[v, :8].tolist() == want
    assert O.count_invalid(codes, O.Q1_0_G128, 256, 128) == 0
    assert np.array_equal(O.pack(t, O.Q1_0_G128), codes)


def test_q1_hand_packed():
    t = np.full((1, 128), -1, dtype=np.int8)
    t[0, [0, 3, 9, 127]] = 1
    p = O.pack(t, O.Q1_0_G128)
    assert p[0, 0] == 0b00001001 and p[0, 1] == 0b00000010 and p[0, 15] == 0x80 and p[0, 2:15].sum() == 0
    with pytest.raises(ValueError):
        O.pack(np.zeros((1, 128), dtype=np.int8), O.Q1_0_G128)  # 0 is not a binary code


def test_binarize_rule():
    s = np.array([[1.0], [-2.0], [0.0]], dtype=np.float16)
    w = np.array([[0.5, -0.5, 0.0, np.nan] + [1.0] * 124,
                  [0.5, -0.5, 0.0, np.nan] + [1.0] * 124,
                  [0.5, -0.5, 0.0, np.nan] + [1.0] * 124], dtype=np.float16)
    t = O.binarize(w, s)
    assert t[0, :4].tolist() == [1, -1, 1, 1]
    assert t[1, :4].tolist() == [-1, 1, 1, 1]
    assert t[2, :4].tolist() == [1, 1, 1, 1]
    # binarizing s * t reproduces t (lossless re-encode, [Metal-8B])
    tt = np.where(synth.ternary_codes(8, 256, seed=3) >= 0, 1, -1).astype(np.int8)
    sc = synth.group_scales(8, 2, seed=3)
    assert np.array_equal(O.binarize(O.dequantize(tt, sc).astype(np.float16), sc), tt)


def test_q1_gemv_integer_bruteforce():
    rng = np.random.default_rng(41)
    t = np.where(rng.random((9, 256)) < 0.5, -1, 1).astype(np.int8)
    x = rng.integers(-3, 4, size=(2, 256)).astype(np.float16)
    ones = np.ones((9, 2), dtype=np.float16)
    y, a = O.gemv(O.pack(t, O.Q1_0_G128), ones, x, O.Q1_0_G128, 256)
    want = np.array([[sum(int(t[r, c]) * int(x[b, c]) for c in range(256)) for r in range(9)] for b in range(2)])
    assert np.array_equal(y, want)
