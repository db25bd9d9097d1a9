"""GPU parity of tern_pack / tern_unpack (through the C ABI) against the oracle: bit-exact bytes,
codes and fp16 values, including ties, special values and the invalid-code count."""
import numpy as np
import pytest

import oracle as O
from gemm_tern_gemv_b200 import synth
from tests.gpu_cases import pack_rows, ternarize_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402

LAYOUTS = [T.Q2_0_G128, T.T3_5PB_G128]


def _gpu_pack(w, s, layout):
    W = T.pack(torch.from_numpy(w).cuda(), torch.from_numpy(s).cuda(), layout)
    torch.cuda.synchronize()
    return W, W.codes.cpu().numpy()


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("n,k", [(1, 128), (3, 256), (17, 384), (64, 640), (100, 1152), (7, 4096), (5, 17408)])
def test_pack_matches_oracle(layout, n, k):
    t = synth.ternary_codes(n, k, seed=n + k)
    s = synth.group_scales(n, k // 128, seed=n + k)
    w = synth.latents(t, s, seed=n + k)
    _, got = _gpu_pack(w, s, layout)
    want = O.pack(O.ternarize(w, s), layout)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("layout", LAYOUTS)
def test_pack_ties_and_specials(layout):
    n, k = 8, 256
    rng = np.random.default_rng(3)
    s = synth.group_scales(n, k // 128, seed=3)
    s[0, 0] = 0.0
    s[1, 0] = np.float16(np.nan)
    s[2, 0] = -s[2, 0]
    s[3, 0] = np.float16(np.inf)
    s[4, 0] = np.float16(6e-8)  # fp16 subnormal scale
    w = (np.repeat(s.astype(np.float64), 128, axis=1) * rng.choice([-1, -0.5, 0, 0.5, 1, 0.75, -0.25], size=(n, k))).astype(np.float16)
    # exact ties w = +-s/2 in every row; one ulp above and below
    half = (s[:, 1].astype(np.float64) / 2).astype(np.float16)
    w[:, 128] = half
    w[:, 129] = -half
    w[:, 130] = np.nextafter(half, np.float16(np.inf))
    w[:, 131] = np.nextafter(half, np.float16(0))
    w[5, 5] = np.float16(np.nan)
    w[6, 6] = np.float16(np.inf)
    w[6, 7] = np.float16(-np.inf)
    w[7, 8] = np.float16(-0.0)
    _, got = _gpu_pack(w, s, layout)
    want = O.pack(O.ternarize(w, s), layout)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("mi,n,k", [(0, 4096, 4096), (1, 24576, 4096), (2, 4096, 12288)])
def test_pack_8b_shapes(layout, mi, n, k):
    seed = synth.seed_for(5, mi) + 10 * layout
    t = synth.ternary_codes(n, k, seed)
    s = synth.group_scales(n, k // 128, seed)
    w = synth.latents(t, s, seed)
    _, got = _gpu_pack(w, s, layout)
    want = pack_rows(ternarize_rows(w, s), layout)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("n,k", [(5, 128), (33, 1152), (300, 4096)])
def test_unpack_matches_oracle(layout, n, k):
    t = synth.ternary_codes(n, k, seed=k)
    s = synth.group_scales(n, k // 128, seed=k)
    codes = O.pack(t, layout)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    w, tt, bad = T.unpack(W)
    torch.cuda.synchronize()
    assert np.array_equal(tt.cpu().numpy(), t)
    assert int(bad.item()) == 0
    want = O.dequantize(t, s).astype(np.float16)
    assert np.array_equal(w.cpu().numpy().view(np.uint16), want.view(np.uint16))
    # round trip on the GPU: pack(unpack(P)) == P
    W2 = T.pack(w, W.scales, layout)
    torch.cuda.synchronize()
    assert np.array_equal(W2.codes.cpu().numpy(), codes)


@pytest.mark.parametrize("layout", LAYOUTS)
def test_unpack_counts_invalid_codes(layout):
    n, k = 4, 256
    t = synth.ternary_codes(n, k, seed=1)
    codes = O.pack(t, layout)
    if layout == T.Q2_0_G128:
        codes[0, 0] = 0xAA   # four fields == 0b10
        codes[2, 10] = 0x02  # field 0 == 0b10; fields 1..3 are 0 (valid)
    else:
        codes[0, 0] = 243
        codes[3, 7] = 255
    s = synth.group_scales(n, k // 128, seed=1)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    w, tt, bad = T.unpack(W)
    torch.cuda.synchronize()
    assert int(bad.item()) == O.count_invalid(codes, layout, n, k)
    ref = O.unpack(codes, layout, k, check=False)
    inv = np.zeros_like(ref, dtype=bool)
    kk = np.arange(k)
    if layout == T.Q2_0_G128:
        inv = ((codes[:, kk // 4].astype(int) >> (2 * (kk % 4))) & 3) == 2
    else:
        inv = codes[:, kk // 5] > 242
    ref[inv] = 0
    assert np.array_equal(tt.cpu().numpy(), ref)


@pytest.mark.parametrize("layout", [T.Q2_0_G128, T.T3_5PB_G128])
@pytest.mark.parametrize("n,k", [(257, 640), (4096, 4096)])
def test_pack_flips_match_oracle(layout, n, k):
    # QAT step: re-pack perturbed latents against the previous packing and count the changed codes
    t = synth.ternary_codes(n, k, seed=n + k)
    s = synth.group_scales(n, k // 128, seed=n + k)
    w1 = synth.latents(t, s, seed=1)
    w2 = (w1.astype(np.float32) + np.random.default_rng(2).standard_normal(w1.shape).astype(np.float32)
          * 0.2 * np.repeat(s.astype(np.float32), 128, axis=1)).astype(np.float16)
    sg = torch.from_numpy(s).cuda()
    W1 = T.pack(torch.from_numpy(w1).cuda(), sg, layout)
    W2, flips = T.pack_flips(torch.from_numpy(w2).cuda(), sg, W1)
    torch.cuda.synchronize()
    c1, c2 = W1.codes.cpu().numpy(), W2.codes.cpu().numpy()
    assert np.array_equal(c2, O.pack(O.ternarize(w2, s), layout))  # the pack itself is unchanged
    want = O.count_flips(c1, c2, layout, k)
    assert int(flips.item()) == want
    assert want == int((O.ternarize(w1, s) != O.ternarize(w2, s)).sum())
    # the counter accumulates
    T.pack_flips(torch.from_numpy(w2).cuda(), sg, W1, flips=flips)
    torch.cuda.synchronize()
    assert int(flips.item()) == 2 * want
