"""GPU parity of the binary Q1_0_g128 layout (t in {-1, +1}, bit k % 8 of byte k / 8, 1 = +1) through
the C ABI against the fp64 oracle: pack / unpack / flip count bit-exact, and the three products
(register-decode GEMV in pairs of batch rows, tcgen05 GEMM, transposed product) within the product
tolerance |y - y_ref| <= 2e-3 * sum |w x| + 1e-5, exact on integer inputs."""
import numpy as np
import pytest

import oracle as O
from gemm_tern_gemv_b200 import synth
from tests.gpu_cases import check_product, pack_rows, sample_rows, workload

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402

Q1 = T.Q1_0_G128


def _matrix(codes, s, k):
    return T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), Q1, k)


# ------------------------------------------------------------------------------ pack / unpack
@pytest.mark.parametrize("n,k", [(1, 128), (3, 256), (17, 384), (64, 640), (100, 1152), (7, 4096), (5, 17408)])
def test_pack_matches_oracle(n, k):
    t = synth.ternary_codes(n, k, seed=n + k)  # latents around a ternary matrix: zeros included
    s = synth.group_scales(n, k // 128, seed=n + k)
    w = synth.latents(t, s, seed=n + k)
    W = T.pack(torch.from_numpy(w).cuda(), torch.from_numpy(s).cuda(), Q1)
    torch.cuda.synchronize()
    assert np.array_equal(W.codes.cpu().numpy(), O.pack(O.binarize(w, s), Q1))


def test_pack_signs_and_specials():
    n, k = 8, 256
    rng = np.random.default_rng(4)
    s = synth.group_scales(n, k // 128, seed=4)
    s[0, 0] = 0.0
    s[1, 0] = np.float16(np.nan)
    s[2, 0] = -s[2, 0]
    s[3, 0] = np.float16(np.inf)
    s[4, 1] = np.float16(-np.inf)
    w = rng.standard_normal((n, k)).astype(np.float16)
    w[:, 3] = 0.0
    w[:, 4] = np.float16(-0.0)
    w[5, 5] = np.float16(np.nan)
    w[6, 6] = np.float16(np.inf)
    w[6, 7] = np.float16(-np.inf)
    w[7, 8] = np.float16(-6e-8)  # negative subnormal
    W = T.pack(torch.from_numpy(w).cuda(), torch.from_numpy(s).cuda(), Q1)
    torch.cuda.synchronize()
    assert np.array_equal(W.codes.cpu().numpy(), O.pack(O.binarize(w, s), Q1))


@pytest.mark.parametrize("n,k", [(5, 128), (33, 1152), (300, 4096)])
def test_unpack_round_trip(n, k):
    t = synth.binary_codes(n, k, seed=k)
    s = synth.group_scales(n, k // 128, seed=k)
    codes = O.pack(t, Q1)
    W = _matrix(codes, s, k)
    w, tt, bad = T.unpack(W)
    torch.cuda.synchronize()
    assert np.array_equal(tt.cpu().numpy(), t)
    assert int(bad.item()) == 0  # every bit pattern is valid
    assert np.array_equal(w.cpu().numpy().view(np.uint16), O.dequantize(t, s).astype(np.float16).view(np.uint16))
    W2 = T.pack(w, W.scales, Q1)
    torch.cuda.synchronize()
    assert np.array_equal(W2.codes.cpu().numpy(), codes)


def test_every_byte_unpacks():
    n, k = 256, 128
    codes = np.zeros((n, O.row_bytes(Q1, k)), dtype=np.uint8)
    codes[:, :] = np.arange(256, dtype=np.uint8)[:, None]  # row v: every byte = v
    s = np.ones((n, 1), dtype=np.float16)
    _, tt, bad = T.unpack(_matrix(codes, s, k))
    torch.cuda.synchronize()
    assert int(bad.item()) == 0
    assert np.array_equal(tt.cpu().numpy(), O.unpack(codes, Q1, k))


@pytest.mark.parametrize("n,k", [(257, 640), (4096, 4096)])
def test_pack_flips_match_oracle(n, k):
    t = synth.binary_codes(n, k, seed=n + k)
    s = synth.group_scales(n, k // 128, seed=n + k)
    w1 = synth.latents(t, s, seed=1)
    w2 = (w1.astype(np.float32) + np.random.default_rng(2).standard_normal(w1.shape).astype(np.float32)
          * 0.5 * np.repeat(s.astype(np.float32), 128, axis=1)).astype(np.float16)
    sg = torch.from_numpy(s).cuda()
    W1 = T.pack(torch.from_numpy(w1).cuda(), sg, Q1)
    W2, flips = T.pack_flips(torch.from_numpy(w2).cuda(), sg, W1)
    torch.cuda.synchronize()
    c1, c2 = W1.codes.cpu().numpy(), W2.codes.cpu().numpy()
    assert np.array_equal(c2, O.pack(O.binarize(w2, s), Q1))
    want = O.count_flips(c1, c2, Q1, k)
    assert want == int((O.binarize(w1, s) != O.binarize(w2, s)).sum()) > 0
    assert int(flips.item()) == want


# ------------------------------------------------------------------------------ GEMV
def _gemv(codes, s, x, k, workspace=None):
    W = _matrix(codes, s, k)
    y = T.gemv(W, torch.from_numpy(x).cuda(), workspace=workspace)
    torch.cuda.synchronize()
    return W, y.cpu().numpy()


@pytest.mark.parametrize("n,k", [(1, 128), (17, 256), (130, 384), (200, 640), (257, 1152), (1000, 2176),
                                 (64, 5120), (33, 17408)])
@pytest.mark.parametrize("batch", [1, 2, 3, 5, 8, 16, 17, 33, 64])
def test_gemv_small_shapes_full_oracle(n, k, batch):
    codes, s, x = workload(Q1, n, k, batch, seed=n * 7 + k + batch)
    _, y = _gemv(codes, s, x, k)
    y_ref, a = O.gemv(codes, s, x, Q1, k)
    check_product(y, y_ref, a, f"binary n {n} k {k} b {batch}")


@pytest.mark.parametrize("batch", [1, 2, 3, 64])
def test_gemv_integer_inputs_are_exact(batch):
    n, k = 96, 1152
    t = synth.binary_codes(n, k, seed=6)
    s = np.ones((n, k // 128), dtype=np.float16)
    x = np.random.default_rng(6).integers(-2, 3, size=(batch, k)).astype(np.float16)
    _, y = _gemv(pack_rows(t, Q1), s, x, k)
    exact = x.astype(np.int64) @ t.astype(np.int64).T
    assert np.abs(exact).max() <= 2048
    assert np.array_equal(y.astype(np.float64), exact.astype(np.float64))


def test_gemv_closed_forms():
    # all -1 (every byte 0x00: the pattern a zero-filled read would give) and all +1
    n, k, batch = 80, 1024, 3
    s = synth.group_scales(n, k // 128, seed=2)
    x = synth.activations(batch, k, seed=2)
    gs = x.astype(np.float64).reshape(batch, k // 128, 128).sum(axis=2)
    a = np.abs(x.astype(np.float64)) @ np.repeat(s.astype(np.float64), 128, axis=1).T
    for sign in (-1, 1):
        codes = pack_rows(np.full((n, k), sign, np.int8), Q1)
        _, y = _gemv(codes, s, x, k)
        check_product(y, sign * (gs @ s.astype(np.float64).T), a, f"all {sign:+d}")


@pytest.mark.parametrize("k,needs_ws", [(17408, False), (17280, True)])
def test_gemv_split_k_deterministic_and_workspace_reuse(k, needs_ws):
    # n % 8 != 0 keeps batch 5 off the GEMM: three launches of a two-row kernel, one after another.
    # K = 17408 runs them on the int8-plane kernel (K split over a cluster, no workspace); K = 17280
    # (not a multiple of 256) on the register kernel, whose three launches share one workspace.
    n, batch = 1001, 5
    codes, s, x = workload(Q1, n, k, batch, seed=12)
    W = _matrix(codes, s, k)
    ws = T.gemv_workspace(W, batch)
    assert (ws is not None) == needs_ws
    xg = torch.from_numpy(x).cuda()
    y1 = T.gemv(W, xg, workspace=ws).clone()
    y2 = T.gemv(W, xg, workspace=ws).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    rows = sample_rows(n, 256, 2)
    y_ref, a = O.gemv(codes, s, x, Q1, k, rows=rows)
    check_product(y1.cpu().numpy()[:, rows], y_ref, a, "binary split-K")


@pytest.mark.parametrize("mi,n,k", [(0, 4096, 4096), (1, 24576, 4096), (2, 4096, 12288)])
@pytest.mark.parametrize("batch", [1, 4])
def test_gemv_8b_layer_set_sampled(mi, n, k, batch):
    seed = synth.seed_for(2, mi) + 30 + batch
    codes, s, x = workload(Q1, n, k, batch, seed)
    _, y = _gemv(codes, s, x, k)
    r = sample_rows(n, 512, seed)
    y_ref, a = O.gemv(codes, s, x, Q1, k, rows=r)
    check_product(y[:, r], y_ref, a, f"binary {n}x{k} b{batch}")


# ------------------------------------------------------------------------------ GEMM
def _gemm(codes, s, X, k):
    W = _matrix(codes, s, k)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = T.gemm(W, torch.from_numpy(X).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return W, Y.cpu().numpy()


@pytest.mark.parametrize("m,n,k", [(1, 8, 128), (7, 128, 256), (200, 136, 640), (256, 256, 1024), (300, 392, 384),
                                   (513, 128, 2176), (64, 1000, 5120), (33, 24, 17408)])
def test_gemm_small_shapes_full_oracle(m, n, k):
    codes, s, X = workload(Q1, n, k, m, seed=m + n + k + 3)
    _, Y = _gemm(codes, s, X, k)
    Y_ref, A = O.gemm(codes, s, X, Q1, k)
    check_product(Y, Y_ref, A, f"binary gemm {m}x{n}x{k}")


def test_gemm_integer_inputs_are_exact():
    m, n, k = 260, 136, 640  # odd and even 64-weight blocks: both halves of the 16-byte box
    t = synth.binary_codes(n, k, seed=7)
    s = np.ones((n, k // 128), dtype=np.float16)
    X = np.random.default_rng(7).integers(-2, 3, size=(m, k)).astype(np.float16)
    _, Y = _gemm(pack_rows(t, Q1), s, X, k)
    exact = X.astype(np.int64) @ t.astype(np.int64).T
    assert np.array_equal(Y.astype(np.float64), exact.astype(np.float64))


def test_gemm_prefill_shape_sampled():
    m, n, k = 512, 4096, 4096
    codes, s, X = workload(Q1, n, k, m, seed=14)
    _, Y = _gemm(codes, s, X, k)
    rows = sample_rows(m, 64, 14)  # token rows of Y
    Y_ref, A = O.gemm(codes, s, X, Q1, k, rows=rows)
    check_product(Y[rows], Y_ref, A, "binary prefill 512x4096x4096")


# ------------------------------------------------------------------------------ transposed product
@pytest.mark.parametrize("n,k", [(1, 128), (37, 640), (300, 1152), (4096, 4096), (1000, 17408)])
@pytest.mark.parametrize("batch", [1, 3, 8])
def test_gemv_t_matches_oracle(n, k, batch):
    seed = n + k + batch + 5
    codes, s, _ = workload(Q1, n, k, 1, seed)
    dy = synth.activations(batch, n, seed + 1)
    W = _matrix(codes, s, k)
    dx = T.gemv_t(W, torch.from_numpy(dy).cuda()).cpu().numpy().astype(np.float64)
    ref, a = O.gemv_t(codes, s, dy, Q1, k)
    check_product(dx, ref, a, f"binary gemv_t {n}x{k} b{batch}")


def test_gemv_t_integer_exact_and_deterministic():
    n, k = 2049, 1280
    t = synth.binary_codes(n, k, seed=8)
    s = np.ones((n, k // 128), dtype=np.float16)
    dy = np.random.default_rng(8).integers(-1, 2, size=(4, n)).astype(np.float16)
    W = _matrix(pack_rows(t, Q1), s, k)
    dyg = torch.from_numpy(dy).cuda()
    a = T.gemv_t(W, dyg)
    b = T.gemv_t(W, dyg)
    torch.cuda.synchronize()
    exact = dy.astype(np.int64) @ t.astype(np.int64)
    assert np.abs(exact).max() <= 2048
    assert np.array_equal(a.cpu().numpy().astype(np.float64), exact.astype(np.float64))
    assert torch.equal(a, b)
