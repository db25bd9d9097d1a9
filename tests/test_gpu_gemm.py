"""GPU parity of tern_gemm (tcgen05 prefill GEMM, through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest

import oracle as O
from gemm_tern_gemv_b200 import synth
from tests.gpu_cases import check_product, pack_rows, sample_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402


LAYOUTS = [T.Q2_0_G128, T.T3_5PB_G128]


def _run(codes, s, X, k, layout=T.Q2_0_G128):
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = T.gemm(W, torch.from_numpy(X).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return W, Y.cpu().numpy()


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("m,n,k", [(1, 8, 128), (7, 128, 256), (200, 136, 640), (256, 256, 1024), (300, 392, 384),
                                   (513, 128, 2176), (64, 1000, 5120), (33, 24, 17408)])
def test_small_shapes_full_oracle(layout, m, n, k):
    seed = m + n + k + layout
    t = synth.ternary_codes(n, k, seed)
    s = synth.group_scales(n, k // 128, seed)
    X = synth.activations(m, k, seed)
    codes = pack_rows(t, layout)
    _, Y = _run(codes, s, X, k, layout)
    Y_ref, A = O.gemm(codes, s, X, layout, k)
    check_product(Y, Y_ref, A, f"gemm layout {layout} {m}x{n}x{k}")


@pytest.mark.parametrize("layout", LAYOUTS)
def test_integer_inputs_are_exact(layout):
    m, n, k = 260, 136, 640  # base-3: 64-weight blocks start at every digit 0..4 of a byte
    t = synth.ternary_codes(n, k, seed=3)
    s = np.ones((n, k // 128), dtype=np.float16)
    X = np.random.default_rng(3).integers(-2, 3, size=(m, k)).astype(np.float16)
    _, Y = _run(pack_rows(t, layout), s, X, k, layout)
    exact = X.astype(np.int64) @ t.astype(np.int64).T
    assert np.array_equal(Y.astype(np.float64), exact.astype(np.float64))


@pytest.mark.parametrize("layout", LAYOUTS)
def test_gemm_m1_matches_gemv(layout):
    n, k = 1024, 4096
    t = synth.ternary_codes(n, k, seed=4)
    s = synth.group_scales(n, k // 128, seed=4)
    x = synth.activations(1, k, seed=4)
    codes = pack_rows(t, layout)
    W, Y = _run(codes, s, x, k, layout)
    y = T.gemv(W, torch.from_numpy(x).cuda()).cpu().numpy()
    y_ref, a = O.gemv(codes, s, x, layout, k)
    check_product(Y, y_ref, a, "gemm m=1")
    check_product(y, y_ref, a, "gemv")


def test_base3_gemm_exhaustive_bytes():
    # every valid base-3 byte value at every position of a row: t is a function of the byte alone, so
    # with x = e_j the product returns column j of s * t exactly
    k = 1280  # 256 bytes per row
    n = 16
    codes = np.zeros((n, O.row_bytes(T.T3_5PB_G128, k)), dtype=np.uint8)
    for r in range(n):
        codes[r, :256] = (np.arange(256) * 7 + 13 * r) % 243
    s = np.ones((n, k // 128), dtype=np.float16)
    X = np.eye(k, dtype=np.float16)[:300]  # tokens m = unit vectors e_0 .. e_299
    _, Y = _run(codes, s, X, k, T.T3_5PB_G128)
    t = O.unpack(codes, T.T3_5PB_G128, k).astype(np.float64)  # [n][k]
    assert np.array_equal(Y.astype(np.float64), t[:, :300].T)


def test_config5_prefill_gemm():
    # M = 2048 tokens, K = 5120, N = 17408: sampled token rows checked against the oracle
    m, k, n = 2048, 5120, 17408
    seed = synth.seed_for(5, 9)
    t = synth.ternary_codes(n, k, seed)
    s = synth.group_scales(n, k // 128, seed)
    X = synth.activations(m, k, seed)
    codes = pack_rows(t, T.Q2_0_G128)
    del t
    _, Y = _run(codes, s, X, k)
    rows = sample_rows(m, 48, seed)
    Y_ref, A = O.gemm(codes, s, X, T.Q2_0_G128, k, rows=rows)
    check_product(Y[rows], Y_ref, A, "config 5 GEMM")
    # repeated launches give the same bits (no data-dependent scheduling)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), T.Q2_0_G128, k)
    Xg = torch.from_numpy(X).cuda()
    Y2 = T.gemm(W, Xg)
    torch.cuda.synchronize()
    assert np.array_equal(Y2.cpu().numpy().view(np.uint16), Y.view(np.uint16))


def test_config5_prefill_gemm_base3():
    # the prefill shape in the dense base-3 layout, sampled token rows
    m, k, n = 2048, 5120, 17408
    seed = synth.seed_for(5, 10)
    t = synth.ternary_codes(n, k, seed)
    s = synth.group_scales(n, k // 128, seed)
    X = synth.activations(m, k, seed)
    codes = pack_rows(t, T.T3_5PB_G128)
    del t
    _, Y = _run(codes, s, X, k, T.T3_5PB_G128)
    rows = sample_rows(m, 32, seed)
    Y_ref, A = O.gemm(codes, s, X, T.T3_5PB_G128, k, rows=rows)
    check_product(Y[rows], Y_ref, A, "config 5 GEMM base-3")
