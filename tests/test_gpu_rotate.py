"""GPU parity of tern_hadamard_rotate (through the C ABI) against the fp64 oracle.

Tolerance (derived from the arithmetic): the fp16 result is rounded once (2^-11 |y|) after ten fp32
butterfly stages (each adds at most 2^-24 of the running magnitude; bounded with a wide margin by
2^-18 (1/32) sum |x| over the block)."""
import numpy as np
import pytest

import oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402


def _signs(seed):
    return np.where(np.random.default_rng(seed).random(1024) < 0.5, -1, 1).astype(np.int8)


@pytest.mark.parametrize("batch,k", [(1, 1024), (1, 4096), (3, 5120), (8, 4096), (64, 17408), (2, 12288)])
def test_rotate_matches_oracle(batch, k):
    rng = np.random.default_rng(batch * 7 + k)
    x = rng.standard_normal((batch, k)).astype(np.float16)
    s = _signs(k)
    y = T.hadamard_rotate(torch.from_numpy(x).cuda(), torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    ref = O.rotate(x.astype(np.float64), s)
    tol = O.rotate_tolerance(x, ref)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{bad.sum()} outputs out of tolerance, worst {np.max(np.abs(got - ref) - tol)}"


def test_rotate_in_place_and_signs_semantics():
    k = 2048
    x = np.random.default_rng(1).standard_normal((2, k)).astype(np.float16)
    s = _signs(2).astype(np.int16) * np.random.default_rng(3).integers(1, 100, 1024)
    s = np.clip(s, -128, 127).astype(np.int8)   # any negative entry is -1, any other +1
    xg = torch.from_numpy(x).cuda()
    T.hadamard_rotate(xg, torch.from_numpy(s).cuda(), y=xg)
    torch.cuda.synchronize()
    ref = O.rotate(x.astype(np.float64), s)
    assert not (np.abs(xg.cpu().numpy().astype(np.float64) - ref) > O.rotate_tolerance(x, ref)).any()


def test_rotate_basis_vectors_exact():
    # R e_j = s_j H[:, j] / 32 is exactly representable in fp16: the kernel must return it bit-exactly
    k = 1024
    s = _signs(5)
    js = [0, 1, 31, 32, 127, 128, 511, 1023]
    x = np.zeros((len(js), k), dtype=np.float16)
    for r, j in enumerate(js):
        x[r, j] = 1.0
    y = T.hadamard_rotate(torch.from_numpy(x).cuda(), torch.from_numpy(s).cuda()).cpu().numpy()
    assert np.array_equal(y.astype(np.float64), O.rotate(x.astype(np.float64), s))


def test_rotate_then_gemv_equals_gemv_on_rotated_x():
    # f(x) = W (R x): the rotation composes with the ternary product
    from tests.gpu_cases import workload, check_product
    n, k = 512, 4096
    codes, sc, x = workload(T.Q2_0_G128, n, k, 1, seed=21)
    s = _signs(21)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(sc).cuda(), T.Q2_0_G128, k)
    xr = T.hadamard_rotate(torch.from_numpy(x).cuda(), torch.from_numpy(s).cuda())
    y = T.gemv(W, xr).cpu().numpy()
    xr_host = xr.cpu().numpy()
    y_ref, a = O.gemv(codes, sc, xr_host, T.Q2_0_G128, k)
    check_product(y, y_ref, a, "gemv of rotated x")
