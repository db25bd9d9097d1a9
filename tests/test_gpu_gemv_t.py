"""GPU parity of tern_gemv_t (transposed product, through the C ABI) against the fp64 oracle.

Tolerance: the product tolerance |dx - dx_ref| <= 2e-3 * sum_n |w_nk dy_bn| + 1e-5 (fp32 sums, one
fp16 rounding of dx)."""
import numpy as np
import pytest

import oracle as O
from gemm_tern_gemv_b200 import synth
from tests.gpu_cases import check_product, pack_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402

LAYOUTS = [T.Q2_0_G128, T.T3_5PB_G128]


def _case(layout, n, k, batch, seed):
    t = synth.ternary_codes(n, k, seed)
    s = synth.group_scales(n, k // 128, seed)
    dy = synth.activations(batch, n, seed + 1)
    codes = pack_rows(t, layout)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    return W, codes, s, dy


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("n,k", [(1, 128), (37, 640), (300, 1152), (4096, 4096), (1000, 17408)])
@pytest.mark.parametrize("batch", [1, 2, 3, 8])
def test_gemv_t_matches_oracle(layout, n, k, batch):
    W, codes, s, dy = _case(layout, n, k, batch, seed=n + k + batch)
    dx = T.gemv_t(W, torch.from_numpy(dy).cuda()).cpu().numpy().astype(np.float64)
    ref, a = O.gemv_t(codes, s, dy, layout, k)
    check_product(dx, ref, a, f"gemv_t layout {layout} {n}x{k} b{batch}")


@pytest.mark.parametrize("layout", LAYOUTS)
def test_gemv_t_integer_exact_and_deterministic(layout):
    n, k = 2049, 1280
    t = synth.ternary_codes(n, k, seed=5)
    codes = pack_rows(t, layout)
    s = np.ones((n, k // 128), dtype=np.float16)
    dy = np.random.default_rng(5).integers(-2, 3, size=(4, n)).astype(np.float16)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    dyg = torch.from_numpy(dy).cuda()
    a = T.gemv_t(W, dyg)
    b = T.gemv_t(W, dyg)
    torch.cuda.synchronize()
    exact = dy.astype(np.int64) @ t.astype(np.int64)
    assert np.array_equal(a.cpu().numpy().astype(np.float64), exact.astype(np.float64))
    assert torch.equal(a, b)


@pytest.mark.parametrize("layout", LAYOUTS)
def test_gemv_t_8b_shape_sampled(layout):
    n, k = 24576, 4096
    W, codes, s, dy = _case(layout, n, k, 1, seed=31)
    dx = T.gemv_t(W, torch.from_numpy(dy).cuda()).cpu().numpy().astype(np.float64)
    cols = np.random.default_rng(31).choice(k, 256, replace=False)
    ref, a = O.gemv_t(codes, s, dy, layout, k, cols=cols)
    check_product(dx[:, cols], ref, a, "gemv_t 24576x4096 sampled columns")
