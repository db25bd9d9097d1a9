"""tern_gemv_noalloc (through the C ABI) matches tern_gemv on two calls in a row.

The allocation-free entry point serves callers that cannot give the library device memory (a host
runtime that owns every allocation, or a loop where cudaMalloc / cudaFree are not allowed); it keeps
its split-K scratch in a static device array of the library instead of a caller workspace. This
file is collected last so that a run stopping at the first failure has run every other test; it
also passes alone in a fresh process (the first call sets up the array's address).
"""
import ctypes

import numpy as np
import pytest

import oracle as O
from gemm_tern_gemv_b200 import synth
from tests.gpu_cases import check_product, pack_rows, workload

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402


def _noalloc(W, x, y):
    c = W.c()
    return T.lib().tern_gemv_noalloc(ctypes.byref(c), ctypes.c_void_p(x.data_ptr()), x.shape[0],
                                     ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("layout", [T.Q2_0_G128, T.T3_5PB_G128, T.Q1_0_G128])
@pytest.mark.parametrize("n,k,batch", [(4096, 4096, 1), (5120, 17408, 1), (1000, 2176, 3), (4096, 12288, 8),
                                       (24576, 4096, 1), (300, 640, 2)])
def test_noalloc_matches_gemv_twice(layout, n, k, batch):
    codes, s, x = workload(layout, n, k, batch, seed=n + k + batch)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    xg = torch.from_numpy(x).cuda()
    ref = T.gemv(W, xg).cpu().numpy().astype(np.float64)
    _, a = O.gemv(codes, s, x, layout, k)  # sum_k |w_k x_k| of every output: the tolerance scale
    for _ in range(2):  # two calls in a row: the shared scratch must be reusable
        y = torch.full((batch, n), float("nan"), dtype=torch.float16, device="cuda")
        assert _noalloc(W, xg, y) == 0
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64)
        check_product(got, ref, a, f"noalloc layout {layout} {n}x{k} b{batch}")


def test_noalloc_rejects_oversized_scratch():
    # a split-K plan that needs more than the static array is refused before any launch
    n, k, batch = 65536, 17408, 13
    W = T.empty_matrix(T.T3_5PB_G128, n, k)
    need = T.gemv_workspace_bytes(W, batch)
    assert need > 8 * 1024 * 1024
    x = torch.zeros((batch, k), dtype=torch.float16, device="cuda")
    y = torch.zeros((batch, n), dtype=torch.float16, device="cuda")
    assert _noalloc(W, x, y) == 4  # TERN_ERR_WORKSPACE


def test_noalloc_binding_roundtrip():
    n, k = 2048, 4096
    t = synth.ternary_codes(n, k, seed=3)
    s = synth.group_scales(n, k // 128, seed=3)
    x = synth.activations(1, k, seed=3)
    W = T.from_packed(torch.from_numpy(pack_rows(t, T.Q2_0_G128)).cuda(), torch.from_numpy(s).cuda(), T.Q2_0_G128, k)
    xg = torch.from_numpy(x).cuda()
    y1 = T.gemv_noalloc(W, xg)
    y2 = T.gemv(W, xg)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)  # same kernel and plan: identical bits
