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
@pytest.mark.parametrize("n,k,batch", [(4096, 4096, 1), (5120, 17408, 4), (1000, 2176, 3), (4096, 12288, 8),
                                       (24576, 4096, 1), (300, 640, 2)])
def test_noalloc_matches_gemv_twice(layout, n, k, batch):
    codes, s, x = workload(layout, n, k, batch, seed=n + k + batch)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    xg = torch.from_numpy(x).cuda()
    y_ref, a = O.gemv(codes, s, x, layout, k)  # the fp64 oracle and sum_k |w_k x_k| of every output
    ref = T.gemv(W, xg)
    for _ in range(2):  # two calls in a row: the shared scratch must be reusable
        y = torch.full((batch, n), float("nan"), dtype=torch.float16, device="cuda")
        assert _noalloc(W, xg, y) == 0
        torch.cuda.synchronize()
        check_product(y.cpu().numpy().astype(np.float64), y_ref, a, f"noalloc layout {layout} {n}x{k} b{batch}")
        assert torch.equal(y, ref)  # and the same bits as the workspace entry point


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
    # a shape whose plan uses split-K scratch, so the binding reaches the static array
    n, k, batch = 5120, 17408, 4
    t = synth.ternary_codes(n, k, seed=3)
    s = synth.group_scales(n, k // 128, seed=3)
    x = synth.activations(batch, k, seed=3)
    W = T.from_packed(torch.from_numpy(pack_rows(t, T.Q2_0_G128)).cuda(), torch.from_numpy(s).cuda(), T.Q2_0_G128, k)
    assert T.gemv_workspace_bytes(W, batch) > 0
    xg = torch.from_numpy(x).cuda()
    y1 = T.gemv_noalloc(W, xg)
    y2 = T.gemv(W, xg)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)  # same kernel and plan: identical bits
    rows = np.arange(0, n, 7)
    y_ref, a = O.gemv(pack_rows(t, T.Q2_0_G128), s, x, T.Q2_0_G128, k, rows=rows)
    check_product(y1.cpu().numpy()[:, rows], y_ref, a, "noalloc binding")
