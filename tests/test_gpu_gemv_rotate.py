"""y = W (R x) through tern_gemv_opt with rotate_signs, against the oracle and the two-call path.

R = H S / 32 on every 1024-element block of x ("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, section
"블록 단위 하다마드 회전": the weights live in the rotated basis and each layer multiplies by R x).
Where the int8-plane kernel runs it rotates x in its prologue with the transform and fp16 rounding of
tern_hadamard_rotate and keeps its work split, so the result must equal tern_hadamard_rotate followed
by tern_gemv bit for bit; elsewhere the call rotates x into the workspace and runs the same kernels,
so the same equality holds. Against the fp64 oracle W (R x): the product tolerance on
A = sum |w fp16(R x)| plus the rotation's own error bound (rotate_tolerance, twice: the GPU's fp32
transform and the oracle's fp16 rounding of the exact R x) carried through |w|."""
import numpy as np
import pytest

import oracle as O
from tests.gpu_cases import sample_rows, workload

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402


def _signs(seed):
    return np.where(np.random.default_rng(seed).random(1024) < 0.5, -1, 1).astype(np.int8)


def _check_against_oracle(y_gpu, codes, s, x, signs, layout, k, rows, what):
    xr = O.rotate(x.astype(np.float64), signs)           # exact R x; O.gemv rounds it to fp16
    y_ref, a = O.gemv(codes, s, xr, layout, k, rows=rows)
    absw = np.abs(O.dequantize(O.unpack(codes, layout, k, rows=rows), np.asarray(s)[rows]))
    extra = (2.0 * O.rotate_tolerance(x, xr)) @ absw.T    # [batch][rows]
    tol = O.tolerance(a) + extra
    err = np.abs(np.asarray(y_gpu, dtype=np.float64) - y_ref)
    assert np.isfinite(y_gpu).all(), what
    worst = float((err / tol).max())
    assert worst <= 1.0, f"{what}: |y - y_ref| / tol = {worst:.3g}"


# (layout, n, k, batch): one K slice at one and two CTAs per SM, K splits over a CTA pair, binary
# pairs, batches on the register / shared-memory / tcgen05 kernels, a base-3 K the int8-plane kernel
# does not take, a plan without room for the rotation, and a matrix narrower than one row tile
CASES = [(1, 4096, 4096, 1), (2, 24576, 4096, 1), (3, 24576, 4096, 1), (1, 4096, 4096, 2), (2, 4096, 4096, 2),
         (1, 34816, 5120, 1), (2, 4096, 12288, 1), (1, 5120, 17408, 1), (2, 5120, 17408, 1), (3, 4096, 4096, 3),
         (1, 4096, 4096, 3), (2, 4096, 4096, 4), (1, 4096, 4096, 17), (2, 300, 1024, 1), (2, 34816, 5120, 1),
         (1, 17, 1024, 1), (3, 33, 2048, 2)]


@pytest.mark.parametrize("layout,n,k,batch", CASES)
def test_rotated_gemv_equals_rotate_then_gemv_and_oracle(layout, n, k, batch):
    seed = n + k + 7 * batch + layout
    codes, s, x = workload(layout, n, k, batch, seed=seed)
    signs = _signs(seed)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    xg = torch.from_numpy(x).cuda()
    sg = torch.from_numpy(signs).cuda()
    y1 = T.gemv_opt(W, xg, rotate_signs=sg)
    y2 = T.gemv(W, T.hadamard_rotate(xg, sg))
    torch.cuda.synchronize()
    assert torch.equal(y1, y2), f"layout {layout} {n}x{k} b{batch}: fused rotation differs from the two calls"
    rows = sample_rows(n, 96, seed)
    _check_against_oracle(y1.cpu().numpy()[:, rows], codes, s, x, signs, layout, k, rows,
                          f"rotated layout {layout} {n}x{k} b{batch}")


def test_rotated_gemv_static_weights_and_repeat():
    # the launch-overlap flag and a chain of calls on one stream give the same bits as a plain call
    layout, n, k = 2, 24576, 4096
    codes, s, x = workload(layout, n, k, 1, seed=91)
    signs = _signs(91)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    xg, sg = torch.from_numpy(x).cuda(), torch.from_numpy(signs).cuda()
    ref = T.gemv_opt(W, xg, rotate_signs=sg)
    outs = [T.gemv_opt(W, xg, static_weights=True, rotate_signs=sg) for _ in range(4)]
    torch.cuda.synchronize()
    for y in outs:
        assert torch.equal(y, ref)


def test_rotation_changes_the_product():
    # the signs matter: flipping one sign changes R x and so the product (guards against a path that
    # ignores rotate_signs)
    layout, n, k = 1, 4096, 4096
    codes, s, x = workload(layout, n, k, 1, seed=5)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    xg = torch.from_numpy(x).cuda()
    s1 = _signs(5)
    s2 = s1.copy()
    s2[17] = -s2[17]
    y0 = T.gemv(W, xg)
    y1 = T.gemv_opt(W, xg, rotate_signs=torch.from_numpy(s1).cuda())
    y2 = T.gemv_opt(W, xg, rotate_signs=torch.from_numpy(s2).cuda())
    torch.cuda.synchronize()
    assert not torch.equal(y0, y1) and not torch.equal(y1, y2)
