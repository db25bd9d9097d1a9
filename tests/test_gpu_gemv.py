"""GPU parity of tern_gemv (through the C ABI) against the fp64 oracle.

Tolerance: |y - y_ref| <= 2e-3 * sum_k |w_k x_k| + 1e-5 per output (the spec's bound; the fp16
rounding of y adds at most 2^-11 |y| <= 4.9e-4 * A of it). Integer cases must be exact."""
import numpy as np
import pytest

import oracle as O
from gemm_tern_gemv_b200 import synth
from tests.gpu_cases import check_product, sample_rows, workload, pack_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402

LAYOUTS = [T.Q2_0_G128, T.T3_5PB_G128]


def _run(codes, s, x, layout, k, out=None, workspace=None):
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    y = T.gemv(W, torch.from_numpy(x).cuda(), y=out, workspace=workspace)
    torch.cuda.synchronize()
    return W, y.cpu().numpy()


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("n,k", [(1, 128), (17, 256), (130, 384), (200, 640), (257, 1152), (1000, 2176),
                                 (64, 5120), (33, 17408)])
@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5, 8, 13, 16, 33, 64])
def test_small_shapes_full_oracle(layout, n, k, batch):
    codes, s, x = workload(layout, n, k, batch, seed=n * 7 + k + batch)
    _, y = _run(codes, s, x, layout, k)
    y_ref, a = O.gemv(codes, s, x, layout, k)
    check_product(y, y_ref, a, f"layout {layout} n {n} k {k} b {batch}")


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("batch", [1, 4, 64])
def test_integer_inputs_are_exact(layout, batch):
    n, k = 96, 640
    t = synth.ternary_codes(n, k, seed=5)
    s = np.ones((n, k // 128), dtype=np.float16)
    x = np.random.default_rng(5).integers(-2, 3, size=(batch, k)).astype(np.float16)
    codes = pack_rows(t, layout)
    _, y = _run(codes, s, x, layout, k)
    exact = x.astype(np.int64) @ t.astype(np.int64).T
    assert np.abs(exact).max() <= 2048
    assert np.array_equal(y.astype(np.float64), exact.astype(np.float64))


@pytest.mark.parametrize("layout", LAYOUTS)
def test_closed_forms(layout):
    n, k, batch = 80, 1024, 3
    s = synth.group_scales(n, k // 128, seed=2)
    x = synth.activations(batch, k, seed=2)
    zero = pack_rows(np.zeros((n, k), np.int8), layout)
    _, y = _run(zero, s, x, layout, k)
    assert np.abs(y.astype(np.float64)).max() <= 1e-5
    ones = pack_rows(np.ones((n, k), np.int8), layout)
    _, y = _run(ones, s, x, layout, k)
    gs = x.astype(np.float64).reshape(batch, k // 128, 128).sum(axis=2)
    y_ref = gs @ s.astype(np.float64).T
    a = np.abs(x.astype(np.float64)) @ np.repeat(s.astype(np.float64), 128, axis=1).T
    check_product(y, y_ref, a, "all +1")


def test_activation_dynamic_range():
    # tiny, huge and mixed-magnitude activations: the per-group power-of-two scaling keeps them exact
    n, k = 64, 1024
    codes, s, _ = workload(T.Q2_0_G128, n, k, 4, seed=9)
    rng = np.random.default_rng(9)
    x = np.stack([rng.standard_normal(k) * 1e-6, rng.standard_normal(k) * 3e3,
                  rng.standard_normal(k) * np.where(rng.random(k) < 0.01, 1e4, 1e-3),
                  np.zeros(k)]).astype(np.float16)
    _, y = _run(codes, s, x, T.Q2_0_G128, k)
    y_ref, a = O.gemv(codes, s, x, T.Q2_0_G128, k)
    check_product(y, y_ref, a, "dynamic range")


@pytest.mark.parametrize("layout", LAYOUTS)
def test_split_k_deterministic_and_workspace_reuse(layout):
    n, k, batch = 1000, 17408, 4
    codes, s, x = workload(layout, n, k, batch, seed=11)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    ws = T.gemv_workspace(W, batch)
    assert ws is not None  # narrow matrix: split-K path
    xg = torch.from_numpy(x).cuda()
    y1 = T.gemv(W, xg, workspace=ws).clone()
    y2 = T.gemv(W, xg, workspace=ws).clone()
    torch.cuda.synchronize()
    # the second call reuses the workspace: it only matches if the arrival counters reset themselves
    assert torch.equal(y1, y2)
    rows = sample_rows(n, 256, 1)
    y_ref, a = O.gemv(codes, s, x, layout, k, rows=rows)
    check_product(y1.cpu().numpy()[:, rows], y_ref, a, "split-K")


@pytest.mark.parametrize("layout", LAYOUTS + [T.Q1_0_G128])
@pytest.mark.parametrize("n,k,batch", [(1000, 17408, 1), (1000, 17408, 2), (5120, 17408, 1), (300, 5120, 2)])
def test_cluster_k_split_is_deterministic(layout, n, k, batch):
    # batches 1-2 of narrow matrices split K over a thread-block cluster and add the slices through
    # distributed shared memory in a fixed order: no workspace, and repeated calls agree bit for bit
    codes, s, x = workload(layout, n, k, batch, seed=n + k + 17)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    assert T.gemv_workspace(W, batch) is None
    xg = torch.from_numpy(x).cuda()
    y1 = T.gemv(W, xg).clone()
    y2 = T.gemv(W, xg, static_weights=True).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    rows = sample_rows(n, 384, 7)
    y_ref, a = O.gemv(codes, s, x, layout, k, rows=rows)
    check_product(y1.cpu().numpy()[:, rows], y_ref, a, "cluster K split")


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("n,k,batch", [(4096, 4096, 1), (24576, 4096, 2), (4096, 12288, 1), (300, 2048, 1)])
def test_cta_local_reduction_is_deterministic(layout, n, k, batch):
    # these shapes sum each row tile inside one CTA (no workspace); repeated calls agree bit for bit
    codes, s, x = workload(layout, n, k, batch, seed=n + k + 3)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    xg = torch.from_numpy(x).cuda()
    if layout != T.T3_5PB_G128 or k == 4096:
        assert T.gemv_workspace(W, batch) is None
    y1 = T.gemv(W, xg).clone()
    y2 = T.gemv(W, xg, static_weights=True).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    rows = sample_rows(n, 384, 5)
    y_ref, a = O.gemv(codes, s, x, layout, k, rows=rows)
    check_product(y1.cpu().numpy()[:, rows], y_ref, a, "CTA-local reduction")


# ---------------------------------------------------------------- the workload configurations
def _config_case(layout, n, k, batch, seed, rows=512):
    codes, s, x = workload(layout, n, k, batch, seed)
    _, y = _run(codes, s, x, layout, k)
    r = sample_rows(n, rows, seed)
    y_ref, a = O.gemv(codes, s, x, layout, k, rows=r)
    return check_product(y[:, r], y_ref, a, f"layout {layout} {n}x{k} b{batch}")


def test_config1_single_gemv_full():
    # 1024 x 1024, batch 1, Q2_0_g128, seed 0: every output checked
    codes, s, x = workload(T.Q2_0_G128, 1024, 1024, 1, seed=synth.seed_for(1, 0))
    _, y = _run(codes, s, x, T.Q2_0_G128, 1024)
    y_ref, a = O.gemv(codes, s, x, T.Q2_0_G128, 1024)
    check_product(y, y_ref, a, "config 1")


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("mi,n,k", [(0, 4096, 4096), (1, 24576, 4096), (2, 4096, 12288)])
def test_config2_8b_layer_set(layout, mi, n, k):
    _config_case(layout, n, k, 1, synth.seed_for(2, mi) + 10 * layout)


@pytest.mark.parametrize("batch", [1, 8])
def test_config3_lm_head(batch):
    _config_case(T.T3_5PB_G128, 151936, 4096, batch, synth.seed_for(3, batch))


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("mi,n,k", [(0, 34816, 5120), (1, 5120, 17408)])
@pytest.mark.parametrize("batch", [1, 4, 16, 64])
def test_config4_27b_batched(layout, mi, n, k, batch):
    _config_case(layout, n, k, batch, synth.seed_for(4, mi) + 10 * layout + batch, rows=256)
