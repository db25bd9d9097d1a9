"""tern_gemv_ex with TERN_GEMV_STATIC_WEIGHTS (programmatic dependent launch, weights streamed before
the preceding grid completes) gives bit-identical results to tern_gemv, also when each call reads
the previous call's output, when consecutive calls share one workspace, and inside a CUDA graph."""
import numpy as np
import pytest

import oracle as O
from gemm_tern_gemv_b200 import synth
from tests.gpu_cases import check_product, workload

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402

LAYOUTS = [T.Q2_0_G128, T.T3_5PB_G128, T.Q1_0_G128]


def _mat(layout, n, k, seed):
    codes, s, _ = workload(layout, n, k, 1, seed)
    return T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k), codes, s


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("batch", [1, 2])
def test_chain_of_dependent_calls_matches_plain_calls(layout, batch):
    # x -> W1 (4096 x 2048) -> W2 (1024 x 4096) -> W3 (6144 x 1024): every call reads the last output
    shapes = [(4096, 2048), (1024, 4096), (6144, 1024)]
    mats = [_mat(layout, n, k, 40 + i) for i, (n, k) in enumerate(shapes)]
    x = torch.from_numpy(synth.activations(batch, 2048, 41)).cuda()
    ws = [T.gemv_workspace(W, batch) for W, _, _ in mats]

    def run(static):
        h = x
        for (W, _, _), w in zip(mats, ws):
            # scale the activations back to O(1) so later layers stay in fp16 range
            h = T.gemv(W, h, workspace=w, static_weights=static).float().mul_(0.25).to(torch.float16)
        return h

    plain = run(False)
    fast = run(True)
    torch.cuda.synchronize()
    assert torch.equal(plain, fast)
    # the last layer against the oracle, fed the GPU's own input to it
    h = x
    for (W, _, _), w in zip(mats[:-1], ws[:-1]):
        h = T.gemv(W, h, workspace=w, static_weights=True).float().mul_(0.25).to(torch.float16)
    W3, c3, s3 = mats[-1]
    y = T.gemv(W3, h, workspace=ws[-1], static_weights=True)
    y_ref, a = O.gemv(c3, s3, h.cpu().numpy(), layout, 1024)
    check_product(y.cpu().numpy(), y_ref, a, "last layer of the chain")


@pytest.mark.parametrize("layout", LAYOUTS)
def test_back_to_back_calls_share_one_workspace(layout):
    # batch 4 of a narrow matrix runs split-K through the workspace (binary: K = 17280 is not a
    # multiple of 256, which keeps it on the register kernel and its workspace)
    n, batch = 1000, 4
    k = 17280 if layout == T.Q1_0_G128 else 17408
    W, codes, s = _mat(layout, n, k, 50)
    ws = T.gemv_workspace(W, batch)
    assert ws is not None
    xs = [torch.from_numpy(synth.activations(batch, k, 51 + i)).cuda() for i in range(6)]
    ref = [T.gemv(W, x, workspace=ws).clone() for x in xs]
    ys = [torch.empty((batch, n), dtype=torch.float16, device="cuda") for _ in xs]
    for x, y in zip(xs, ys):
        T.gemv(W, x, y=y, workspace=ws, static_weights=True)
    torch.cuda.synchronize()
    for a, b in zip(ref, ys):
        assert torch.equal(a, b)


@pytest.mark.parametrize("layout", LAYOUTS)
def test_static_weights_inside_a_cuda_graph(layout):
    batch = 1
    mats = [_mat(layout, n, k, 60 + i) for i, (n, k) in enumerate([(4096, 4096), (24576, 4096), (4096, 12288)])]
    xs = [torch.from_numpy(synth.activations(batch, W.k, 70 + i)).cuda() for i, (W, _, _) in enumerate(mats)]
    ws = [T.gemv_workspace(W, batch) for W, _, _ in mats]
    ys = [torch.empty((batch, W.n), dtype=torch.float16, device="cuda") for W, _, _ in mats]
    ref = [T.gemv(W, x, workspace=w).clone() for (W, _, _), x, w in zip(mats, xs, ws)]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for (W, _, _), x, y, w in zip(mats, xs, ys, ws):  # warm-up outside capture
            T.gemv(W, x, y=y, workspace=w, static_weights=True)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for (W, _, _), x, y, w in zip(mats, xs, ys, ws):
                T.gemv(W, x, y=y, workspace=w, static_weights=True)
        for y in ys:
            y.zero_()
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    for a, b in zip(ref, ys):
        assert torch.equal(a, b)
    del g
