"""A pipeline wait that runs out is reported, not hung on and not silent.

The pages ask a runtime to refuse loudly what it cannot carry out instead of emitting garbage
("Ternary Bonsai 2 27B ..." discuss.pytorch.kr, the runtime notes after section "블록 단위 하다마드
회전"). tern_gemv_opt takes a bound on every internal pipeline wait; with a bound of 1 ns the
producer's first wait for a free ring slot runs out (the consumers cannot have released it yet), so
the call must come back with TERN_DEVICE_TIMEOUT in the status word, NaN outputs for the abandoned
rows, and a GPU that still computes the next call correctly. Nothing here faults, traps or hangs:
every wait is bounded in the kernel."""
import numpy as np
import pytest

import oracle as O
from tests.gpu_cases import check_product, sample_rows, workload

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gemm_tern_gemv_b200 as T  # noqa: E402


@pytest.mark.parametrize("layout", [T.Q2_0_G128, T.T3_5PB_G128, T.Q1_0_G128])
def test_wait_that_runs_out_sets_status_and_poisons_output(layout):
    n, k = 24576, 4096  # many row tiles per CTA: the producer must wait for a slot early on
    codes, s, x = workload(layout, n, k, 1, seed=77)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), layout, k)
    xg = torch.from_numpy(x).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = T.gemv_opt(W, xg, status=status, wait_limit_ns=1)
    torch.cuda.synchronize()  # the call returns: nothing hangs
    assert int(status.item()) & T.DEVICE_TIMEOUT
    assert torch.isnan(y.float()).any()  # the abandoned rows are NaN, never silently wrong numbers
    # the context is still usable: the default bound gives the right answer and a clean status
    status.zero_()
    y = T.gemv_opt(W, xg, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = sample_rows(n, 256, 3)
    y_ref, a = O.gemv(codes, s, x, layout, k, rows=rows)
    check_product(y.cpu().numpy()[:, rows], y_ref, a, "after a timeout")


def test_status_word_stays_clear_on_a_normal_call():
    n, k = 4096, 12288
    codes, s, x = workload(T.Q2_0_G128, n, k, 2, seed=78)
    W = T.from_packed(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), T.Q2_0_G128, k)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = T.gemv_opt(W, torch.from_numpy(x).cuda(), status=status, static_weights=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert not torch.isnan(y.float()).any()
