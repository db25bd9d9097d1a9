"""The C-ABI library loads, exports every symbol include/tern.h declares, and its host-only logic
(size arithmetic, status strings, argument validation) behaves as documented. No GPU needed: the
validation paths return before any launch, and pointer arguments here are never dereferenced."""
import ctypes
import os
import re
import subprocess

import pytest

import gemm_tern_gemv_b200 as T
import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tern.h")


@pytest.fixture(scope="module")
def lib():
    from gemm_tern_gemv_b200 import build
    build.build()
    return T.lib()


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"TERN_API\s+[\w\s\*]+?\b(tern_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("tern_pack", "tern_unpack", "tern_gemv", "tern_gemm", "tern_gemv_workspace_bytes",
              "tern_row_bytes", "tern_packed_bytes", "tern_bits_per_weight", "tern_status_string",
              "tern_hadamard_rotate"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", T.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(tern_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(lib, n)
    assert set(T.SIGNATURES) >= set(_declared())


def test_size_arithmetic_matches_oracle(lib):
    for layout in (T.Q2_0_G128, T.T3_5PB_G128, T.Q1_0_G128):
        for k in list(range(128, 20000, 128)) + [151936 // 128 * 128]:
            assert T.row_bytes(layout, k) == O.row_bytes(layout, k)
            assert T.packed_bytes(layout, 7, k) == O.packed_bytes(layout, 7, k)
            assert T.bits_per_weight(layout, k) == pytest.approx(O.bits_per_weight(layout, k), abs=0, rel=1e-15)
    assert T.bits_per_weight(T.Q2_0_G128, 4096) == 2.125
    assert T.bits_per_weight(T.T3_5PB_G128, 5120) == 1.725
    assert T.bits_per_weight(T.Q1_0_G128, 4096) == 1.125
    assert lib.tern_row_bytes(4, 128) == -1
    assert lib.tern_row_bytes(0, 128) == -1
    assert lib.tern_row_bytes(1, 100) == -1
    assert lib.tern_row_bytes(1, 0) == -1
    assert lib.tern_packed_bytes(1, 0, 128) == -1
    assert lib.tern_bits_per_weight(9, 128) == -1.0


def test_status_strings(lib):
    for s in range(8):
        assert lib.tern_status_string(s).decode()
    assert lib.tern_status_string(0).decode() == "ok"
    assert lib.tern_status_string(99).decode() == "unknown status"


# 16-byte aligned and never dereferenced: every call below is rejected on the host before a launch
FAKE = 0x7F0000000000


def _mat(**kw):
    d = dict(layout=1, n=64, k=1024, codes=FAKE, code_row_stride=256, scales=FAKE + 4096, scale_row_stride=8)
    d.update(kw)
    return T.TernMatrixC(d["layout"], d["n"], d["k"], d["codes"], d["code_row_stride"], d["scales"],
                         d["scale_row_stride"])


@pytest.mark.parametrize("kw,status", [
    (dict(layout=0), 2), (dict(layout=4), 2), (dict(n=0), 1), (dict(k=1000), 1), (dict(k=0), 1),
    (dict(codes=0), 1), (dict(scales=0), 1), (dict(code_row_stride=128), 1), (dict(scale_row_stride=4), 1),
    (dict(codes=FAKE + 8), 3), (dict(scales=FAKE + 2), 3), (dict(code_row_stride=264), 3),
    (dict(scale_row_stride=12), 3),
])
def test_gemv_rejects_bad_matrix(lib, kw, status):
    m = _mat(**kw)
    st = lib.tern_gemv(ctypes.byref(m), ctypes.c_void_p(FAKE), 1, ctypes.c_void_p(FAKE), None, 0, None)
    assert st == status


def test_gemv_ex_rejects_unknown_flags(lib):
    m = _mat()
    args = (ctypes.byref(m), ctypes.c_void_p(FAKE), 1, ctypes.c_void_p(FAKE), None, 0)
    assert lib.tern_gemv_ex(*args, 2, None) == 1
    assert lib.tern_gemv_ex(*args, 0x80000000, None) == 1
    # a valid flag passes the flag check and stops at the next host-side check (missing workspace;
    # batch 4 of this shape runs split-K)
    w = _mat(n=5120, k=17408, code_row_stride=4352, scale_row_stride=136)
    assert lib.tern_gemv_ex(ctypes.byref(w), ctypes.c_void_p(FAKE), 4, ctypes.c_void_p(FAKE), None, 0, 1, None) == 4


def test_gemv_rejects_bad_batch_and_buffers(lib):
    m = _mat()
    assert lib.tern_gemv(ctypes.byref(m), ctypes.c_void_p(FAKE), 0, ctypes.c_void_p(FAKE), None, 0, None) == 1
    assert lib.tern_gemv(ctypes.byref(m), ctypes.c_void_p(FAKE), 65, ctypes.c_void_p(FAKE), None, 0, None) == 1
    assert lib.tern_gemv(ctypes.byref(m), None, 1, ctypes.c_void_p(FAKE), None, 0, None) == 1
    assert lib.tern_gemv(ctypes.byref(m), ctypes.c_void_p(FAKE + 2), 1, ctypes.c_void_p(FAKE), None, 0, None) == 3
    assert lib.tern_gemv(None, ctypes.c_void_p(FAKE), 1, ctypes.c_void_p(FAKE), None, 0, None) == 1


def test_gemv_workspace_size_and_rejection(lib):
    # a narrow matrix with a long K at batch 4 needs split-K workspace; too little is refused before
    # any launch
    m = _mat(n=5120, k=17408, code_row_stride=4352, scale_row_stride=136)
    need = lib.tern_gemv_workspace_bytes(ctypes.byref(m), 4)
    assert need > 0 and need % 16 == 0
    assert lib.tern_gemv(ctypes.byref(m), ctypes.c_void_p(FAKE), 4, ctypes.c_void_p(FAKE), None, 0, None) == 4
    assert lib.tern_gemv(ctypes.byref(m), ctypes.c_void_p(FAKE), 4, ctypes.c_void_p(FAKE),
                         ctypes.c_void_p(FAKE), need - 16, None) == 4
    assert lib.tern_gemv(ctypes.byref(m), ctypes.c_void_p(FAKE), 4, ctypes.c_void_p(FAKE),
                         ctypes.c_void_p(FAKE + 8), need, None) == 3
    # batches 1 and 2 split K over thread-block clusters instead and need none, in every layout
    for layout, rb in ((1, 4352), (2, 3488), (3, 2176)):
        w = _mat(layout=layout, n=5120, k=17408, code_row_stride=rb, scale_row_stride=136)
        assert lib.tern_gemv_workspace_bytes(ctypes.byref(w), 1) == 0
        assert lib.tern_gemv_workspace_bytes(ctypes.byref(w), 2) == 0
    # a matrix of one 128-weight group per row is never split and needs none; neither do the 8B-class
    # decode shapes at batch 1, whose tiles are summed inside each CTA
    one = _mat(n=4096, k=128, code_row_stride=32, scale_row_stride=8)
    assert lib.tern_gemv_workspace_bytes(ctypes.byref(one), 1) == 0
    for layout, rb in ((1, 1024), (2, 832), (3, 512)):
        for n in (4096, 24576):
            sq = _mat(layout=layout, n=n, k=4096, code_row_stride=rb, scale_row_stride=32)
            assert lib.tern_gemv_workspace_bytes(ctypes.byref(sq), 1) == 0
    # the size is a pure function of the arguments; batch outside 1..64 gives 0
    big = _mat(n=151936, k=4096, code_row_stride=1024, scale_row_stride=32)
    assert lib.tern_gemv_workspace_bytes(ctypes.byref(big), 1) == lib.tern_gemv_workspace_bytes(ctypes.byref(big), 1)
    assert lib.tern_gemv_workspace_bytes(ctypes.byref(big), 0) == 0
    assert lib.tern_gemv_workspace_bytes(ctypes.byref(big), 65) == 0
    assert lib.tern_gemv_workspace_bytes(None, 1) == 0


def test_binary_gemv_workspace_is_that_of_two_rows(lib):
    # binary batches below the GEMM's run as pairs of rows, one launch after another on the stream,
    # so every such batch reuses the workspace of a two-row launch (none on the int8-plane kernel;
    # K = 17280 is not a multiple of 256 and runs on the register kernel, which needs one)
    for k, rb, need in ((17408, 2176, False), (17280, 2160, True)):
        m = _mat(layout=3, n=5120, k=k, code_row_stride=rb, scale_row_stride=k // 128 + 7 & ~7)
        two = lib.tern_gemv_workspace_bytes(ctypes.byref(m), 2)
        assert (two > 0) == need
        for b in (3, 4):
            assert lib.tern_gemv_workspace_bytes(ctypes.byref(m), b) == two
    m = _mat(layout=3, n=5120, k=17408, code_row_stride=2176, scale_row_stride=136)
    for b in (5, 16, 17):  # the GEMM kernel takes binary batches from 5 on (n % 8 == 0)
        assert lib.tern_gemv_workspace_bytes(ctypes.byref(m), b) == 0
    odd = _mat(layout=3, n=5121, k=17408, code_row_stride=2176, scale_row_stride=136)
    assert lib.tern_gemv_workspace_bytes(ctypes.byref(odd), 16) == lib.tern_gemv_workspace_bytes(ctypes.byref(odd), 2)


def test_pack_unpack_gemm_reject(lib):
    P = lambda v: ctypes.c_void_p(v)
    assert lib.tern_pack(4, 4, 128, P(FAKE), 128, P(FAKE), 8, P(FAKE), 32, None) == 2
    assert lib.tern_pack(3, 4, 256, P(FAKE), 256, P(FAKE), 8, P(FAKE), 16, None) == 1  # binary row needs 32
    assert lib.tern_pack(1, 4, 130, P(FAKE), 136, P(FAKE), 8, P(FAKE), 48, None) == 1
    assert lib.tern_pack(1, 4, 128, P(FAKE), 120, P(FAKE), 8, P(FAKE), 32, None) == 1
    assert lib.tern_pack(1, 4, 128, P(FAKE + 4), 128, P(FAKE), 8, P(FAKE), 32, None) == 3
    assert lib.tern_pack(2, 4, 128, P(FAKE), 128, P(FAKE), 8, P(FAKE), 16, None) == 1  # base-3 row needs 32
    m = _mat()
    assert lib.tern_unpack(ctypes.byref(m), None, 1024, None, 1024, None, None) == 1
    assert lib.tern_unpack(ctypes.byref(m), P(FAKE), 1000, None, 0, None, None) == 1
    assert lib.tern_unpack(ctypes.byref(m), P(FAKE), 1028, None, 0, None, None) == 3
    t3 = _mat(layout=2, code_row_stride=208)
    assert lib.tern_gemm(ctypes.byref(t3), P(FAKE), 0, P(FAKE), None, None) == 1  # base-3 accepted up to m
    q1 = _mat(layout=3, code_row_stride=128)
    assert lib.tern_gemm(ctypes.byref(q1), P(FAKE), 0, P(FAKE), None, None) == 1  # binary accepted up to m
    assert lib.tern_gemm(ctypes.byref(_mat(layout=4)), P(FAKE), 16, P(FAKE), None, None) == 2
    assert lib.tern_gemm(ctypes.byref(m), P(FAKE), 0, P(FAKE), None, None) == 1
    assert lib.tern_gemm(ctypes.byref(_mat(n=60)), P(FAKE), 16, P(FAKE), None, None) == 3


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(T, "_lib", None)
    monkeypatch.setattr(T, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="missing"):
        T.lib()


def test_hadamard_rotate_rejects_before_launch(lib):
    P = lambda v: ctypes.c_void_p(v)
    f = lib.tern_hadamard_rotate
    assert f(None, 1, 1024, P(FAKE), P(FAKE), None) == 1
    assert f(P(FAKE), 1, 1024, None, P(FAKE), None) == 1
    assert f(P(FAKE), 0, 1024, P(FAKE), P(FAKE), None) == 1
    assert f(P(FAKE), 1, 1000, P(FAKE), P(FAKE), None) == 1
    assert f(P(FAKE), 1, 0, P(FAKE), P(FAKE), None) == 1
    assert f(P(FAKE + 1), 1, 1024, P(FAKE), P(FAKE), None) == 3
    assert f(P(FAKE), 1, 1024, P(FAKE), P(FAKE + 1), None) == 3


def test_pack_flips_rejects_before_launch(lib):
    P = lambda v: ctypes.c_void_p(v)
    f = lib.tern_pack_flips
    ok = (1, 4, 128, P(FAKE), 128, P(FAKE + 4096), 8, P(FAKE + 8192), 32)
    assert f(*ok, None, 32, P(FAKE + 16384), None) == 1                       # no previous codes
    assert f(*ok, P(FAKE + 12288), 32, None, None) == 1                       # no counter
    assert f(*ok, P(FAKE + 8192), 32, P(FAKE + 16384), None) == 1             # previous == output
    assert f(*ok, P(FAKE + 12288), 16, P(FAKE + 16384), None) == 1            # short previous stride
    assert f(*ok, P(FAKE + 12296), 32, P(FAKE + 16384), None) == 3            # misaligned previous codes
    assert f(*ok, P(FAKE + 12288), 32, P(FAKE + 16388), None) == 3            # misaligned counter


def test_gemv_t_rejects_before_launch(lib):
    P = lambda v: ctypes.c_void_p(v)
    m = _mat(n=4096, k=4096, code_row_stride=1024, scale_row_stride=32)
    need = lib.tern_gemv_t_workspace_bytes(ctypes.byref(m), 1)
    assert need > 0 and need % 4 == 0
    assert lib.tern_gemv_t_workspace_bytes(ctypes.byref(m), 9) == 0
    assert lib.tern_gemv_t(ctypes.byref(m), P(FAKE), 9, P(FAKE), None, 0, None) == 1
    assert lib.tern_gemv_t(ctypes.byref(m), None, 1, P(FAKE), None, 0, None) == 1
    assert lib.tern_gemv_t(ctypes.byref(m), P(FAKE + 1), 1, P(FAKE), None, 0, None) == 3
    assert lib.tern_gemv_t(ctypes.byref(m), P(FAKE), 1, P(FAKE), None, 0, None) == 4
    assert lib.tern_gemv_t(ctypes.byref(m), P(FAKE), 1, P(FAKE), P(FAKE + 8), need, None) == 3


def test_noalloc_scratch_claim_of_the_header(lib):
    # tern.h: batch <= 8 fits the static scratch for N <= 151936 at K = 4096 and for N <= 34816 up to
    # K = 17408 (the plan arithmetic is host-side, so the workspace size can be checked without a GPU)
    limit = 8 << 20
    for layout, rb in ((1, lambda k: k // 4), (2, lambda k: -(-(-(-k // 5)) // 16) * 16), (3, lambda k: k // 8)):
        for b in range(1, 9):
            for n in (128, 4096, 24576, 65536, 151936):
                m = _mat(layout=layout, n=n, k=4096, code_row_stride=rb(4096), scale_row_stride=32)
                assert lib.tern_gemv_workspace_bytes(ctypes.byref(m), b) <= limit
            for k in (1024, 5120, 12288, 17408):
                for n in (1000, 5120, 34816, 151936 if k == 4096 else 34816):
                    m = _mat(layout=layout, n=n, k=k, code_row_stride=rb(k), scale_row_stride=k // 128)
                    assert lib.tern_gemv_workspace_bytes(ctypes.byref(m), b) <= limit


def test_device_result_turns_device_words_into_statuses(lib):
    # TERN_DEVICE_TIMEOUT wins over an invalid-code count; both map to the reserved statuses
    assert lib.tern_device_result(0, 0) == 0
    assert lib.tern_device_result(1, 0) == 6   # TERN_ERR_TIMEOUT
    assert lib.tern_device_result(1, 5) == 6
    assert lib.tern_device_result(0, 3) == 5   # TERN_ERR_INVALID_CODE
    assert lib.tern_device_result(2, 0) == 0   # bits other than TERN_DEVICE_TIMEOUT are not errors
    assert lib.tern_device_result(0, -1) == 0


def test_gemv_opt_rejects_before_launch(lib):
    import gemm_tern_gemv_b200 as T
    m = _mat()
    args = (ctypes.byref(m), ctypes.c_void_p(FAKE), 1, ctypes.c_void_p(FAKE), None, 0)
    bad_flag = T.TernGemvOptsC(2, None, 0)
    assert lib.tern_gemv_opt(*args, ctypes.byref(bad_flag), None) == 1
    misaligned = T.TernGemvOptsC(0, FAKE + 2, 0)
    assert lib.tern_gemv_opt(*args, ctypes.byref(misaligned), None) == 3


def test_rotated_gemv_checks_and_workspace(lib):
    import gemm_tern_gemv_b200 as T
    # K must be a multiple of the 1024-element rotation block; rejected before any CUDA call
    m = _mat(k=1152, code_row_stride=288, scale_row_stride=16)
    rot = T.TernGemvOptsC(0, None, 0, FAKE + 8192)
    args = (ctypes.byref(m), ctypes.c_void_p(FAKE), 1, ctypes.c_void_p(FAKE), None, 0)
    assert lib.tern_gemv_opt(*args, ctypes.byref(rot), None) == 1
    assert lib.tern_gemv_opt_workspace_bytes(ctypes.byref(m), 1, ctypes.byref(rot)) == 0
    plain = T.TernGemvOptsC(0, None, 0, None)
    for layout, rb in ((1, 1024), (2, 832), (3, 512)):
        for b in (1, 2, 3, 4, 17):
            m = _mat(layout=layout, n=4096, k=4096, code_row_stride=rb, scale_row_stride=32)
            base = lib.tern_gemv_workspace_bytes(ctypes.byref(m), b)
            # without a rotation the size is tern_gemv_workspace_bytes'
            assert lib.tern_gemv_opt_workspace_bytes(ctypes.byref(m), b, ctypes.byref(plain)) == base
            need = lib.tern_gemv_opt_workspace_bytes(ctypes.byref(m), b, ctypes.byref(rot))
            # batches 1-2 rotate inside the int8-plane kernel (binary: also 3-4, as pairs); the rest
            # add the rotated x after the GEMV's own workspace, 256-byte aligned
            fused = b <= 2 or (layout == 3 and b <= 4)
            assert need == (base if fused else (base + 255) // 256 * 256 + b * 4096 * 2), (layout, b, base, need)


def _describe(lib, layout, n, k, b, signs=None):
    import gemm_tern_gemv_b200 as T
    rb = {1: k // 4, 2: -(-(-(-k // 5)) // 16) * 16, 3: k // 8}[layout]
    m = _mat(layout=layout, n=n, k=k, code_row_stride=rb, scale_row_stride=max(8, -(-(k // 128) // 8) * 8))
    o = T.TernGemvOptsC(0, None, 0, signs)
    info = T.TernGemvPlanInfoC()
    st = lib.tern_gemv_plan_describe(ctypes.byref(m), b, ctypes.byref(o), ctypes.byref(info))
    return st, info, m, o


def test_plan_description_follows_the_planner_rules(lib):
    # (148-SM B200 planning without a GPU) the int8-plane kernel takes batches 1-2 with one K slice
    # when it fits: two CTAs of 8 warps per SM from 14 row tiles per SM, 8 warps for at most two tiles,
    # else one CTA of 16; a slice that does not fit splits K over a pair of CTAs with 12 warps
    expect = {  # (layout, n, k, batch): (k_slices, ctas_per_sm, warps)
        (1, 4096, 4096, 1): (1, 1, 8), (1, 24576, 4096, 1): (1, 1, 16), (2, 24576, 4096, 1): (1, 1, 16),
        (2, 151936, 4096, 1): (1, 2, 8), (1, 34816, 5120, 1): (1, 2, 8), (2, 4096, 12288, 1): (2, 1, 12),
        (1, 5120, 17408, 1): (2, 1, 12), (2, 5120, 17408, 1): (2, 1, 12), (3, 24576, 4096, 1): (1, 1, 16),
    }
    for (layout, n, k, b), (ks, cps, nw) in expect.items():
        st, info, m, _ = _describe(lib, layout, n, k, b)
        assert st == 0
        assert info.kernel == 1 and info.launches == 1, (layout, n, k, b)
        assert (info.k_slices, info.ctas_per_sm, info.warps) == (ks, cps, nw), (layout, n, k, b, info.k_slices,
                                                                                info.ctas_per_sm, info.warps)
        assert info.stages >= 2 and info.workspace_bytes == lib.tern_gemv_workspace_bytes(ctypes.byref(m), b) == 0
    # batch 2 of the LM head stays on the older kernels (a K split there would keep a partial per tile)
    st, info, _, _ = _describe(lib, 2, 151936, 4096, 2)
    assert st == 0 and info.kernel != 1
    # binary batches 3-4 run as pairs of rows on the int8-plane kernel; batch 17 with N % 8 == 0 on tcgen05
    st, info, _, _ = _describe(lib, 3, 4096, 4096, 3)
    assert st == 0 and info.kernel == 1 and info.launches == 2
    for layout in (1, 2, 3):
        st, info, _, _ = _describe(lib, layout, 4096, 4096, 17)
        assert st == 0 and info.kernel == 4 and info.launches == 1
    # every described plan is self-consistent over a sweep of shapes and batches
    for layout in (1, 2, 3):
        for n in (1, 17, 4096, 34816):
            for k in (1024, 4096, 5120, 17408):
                for b in (1, 2, 3, 8, 16, 64):
                    st, info, m, o = _describe(lib, layout, n, k, b)
                    assert st == 0
                    assert 1 <= info.kernel <= 4 and info.launches >= 1 and info.k_slices >= 1
                    assert info.workspace_bytes == lib.tern_gemv_opt_workspace_bytes(ctypes.byref(m), b, ctypes.byref(o))
                    if info.kernel == 1:
                        assert b <= 2 or layout == 3
                        assert info.k_slices in (1, 2, 4) and info.ctas_per_sm in (1, 2) and info.stages >= 2
                        assert info.warps <= (8 if info.ctas_per_sm == 2 else 17)


def test_plan_description_of_the_rotation(lib):
    signs = FAKE + 8192
    st, info, m, o = _describe(lib, 1, 4096, 4096, 1, signs)
    assert st == 0 and info.rotation_fused == 1 and info.launches == 1 and info.workspace_bytes == 0
    st, info, m, o = _describe(lib, 1, 4096, 4096, 3, signs)  # register kernel: rotate into the workspace
    assert st == 0 and info.rotation_fused == 0 and info.launches == 2
    assert info.workspace_bytes == lib.tern_gemv_opt_workspace_bytes(ctypes.byref(m), 3, ctypes.byref(o)) > 0
    st, info, _, _ = _describe(lib, 1, 4096, 1152, 1, signs)
    assert st == 1  # K is not a multiple of the 1024-element rotation block
