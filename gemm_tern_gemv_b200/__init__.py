"""Python binding of libtern.so: ternary group-scaled GEMV / GEMM / pack / unpack on B200.

Argument marshalling only. Every step of the computation runs in the library's CUDA kernels;
PyTorch supplies device memory and the current CUDA stream. There is no fallback: if libtern.so
is missing or cannot be loaded, every call raises.

    W = pack(w_fp16, scales_fp16, layout=Q2_0_G128)     # ternarize + pack on the GPU
    y = gemv(W, x)                                       # x [batch][K] fp16 -> y [batch][N] fp16
    Y = gemm(W, X)                                       # X [M][K] fp16 -> Y [M][N] fp16
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

Q2_0_G128 = 1
T3_5PB_G128 = 2
Q1_0_G128 = 3
GROUP = 128
GEMV_MAX_BATCH = 64
GEMV_STATIC_WEIGHTS = 1
DEVICE_TIMEOUT = 1

STATUS = {0: "TERN_OK", 1: "TERN_ERR_INVALID_ARG", 2: "TERN_ERR_UNSUPPORTED", 3: "TERN_ERR_ALIGNMENT",
          4: "TERN_ERR_WORKSPACE", 5: "TERN_ERR_INVALID_CODE", 6: "TERN_ERR_TIMEOUT", 7: "TERN_ERR_CUDA"}

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtern.so")


class TernError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_status_string(status)})")


class TernGemvOptsC(ctypes.Structure):
    _fields_ = [("flags", ctypes.c_uint32), ("device_status", ctypes.c_void_p), ("wait_limit_ns", ctypes.c_uint64),
                ("rotate_signs", ctypes.c_void_p)]


class TernGemvPlanInfoC(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("launches", ctypes.c_int32), ("k_slices", ctypes.c_int32),
                ("ctas_per_sm", ctypes.c_int32), ("warps", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("rotation_fused", ctypes.c_int32), ("reserved", ctypes.c_int32), ("workspace_bytes", ctypes.c_uint64)]


GEMV_KERNELS = {1: "int8-planes", 2: "register", 3: "shared-memory", 4: "tcgen05"}


class TernMatrixC(ctypes.Structure):
    _fields_ = [("layout", ctypes.c_int32), ("n", ctypes.c_int64), ("k", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("code_row_stride", ctypes.c_int64),
                ("scales", ctypes.c_void_p), ("scale_row_stride", ctypes.c_int64)]


_lib = None

# name -> (restype, argtypes)
SIGNATURES = {
    "tern_row_bytes": (ctypes.c_int64, [ctypes.c_int32, ctypes.c_int64]),
    "tern_packed_bytes": (ctypes.c_int64, [ctypes.c_int32, ctypes.c_int64, ctypes.c_int64]),
    "tern_bits_per_weight": (ctypes.c_double, [ctypes.c_int32, ctypes.c_int64]),
    "tern_pack": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                 ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]),
    "tern_unpack": (ctypes.c_int, [ctypes.POINTER(TernMatrixC), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                   ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]),
    "tern_gemv_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(TernMatrixC), ctypes.c_int64]),
    "tern_gemv": (ctypes.c_int, [ctypes.POINTER(TernMatrixC), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "tern_gemv_ex": (ctypes.c_int, [ctypes.POINTER(TernMatrixC), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_void_p]),
    "tern_gemv_opt": (ctypes.c_int, [ctypes.POINTER(TernMatrixC), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(TernGemvOptsC), ctypes.c_void_p]),
    "tern_gemv_opt_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(TernMatrixC), ctypes.c_int64,
                                                        ctypes.POINTER(TernGemvOptsC)]),
    "tern_gemv_plan_describe": (ctypes.c_int, [ctypes.POINTER(TernMatrixC), ctypes.c_int64,
                                               ctypes.POINTER(TernGemvOptsC), ctypes.POINTER(TernGemvPlanInfoC)]),
    "tern_gemv_noalloc": (ctypes.c_int, [ctypes.POINTER(TernMatrixC), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                         ctypes.c_void_p]),
    "tern_gemm": (ctypes.c_int, [ctypes.POINTER(TernMatrixC), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_void_p]),
    "tern_pack_flips": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                       ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                       ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]),
    "tern_gemv_t_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(TernMatrixC), ctypes.c_int64]),
    "tern_gemv_t": (ctypes.c_int, [ctypes.POINTER(TernMatrixC), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "tern_hadamard_rotate": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_void_p]),
    "tern_device_result": (ctypes.c_int, [ctypes.c_uint32, ctypes.c_int64]),
    "tern_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "tern_version": (ctypes.c_int32, []),
}


def lib() -> ctypes.CDLL:
    """The loaded libtern.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m gemm_tern_gemv_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _status_string(status: int) -> str:
    try:
        return lib().tern_status_string(status).decode()
    except Exception:  # pragma: no cover - only used while formatting an error
        return "?"


def _check(status: int, what: str) -> None:
    if status != 0:
        raise TernError(status, what)


def check_device_result(status=None, invalid_count=None) -> None:
    """Reads back a device status word and / or an invalid-code counter and raises TernError with
    TERN_ERR_TIMEOUT / TERN_ERR_INVALID_CODE when they report a failure (tern_device_result)."""
    st = int(status.item()) & 0xFFFFFFFF if status is not None else 0
    bad = int(invalid_count.item()) if invalid_count is not None else 0
    _check(lib().tern_device_result(st, bad), "device result")


def row_bytes(layout: int, k: int) -> int:
    return int(lib().tern_row_bytes(layout, k))


def packed_bytes(layout: int, n: int, k: int) -> int:
    return int(lib().tern_packed_bytes(layout, n, k))


def bits_per_weight(layout: int, k: int) -> float:
    return float(lib().tern_bits_per_weight(layout, k))


def version() -> int:
    return int(lib().tern_version())


# ------------------------------------------------------------------------------- torch plumbing
def _torch():
    import torch
    return torch


def _stream_handle():
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def scale_stride(k: int) -> int:
    """Row stride (in halves) used for scale tensors: k/128 rounded up to a multiple of 8."""
    g = k // GROUP
    return (g + 7) // 8 * 8


@dataclass
class TernMatrix:
    """A packed ternary matrix on the GPU: codes uint8 [n][code_row_stride], scales fp16 [n][>=k/128]."""
    layout: int
    n: int
    k: int
    codes: "object"   # torch.uint8 cuda tensor [n][stride]
    scales: "object"  # torch.float16 cuda tensor [n][sstride]

    def c(self) -> TernMatrixC:
        return TernMatrixC(self.layout, self.n, self.k, self.codes.data_ptr(), self.codes.stride(0),
                           self.scales.data_ptr(), self.scales.stride(0))

    @property
    def nbytes(self) -> int:
        """Algorithmic bytes of the packed weights: code rows + k/128 scales per row."""
        return self.n * row_bytes(self.layout, self.k) + self.n * (self.k // GROUP) * 2


def empty_matrix(layout: int, n: int, k: int, device="cuda") -> TernMatrix:
    torch = _torch()
    codes = torch.empty((n, row_bytes(layout, k)), dtype=torch.uint8, device=device)
    scales = torch.zeros((n, scale_stride(k)), dtype=torch.float16, device=device)
    return TernMatrix(layout, n, k, codes, scales)


def as_scales(scales, k: int):
    """fp16 cuda tensor [n][k/128] -> a [n][scale_stride(k)] tensor with 16-byte aligned rows."""
    torch = _torch()
    g = k // GROUP
    if scales.stride(0) % 8 == 0 and scales.stride(1) == 1 and scales.shape[1] >= g and scales.data_ptr() % 16 == 0:
        return scales
    out = torch.zeros((scales.shape[0], scale_stride(k)), dtype=torch.float16, device=scales.device)
    out[:, :g] = scales[:, :g]
    return out


def pack(w, scales, layout: int = Q2_0_G128, out: TernMatrix | None = None) -> TernMatrix:
    """Ternarize fp16 latents w [n][k] with their group scales [n][k/128] and pack them (tern_pack).

    The returned matrix holds the codes and (a 16-byte-row-aligned copy of) the scales."""
    torch = _torch()
    n, k = w.shape
    scales = as_scales(scales, k)
    if out is None:
        codes = torch.empty((n, row_bytes(layout, k)), dtype=torch.uint8, device=w.device)
        out = TernMatrix(layout, n, k, codes, scales)
    st = lib().tern_pack(layout, n, k, _ptr(w), w.stride(0), _ptr(scales), scales.stride(0), _ptr(out.codes),
                         out.codes.stride(0), _stream_handle())
    _check(st, "tern_pack")
    return out


def pack_flips(w, scales, prev: TernMatrix, out: TernMatrix | None = None, flips=None):
    """Re-pack w like pack() and count the weights whose code changed against `prev`
    (tern_pack_flips). Returns (matrix, flips) with flips a device int64 tensor (added to when given)."""
    torch = _torch()
    n, k = w.shape
    scales = as_scales(scales, k)
    if out is None:
        codes = torch.empty((n, row_bytes(prev.layout, k)), dtype=torch.uint8, device=w.device)
        out = TernMatrix(prev.layout, n, k, codes, scales)
    if flips is None:
        flips = torch.zeros(1, dtype=torch.int64, device=w.device)
    st = lib().tern_pack_flips(prev.layout, n, k, _ptr(w), w.stride(0), _ptr(scales), scales.stride(0),
                               _ptr(out.codes), out.codes.stride(0), _ptr(prev.codes), prev.codes.stride(0),
                               _ptr(flips), _stream_handle())
    _check(st, "tern_pack_flips")
    return out, flips


def from_packed(codes, scales, layout: int, k: int) -> TernMatrix:
    """Wrap already-packed codes (uint8 [n][>=row_bytes]) and scales as a TernMatrix (device copies)."""
    torch = _torch()
    n = codes.shape[0]
    return TernMatrix(layout, n, k, codes.contiguous(), as_scales(scales, k).contiguous())


def unpack(W: TernMatrix, want_w: bool = True, want_t: bool = True):
    """(w fp16 [n][k] = s*t, t int8 [n][k], invalid-code count) — test/debug path."""
    torch = _torch()
    dev = W.codes.device
    w = torch.empty((W.n, W.k), dtype=torch.float16, device=dev) if want_w else None
    t = torch.empty((W.n, W.k), dtype=torch.int8, device=dev) if want_t else None
    cnt = torch.zeros(1, dtype=torch.int32, device=dev)
    c = W.c()
    st = lib().tern_unpack(ctypes.byref(c), _ptr(w), W.k, _ptr(t), W.k, _ptr(cnt), _stream_handle())
    _check(st, "tern_unpack")
    return w, t, cnt


def gemv_workspace_bytes(W: TernMatrix, batch: int) -> int:
    c = W.c()
    return int(lib().tern_gemv_workspace_bytes(ctypes.byref(c), batch))


def gemv_workspace(W: TernMatrix, batch: int):
    """A zero-initialised workspace tensor suitable for gemv(W, x) with this batch (or None)."""
    torch = _torch()
    nb = gemv_workspace_bytes(W, batch)
    return torch.zeros(nb, dtype=torch.uint8, device=W.codes.device) if nb else None


def gemv(W: TernMatrix, x, y=None, workspace=None, static_weights: bool = False):
    """y [batch][n] = x [batch][k] @ W^T with W ternary (tern_gemv; tern_gemv_ex with
    TERN_GEMV_STATIC_WEIGHTS when `static_weights`: no pending GPU work writes W)."""
    torch = _torch()
    if x.dim() == 1:
        x = x.unsqueeze(0)
    batch = x.shape[0]
    x = x.contiguous()
    if y is None:
        y = torch.empty((batch, W.n), dtype=torch.float16, device=x.device)
    if workspace is None:
        workspace = gemv_workspace(W, batch)
    wsb = workspace.numel() if workspace is not None else 0
    c = W.c()
    if static_weights:
        st = lib().tern_gemv_ex(ctypes.byref(c), _ptr(x), batch, _ptr(y), _ptr(workspace), wsb,
                                GEMV_STATIC_WEIGHTS, _stream_handle())
        _check(st, "tern_gemv_ex")
    else:
        st = lib().tern_gemv(ctypes.byref(c), _ptr(x), batch, _ptr(y), _ptr(workspace), wsb, _stream_handle())
        _check(st, "tern_gemv")
    return y


def _opts(static_weights=False, status=None, wait_limit_ns=0, rotate_signs=None):
    return TernGemvOptsC(GEMV_STATIC_WEIGHTS if static_weights else 0, _ptr(status) if status is not None else None,
                         int(wait_limit_ns), _ptr(rotate_signs) if rotate_signs is not None else None)


def gemv_opt_workspace_bytes(W: TernMatrix, batch: int, rotate_signs=None) -> int:
    """tern_gemv_opt_workspace_bytes for these options (only the rotation changes the size)."""
    c = W.c()
    o = _opts(rotate_signs=rotate_signs)
    return int(lib().tern_gemv_opt_workspace_bytes(ctypes.byref(c), batch, ctypes.byref(o)))


def gemv_plan_describe(W: TernMatrix, batch: int, rotate_signs=None, static_weights: bool = False) -> dict:
    """tern_gemv_plan_describe: the kernel and work split tern_gemv_opt would use (host only)."""
    c = W.c()
    o = _opts(static_weights, None, 0, rotate_signs)
    info = TernGemvPlanInfoC()
    _check(lib().tern_gemv_plan_describe(ctypes.byref(c), batch, ctypes.byref(o), ctypes.byref(info)),
           "tern_gemv_plan_describe")
    d = {f: getattr(info, f) for f, _ in TernGemvPlanInfoC._fields_ if f != "reserved"}
    d["kernel"] = GEMV_KERNELS.get(d["kernel"], d["kernel"])
    return d


def gemv_opt(W: TernMatrix, x, y=None, workspace=None, static_weights: bool = False, status=None,
             wait_limit_ns: int = 0, rotate_signs=None):
    """tern_gemv_opt: gemv with an optional device status word (uint32 tensor, TERN_DEVICE_TIMEOUT is
    OR-ed in when a pipeline wait runs out), a bound on each wait (0 = the library default) and an
    optional block Hadamard rotation of x (int8 tensor of 1024 signs: y = W (R x))."""
    torch = _torch()
    if x.dim() == 1:
        x = x.unsqueeze(0)
    batch = x.shape[0]
    x = x.contiguous()
    if y is None:
        y = torch.empty((batch, W.n), dtype=torch.float16, device=x.device)
    if workspace is None:
        nb = gemv_opt_workspace_bytes(W, batch, rotate_signs)
        workspace = torch.zeros(nb, dtype=torch.uint8, device=W.codes.device) if nb else None
    wsb = workspace.numel() if workspace is not None else 0
    c = W.c()
    o = _opts(static_weights, status, wait_limit_ns, rotate_signs)
    st = lib().tern_gemv_opt(ctypes.byref(c), _ptr(x), batch, _ptr(y), _ptr(workspace), wsb, ctypes.byref(o),
                             _stream_handle())
    _check(st, "tern_gemv_opt")
    return y


def gemv_noalloc(W: TernMatrix, x, y=None):
    """tern_gemv_noalloc: the GEMV without a caller workspace (split-K scratch in a static device
    array of the library; calls on one device must not overlap on the GPU)."""
    torch = _torch()
    if x.dim() == 1:
        x = x.unsqueeze(0)
    x = x.contiguous()
    if y is None:
        y = torch.empty((x.shape[0], W.n), dtype=torch.float16, device=x.device)
    c = W.c()
    st = lib().tern_gemv_noalloc(ctypes.byref(c), _ptr(x), x.shape[0], _ptr(y), _stream_handle())
    _check(st, "tern_gemv_noalloc")
    return y


def gemv_t(W: TernMatrix, dy, dx=None, workspace=None):
    """dx [batch][k] = dy [batch][n] @ W (tern_gemv_t, the STE-backward input gradient), batch <= 8."""
    torch = _torch()
    if dy.dim() == 1:
        dy = dy.unsqueeze(0)
    dy = dy.contiguous()
    batch = dy.shape[0]
    if dx is None:
        dx = torch.empty((batch, W.k), dtype=torch.float16, device=dy.device)
    c = W.c()
    if workspace is None:
        nb = int(lib().tern_gemv_t_workspace_bytes(ctypes.byref(c), batch))
        workspace = torch.empty(nb, dtype=torch.uint8, device=dy.device) if nb else None
    wsb = workspace.numel() if workspace is not None else 0
    st = lib().tern_gemv_t(ctypes.byref(c), _ptr(dy), batch, _ptr(dx), _ptr(workspace), wsb, _stream_handle())
    _check(st, "tern_gemv_t")
    return dx


def hadamard_rotate(x, signs, y=None):
    """y = R x per 1024-block of every row, R = H S / 32 (tern_hadamard_rotate); x fp16 [batch][k] or
    [k], signs int8 [1024] on the device (negative = -1). y may be x itself (in place)."""
    torch = _torch()
    squeeze = x.dim() == 1
    x2 = (x.unsqueeze(0) if squeeze else x).contiguous()
    if y is None:
        y = torch.empty_like(x2)
    elif squeeze:
        y = y.view(1, -1)
    st = lib().tern_hadamard_rotate(_ptr(x2), x2.shape[0], x2.shape[1], _ptr(signs), _ptr(y), _stream_handle())
    _check(st, "tern_hadamard_rotate")
    return y[0] if squeeze else y


def gemm(W: TernMatrix, X, Y=None, status=None):
    """Y [m][n] = X [m][k] @ W^T on tcgen05 tensor cores (tern_gemm)."""
    torch = _torch()
    X = X.contiguous()
    m = X.shape[0]
    if Y is None:
        Y = torch.empty((m, W.n), dtype=torch.float16, device=X.device)
    c = W.c()
    st = lib().tern_gemm(ctypes.byref(c), _ptr(X), m, _ptr(Y), _ptr(status), _stream_handle())
    _check(st, "tern_gemm")
    return Y
