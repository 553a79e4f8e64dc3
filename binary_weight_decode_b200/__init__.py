"""Python binding of libbisco (binary-weight decode GEMV for B200).

Argument marshalling only: every step of the computation runs in the CUDA
library. PyTorch provides device memory and streams. Importing this package
fails loudly if ``libbisco.so`` has not been built
(``python binary_weight_decode_b200/build.py``).

The functions carry the names of the C entry points in ``include/bisco.h``.
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbisco.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python binary_weight_decode_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

BISCO_OK, BISCO_ERR_INVALID_ARG, BISCO_ERR_UNSUPPORTED, BISCO_ERR_CUDA, BISCO_ERR_TIMEOUT, BISCO_ERR_WORKSPACE = range(6)
BISCO_F32, BISCO_BF16 = 0, 1

BISCO_PATH_AUTO, BISCO_PATH_LOOKUP_TABLE, BISCO_PATH_SMALL_BATCH_ONLY, BISCO_PATH_INTEGER_MMA = 0, 1, 2, 3
(BISCO_KERNEL_LUT_WARP, BISCO_KERNEL_LUT_STREAM, BISCO_KERNEL_LUT_ROWS, BISCO_KERNEL_INTEGER_MMA,
 BISCO_KERNEL_TENSOR_CORE, BISCO_KERNEL_REFINE) = 1, 2, 3, 4, 5, 6

EXPORTED = [
    "bisco_packed_words", "bisco_pack", "bisco_unpack", "bisco_workspace_size", "bisco_workspace_init",
    "bisco_gemv", "bisco_sync_status", "bisco_bench", "bisco_status_string", "bisco_gemv_noalloc",
    "bisco_set_path_policy", "bisco_plan_kernels", "bisco_debug_set_wait_test",
    "bisco_fluxbin_signs", "bisco_biloco_workspace_size", "bisco_biloco_decompose",
    "bisco_group_workspace_size", "bisco_gemv_group", "bisco_plan_group_kernels",
]


class bisco_layer(ctypes.Structure):
    _fields_ = [
        ("out", ctypes.c_int32), ("in_", ctypes.c_int32), ("num_bases", ctypes.c_int32),
        ("bits", ctypes.c_void_p), ("row_scale", ctypes.c_void_p), ("col_scale", ctypes.c_void_p),
        ("scale_dtype", ctypes.c_int32), ("rank", ctypes.c_int32),
        ("v_bits", ctypes.c_void_p), ("ut_bits", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
        ("n_sal", ctypes.c_int32), ("sal_stride", ctypes.c_int32),
        ("sal_idx", ctypes.c_void_p), ("sal_q", ctypes.c_void_p), ("sal_scale", ctypes.c_void_p),
        ("row_group", ctypes.c_int32),
        ("ref_bases", ctypes.c_int32), ("n_ref", ctypes.c_int32), ("ref_idx", ctypes.c_void_p),
        ("ref_bits", ctypes.c_void_p), ("ref_row_scale", ctypes.c_void_p), ("ref_col_scale", ctypes.c_void_p),
    ]


class bisco_bench_args(ctypes.Structure):
    _fields_ = [
        ("layers", ctypes.POINTER(bisco_layer)), ("n_layers", ctypes.c_int32),
        ("X", ctypes.c_void_p), ("x_dtype", ctypes.c_int32), ("M", ctypes.c_int32),
        ("Y", ctypes.c_void_p), ("y_dtype", ctypes.c_int32),
        ("ws", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t),
        ("warmup", ctypes.c_int32), ("reps", ctypes.c_int32), ("stream", ctypes.c_void_p),
    ]


class bisco_bench_result(ctypes.Structure):
    _fields_ = [("us_per_gemv", ctypes.c_double), ("us_per_replay", ctypes.c_double),
                ("kernels_per_gemv", ctypes.c_int32)]


_P = ctypes.c_void_p
_lib.bisco_packed_words.argtypes = [ctypes.c_int64, ctypes.c_int64]
_lib.bisco_packed_words.restype = ctypes.c_int64
_lib.bisco_pack.argtypes = [_P, ctypes.c_int64, ctypes.c_int64, _P]
_lib.bisco_pack.restype = ctypes.c_int
_lib.bisco_unpack.argtypes = [_P, ctypes.c_int64, ctypes.c_int64, _P]
_lib.bisco_unpack.restype = ctypes.c_int
_lib.bisco_workspace_size.argtypes = [ctypes.POINTER(bisco_layer), ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
_lib.bisco_workspace_size.restype = ctypes.c_int
_lib.bisco_workspace_init.argtypes = [_P, ctypes.c_size_t, _P]
_lib.bisco_workspace_init.restype = ctypes.c_int
_lib.bisco_gemv.argtypes = [ctypes.POINTER(bisco_layer), _P, ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int32,
                            _P, ctypes.c_size_t, _P]
_lib.bisco_gemv.restype = ctypes.c_int
_lib.bisco_gemv_noalloc.argtypes = [ctypes.POINTER(bisco_layer), _P, ctypes.c_int32, ctypes.c_int32, _P,
                                    ctypes.c_int32, _P]
_lib.bisco_gemv_noalloc.restype = ctypes.c_int
_lib.bisco_sync_status.argtypes = [_P, _P]
_lib.bisco_sync_status.restype = ctypes.c_int
_lib.bisco_bench.argtypes = [ctypes.POINTER(bisco_bench_args), ctypes.POINTER(bisco_bench_result)]
_lib.bisco_bench.restype = ctypes.c_int
_lib.bisco_status_string.argtypes = [ctypes.c_int]
_lib.bisco_status_string.restype = ctypes.c_char_p
_lib.bisco_set_path_policy.argtypes = [ctypes.c_int32]
_lib.bisco_set_path_policy.restype = ctypes.c_int
_lib.bisco_plan_kernels.argtypes = [ctypes.POINTER(bisco_layer), ctypes.c_int32, ctypes.c_int32, ctypes.c_size_t,
                                    ctypes.POINTER(ctypes.c_int32), ctypes.c_int32]
_lib.bisco_plan_kernels.restype = ctypes.c_int32
_lib.bisco_debug_set_wait_test.argtypes = [ctypes.c_int32, ctypes.c_uint64]
_lib.bisco_debug_set_wait_test.restype = ctypes.c_int
_lib.bisco_group_workspace_size.argtypes = [ctypes.POINTER(bisco_layer), ctypes.c_int32, ctypes.c_int32,
                                            ctypes.POINTER(ctypes.c_size_t)]
_lib.bisco_group_workspace_size.restype = ctypes.c_int
_lib.bisco_gemv_group.argtypes = [ctypes.POINTER(bisco_layer), ctypes.c_int32, _P, ctypes.c_int32, ctypes.c_int32,
                                  ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32, _P, ctypes.c_size_t, _P]
_lib.bisco_gemv_group.restype = ctypes.c_int
_lib.bisco_plan_group_kernels.argtypes = [ctypes.POINTER(bisco_layer), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_size_t, ctypes.POINTER(ctypes.c_int32), ctypes.c_int32]
_lib.bisco_plan_group_kernels.restype = ctypes.c_int32
_lib.bisco_fluxbin_signs.argtypes = [_P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, _P, _P, ctypes.c_int32, _P, _P]
_lib.bisco_fluxbin_signs.restype = ctypes.c_int
_lib.bisco_biloco_workspace_size.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                             ctypes.POINTER(ctypes.c_size_t)]
_lib.bisco_biloco_workspace_size.restype = ctypes.c_int
_lib.bisco_biloco_decompose.argtypes = [_P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P, _P,
                                        _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.bisco_biloco_decompose.restype = ctypes.c_int


class BiscoError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {bisco_status_string(status)}")


def _check(st: int, where: str):
    if st != BISCO_OK:
        raise BiscoError(st, where)


def bisco_status_string(status: int) -> str:
    return _lib.bisco_status_string(int(status)).decode()


def bisco_packed_words(rows: int, cols: int) -> int:
    return int(_lib.bisco_packed_words(rows, cols))


def bisco_pack(signs: np.ndarray) -> np.ndarray:
    """Dense int8 +1/-1 matrix (host) -> packed uint32 words (host)."""
    s = np.ascontiguousarray(signs, dtype=np.int8)
    if s.ndim != 2:
        raise ValueError("signs must be 2-D")
    rows, cols = s.shape
    out = np.empty(max(bisco_packed_words(rows, cols), 1), dtype=np.uint32)
    _check(_lib.bisco_pack(s.ctypes.data, rows, cols, out.ctypes.data), "bisco_pack")
    return out


def bisco_unpack(words: np.ndarray, rows: int, cols: int) -> np.ndarray:
    w = np.ascontiguousarray(words, dtype=np.uint32)
    if w.size < bisco_packed_words(rows, cols):
        raise ValueError("packed buffer too small")
    out = np.empty((rows, cols), dtype=np.int8)
    _check(_lib.bisco_unpack(w.ctypes.data, rows, cols, out.ctypes.data), "bisco_unpack")
    return out


# --------------------------------------------------------------------------
# device side (torch tensors for memory and streams)
# --------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BISCO_BF16
    if t.dtype == torch.float32:
        return BISCO_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream_ptr(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class DeviceLayer:
    """Uploads a host layer (numpy arrays in the packed format) and holds its device
    tensors alive together with the ``bisco_layer`` descriptor that points at them."""

    def __init__(self, host, device="cuda"):
        torch = _torch()

        def up(a, dt=None):
            if a is None:
                return None
            a = np.ascontiguousarray(a)
            if a.dtype == np.uint16:          # bf16 bit patterns
                return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
            if a.dtype == np.uint32:
                return torch.from_numpy(a.view(np.int32)).to(device)
            return torch.from_numpy(a).to(device)

        self.host = host
        self.row_group = int(getattr(host, "group", 0) or 0)
        self.out, self.in_, self.K = host.out, host.in_, host.K
        self.rank, self.n_sal = host.rank, host.n_sal
        self.bits = up(host.bits) if host.K else None
        rs = host.row_scale
        if host.K and self.row_group:  # host [K][out][groups] -> device [K][groups][out]
            rs = np.ascontiguousarray(np.asarray(rs).reshape(host.K, host.out, -1).transpose(0, 2, 1))
        self.row_scale = up(rs) if host.K else None
        self.col_scale = up(host.col_scale) if host.K else None
        self.v_bits = up(host.v_bits)
        self.ut_bits = up(host.ut_bits)
        self.alpha = up(host.alpha)
        self.sal_idx = up(host.sal_idx)
        self.sal_q = up(host.sal_q)
        self.sal_scale = up(host.sal_scale)
        self.ref_K = int(getattr(host, "ref_K", 0) or 0)
        self.n_ref = len(host.ref_idx) if self.ref_K else 0
        self.ref_idx = self.ref_bits = self.ref_row_scale = self.ref_col_scale = None
        if self.ref_K:
            self.ref_idx = up(np.asarray(host.ref_idx, dtype=np.int32))
            self.ref_bits = up(host.ref_bits)
            # host [Ks][out][groups] -> device [Ks][groups][out], like the global row scales
            self.ref_row_scale = up(np.ascontiguousarray(
                np.asarray(host.ref_row_scale).reshape(self.ref_K, host.out, -1).transpose(0, 2, 1)))
            self.ref_col_scale = up(host.ref_col_scale)
        ptr = lambda t: (t.data_ptr() if t is not None else None)  # noqa: E731
        self.desc = bisco_layer(
            out=host.out, in_=host.in_, num_bases=host.K,
            bits=ptr(self.bits), row_scale=ptr(self.row_scale), col_scale=ptr(self.col_scale),
            scale_dtype=BISCO_BF16 if host.scale_dtype == "bf16" else BISCO_F32,
            rank=host.rank, v_bits=ptr(self.v_bits), ut_bits=ptr(self.ut_bits), alpha=ptr(self.alpha),
            n_sal=host.n_sal, sal_stride=host.sal_stride if host.n_sal else 0,
            sal_idx=ptr(self.sal_idx), sal_q=ptr(self.sal_q), sal_scale=ptr(self.sal_scale),
            row_group=self.row_group, ref_bases=self.ref_K, n_ref=self.n_ref, ref_idx=ptr(self.ref_idx),
            ref_bits=ptr(self.ref_bits), ref_row_scale=ptr(self.ref_row_scale),
            ref_col_scale=ptr(self.ref_col_scale))

    def clone(self):
        """Another device copy of the same layer (same values, separate device buffers)."""
        c = DeviceLayer.__new__(DeviceLayer)
        c.host = self.host
        c.out, c.in_, c.K, c.rank, c.n_sal = self.out, self.in_, self.K, self.rank, self.n_sal
        c.row_group, c.ref_K, c.n_ref = self.row_group, self.ref_K, self.n_ref
        for n in ("bits", "row_scale", "col_scale", "v_bits", "ut_bits", "alpha", "sal_idx", "sal_q", "sal_scale",
                  "ref_idx", "ref_bits", "ref_row_scale", "ref_col_scale"):
            t = getattr(self, n)
            setattr(c, n, t.clone() if t is not None else None)
        ptr = lambda t: (t.data_ptr() if t is not None else None)  # noqa: E731
        d = self.desc
        c.desc = bisco_layer(
            out=d.out, in_=d.in_, num_bases=d.num_bases, bits=ptr(c.bits), row_scale=ptr(c.row_scale),
            col_scale=ptr(c.col_scale), scale_dtype=d.scale_dtype, rank=d.rank, v_bits=ptr(c.v_bits),
            ut_bits=ptr(c.ut_bits), alpha=ptr(c.alpha), n_sal=d.n_sal, sal_stride=d.sal_stride,
            sal_idx=ptr(c.sal_idx), sal_q=ptr(c.sal_q), sal_scale=ptr(c.sal_scale), row_group=d.row_group,
            ref_bases=d.ref_bases, n_ref=d.n_ref, ref_idx=ptr(c.ref_idx), ref_bits=ptr(c.ref_bits),
            ref_row_scale=ptr(c.ref_row_scale), ref_col_scale=ptr(c.ref_col_scale))
        return c

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   [self.bits, self.row_scale, self.col_scale, self.v_bits, self.ut_bits, self.alpha,
                    self.sal_idx, self.sal_q, self.sal_scale, self.ref_idx, self.ref_bits, self.ref_row_scale,
                    self.ref_col_scale] if t is not None)


def _desc(layer):
    return layer.desc if isinstance(layer, DeviceLayer) else layer


def bisco_workspace_size(layer, M: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.bisco_workspace_size(ctypes.byref(_desc(layer)), M, ctypes.byref(n)), "bisco_workspace_size")
    return int(n.value)


def bisco_workspace_init(ws, stream=None):
    _check(_lib.bisco_workspace_init(ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size(),
                                     _stream_ptr(stream)), "bisco_workspace_init")


def alloc_workspace(layers, M: int, device="cuda"):
    """Zero-initialised workspace large enough for every layer in `layers` at batch M."""
    torch = _torch()
    n = max(bisco_workspace_size(L, M) for L in layers)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    bisco_workspace_init(ws)
    return ws


def bisco_gemv(layer, X, Y, ws, stream=None):
    """Y[M, out] = X[M, in] @ W^T on the device (asynchronous on `stream`)."""
    M = X.shape[0] if X.dim() == 2 else 1
    st = _lib.bisco_gemv(ctypes.byref(_desc(layer)), ctypes.c_void_p(X.data_ptr()), _dtype_code(X), M,
                         ctypes.c_void_p(Y.data_ptr()), _dtype_code(Y), ctypes.c_void_p(ws.data_ptr()),
                         ws.numel() * ws.element_size(), _stream_ptr(stream))
    _check(st, "bisco_gemv")
    return Y


def bisco_gemv_noalloc(layer, X, Y, stream=None):
    """bisco_gemv with the library's built-in scratch array instead of a workspace."""
    M = X.shape[0] if X.dim() == 2 else 1
    st = _lib.bisco_gemv_noalloc(ctypes.byref(_desc(layer)), ctypes.c_void_p(X.data_ptr()), _dtype_code(X), M,
                                 ctypes.c_void_p(Y.data_ptr()), _dtype_code(Y), _stream_ptr(stream))
    _check(st, "bisco_gemv_noalloc")
    return Y


def bisco_sync_status(ws, stream=None) -> int:
    return int(_lib.bisco_sync_status(_stream_ptr(stream), ctypes.c_void_p(ws.data_ptr())))


def bisco_bench(layers, X, Y, ws, warmup: int = 3, reps: int = 10, stream=None) -> dict:
    arr = (bisco_layer * len(layers))(*[_desc(L) for L in layers])
    M = X.shape[0]
    args = bisco_bench_args(layers=arr, n_layers=len(layers), X=X.data_ptr(), x_dtype=_dtype_code(X), M=M,
                            Y=Y.data_ptr(), y_dtype=_dtype_code(Y), ws=ws.data_ptr(),
                            ws_bytes=ws.numel() * ws.element_size(), warmup=warmup, reps=reps,
                            stream=_stream_ptr(stream).value)
    res = bisco_bench_result()
    _check(_lib.bisco_bench(ctypes.byref(args), ctypes.byref(res)), "bisco_bench")
    return {"us_per_gemv": res.us_per_gemv, "us_per_replay": res.us_per_replay,
            "kernels_per_gemv": res.kernels_per_gemv}


def bisco_set_path_policy(policy: int):
    """Process-wide choice of kernel family (BISCO_PATH_*); see include/bisco.h."""
    _check(_lib.bisco_set_path_policy(int(policy)), "bisco_set_path_policy")


def bisco_plan_kernels(layer, M: int, x_dtype: int, ws_bytes: int) -> list:
    """Kernel kinds (BISCO_KERNEL_*) that bisco_gemv would launch, in order."""
    cap = 64
    buf = (ctypes.c_int32 * cap)()
    n = int(_lib.bisco_plan_kernels(ctypes.byref(_desc(layer)), M, x_dtype, ws_bytes, buf, cap))
    if n < 0:
        raise BiscoError(BISCO_ERR_INVALID_ARG, "bisco_plan_kernels")
    if n > cap:
        buf = (ctypes.c_int32 * n)()
        n = int(_lib.bisco_plan_kernels(ctypes.byref(_desc(layer)), M, x_dtype, ws_bytes, buf, n))
    return [int(buf[i]) for i in range(n)]


def bisco_debug_set_wait_test(skip_tile: int, wait_ns: int = 0):
    """Test hook for the integer kernel's bounded waits (skip_tile = -1 turns it off)."""
    _check(_lib.bisco_debug_set_wait_test(int(skip_tile), int(wait_ns)), "bisco_debug_set_wait_test")


def bisco_fluxbin_signs(W, row_scale, col_scale, group=0, stream=None):
    """Packed joint signs of Kb bases ([Kb, packed_words] int32 on W's device) for fp64
    device tensors W [rows, cols], row_scale [Kb, rows] (or [Kb, groups, rows] with
    group > 0) and col_scale [Kb, cols]; see include/bisco.h."""
    torch = _torch()
    rows, cols = W.shape
    Kb = col_scale.shape[0]
    for t in (W, row_scale, col_scale):
        if t.dtype != torch.float64 or not t.is_contiguous():
            raise BiscoError(BISCO_ERR_INVALID_ARG, "bisco_fluxbin_signs")
    bits = torch.empty((Kb, bisco_packed_words(rows, cols)), dtype=torch.int32, device=W.device)
    _check(_lib.bisco_fluxbin_signs(ctypes.c_void_p(W.data_ptr()), rows, cols, Kb,
                                    ctypes.c_void_p(row_scale.data_ptr()), ctypes.c_void_p(col_scale.data_ptr()),
                                    int(group), ctypes.c_void_p(bits.data_ptr()), _stream_ptr(stream)),
           "bisco_fluxbin_signs")
    return bits


def bisco_biloco_decompose(W, v0, rounds=5, stream=None):
    """Binary low-rank decomposition of an fp64 device matrix W [rows, cols] from starting
    signs v0 [rank, cols] (int8, +-1): returns U [rows, rank], V [rank, cols] (int8) and the
    greedy and refit coefficients [rank] (fp64); see include/bisco.h."""
    torch = _torch()
    rows, cols = W.shape
    rank = v0.shape[0]
    if W.dtype != torch.float64 or v0.dtype != torch.int8 or not W.is_contiguous() or not v0.is_contiguous():
        raise BiscoError(BISCO_ERR_INVALID_ARG, "bisco_biloco_decompose")
    n = ctypes.c_size_t(0)
    _check(_lib.bisco_biloco_workspace_size(rows, cols, rank, ctypes.byref(n)), "bisco_biloco_workspace_size")
    ws = torch.empty(int(n.value), dtype=torch.uint8, device=W.device)
    U = torch.empty((rows, rank), dtype=torch.int8, device=W.device)
    V = torch.empty((rank, cols), dtype=torch.int8, device=W.device)
    ag = torch.empty(rank, dtype=torch.float64, device=W.device)
    ar = torch.empty(rank, dtype=torch.float64, device=W.device)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    _check(_lib.bisco_biloco_decompose(p(W), rows, cols, rank, int(rounds), p(v0), p(U), p(V), p(ag), p(ar), p(ws),
                                       int(n.value), _stream_ptr(stream)), "bisco_biloco_decompose")
    return U, V, ag, ar


def _layer_array(layers):
    arr = (bisco_layer * len(layers))()
    for i, L in enumerate(layers):
        arr[i] = _desc(L)
    return arr


def bisco_group_workspace_size(layers, M: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.bisco_group_workspace_size(_layer_array(layers), len(layers), M, ctypes.byref(n)),
           "bisco_group_workspace_size")
    return int(n.value)


def alloc_group_workspace(layers, M: int, device="cuda"):
    """Zero-initialised workspace for bisco_gemv_group over `layers` at batch M."""
    torch = _torch()
    ws = torch.empty(bisco_group_workspace_size(layers, M), dtype=torch.uint8, device=device)
    bisco_workspace_init(ws)
    return ws


def bisco_gemv_group(layers, X, Ys, ws, stream=None):
    """Ys[j][M, out_j] = X[M, in] @ W_j^T for layers sharing X, in one call."""
    M = X.shape[0] if X.dim() == 2 else 1
    ptrs = (ctypes.c_void_p * len(Ys))(*[y.data_ptr() for y in Ys])
    ydt = _dtype_code(Ys[0])
    if any(_dtype_code(y) != ydt for y in Ys):
        raise BiscoError(BISCO_ERR_INVALID_ARG, "bisco_gemv_group")
    _check(_lib.bisco_gemv_group(_layer_array(layers), len(layers), ctypes.c_void_p(X.data_ptr()), _dtype_code(X), M,
                                 ptrs, ydt, ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size(),
                                 _stream_ptr(stream)), "bisco_gemv_group")
    return Ys


def bisco_plan_group_kernels(layers, M: int, x_dtype: int, ws_bytes: int) -> list:
    cap = 256
    buf = (ctypes.c_int32 * cap)()
    n = int(_lib.bisco_plan_group_kernels(_layer_array(layers), len(layers), M, x_dtype, ws_bytes, buf, cap))
    if n < 0:
        raise BiscoError(BISCO_ERR_INVALID_ARG, "bisco_plan_group_kernels")
    return [int(buf[i]) for i in range(min(n, cap))]
