"""Thin ctypes binding of libs12.so (C ABI in include/s12.h).

Argument marshalling only: every step of the compute path runs in the CUDA
library.  torch provides device memory and streams.  The functions keep the
C names (``s12_encode``, ``s12_open``, ``s12_decode``, ``s12_gemv``,
``s12_gemm_skinny``, ``s12_stats``, ``s12_bf16_gemv``).

There is no CPU fallback: if libs12.so is missing or the device is not a
B200-class part, calls raise.
"""
from __future__ import annotations

import ctypes as C
import os
import numpy as np

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libs12.so")

S12_OK = 0
S12_ERR_ARG = 1
S12_ERR_SHAPE = 2
S12_ERR_ALIGN = 3
S12_ERR_CAPACITY = 4
S12_ERR_CORRUPT = 5
S12_ERR_CUDA = 6
S12_ERR_DEVICE = 7

S12_FLAG_ESC_COUNT = 1
S12_FLAG_ESC_RANGE = 2
S12_FLAG_BASE = 4
S12_FLAG_TIMEOUT = 8

EXPORTED = (
    "s12_error_string", "s12_device_check", "s12_container_bytes", "s12_encode_ws_bytes", "s12_encode",
    "s12_open", "s12_decode", "s12_gemv_ws_bytes", "s12_gemv", "s12_gemv_multi_ws_bytes", "s12_gemv_multi",
    "s12_gemv_noalloc", "s12_gemv_swiglu", "s12_gemv_bf16", "s12_gemm_ws_bytes", "s12_gemm_skinny",
    "s12_gemm_skinny_bf16", "s12_gemm_multi_ws_bytes",
    "s12_gemm_skinny_multi", "s12_validate_host", "s12_plane_hashes_host", "s12_fnv1a64",
    "s12_to_v2_host", "s12_from_v2_host", "s12_to_v3_host", "s12_from_v3_host", "s12_load_bf16",
    "s12_stats_ws_bytes",
    "s12_stats", "s12_bf16_gemv",
)


class S12Error(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = _lib().s12_error_string(status).decode() if _LIB is not None else str(status)
        super().__init__(f"{what}: {msg}")
        self.status = status


class View(C.Structure):
    _fields_ = [
        ("rows", C.c_uint64), ("cols", C.c_uint64), ("n_tiles", C.c_uint64), ("n_esc", C.c_uint64),
        ("container_bytes", C.c_uint64), ("container", C.c_void_p), ("raw", C.c_void_p),
        ("code", C.c_void_p), ("base", C.c_void_p), ("esc_off", C.c_void_p), ("esc", C.c_void_p),
        ("version", C.c_uint32), ("reserved", C.c_uint32), ("tmeta", C.c_void_p), ("row_esc", C.c_void_p),
        ("symtab", C.c_void_p),
    ]


class Stats(C.Structure):
    _fields_ = [
        ("rows", C.c_uint64), ("cols", C.c_uint64), ("n_tiles", C.c_uint64), ("n_esc", C.c_uint64),
        ("container_bytes", C.c_uint64), ("payload_bytes", C.c_uint64), ("header_bytes", C.c_uint64),
        ("escape_bytes", C.c_uint64), ("escape_rate", C.c_double), ("bits_per_weight", C.c_double),
        ("ratio_vs_bf16", C.c_double), ("payload_ratio", C.c_double), ("exp_entropy_bits", C.c_double),
        ("exp_hist", C.c_uint64 * 256),
    ]


_LIB = None
_P = C.c_void_p
_I64 = C.c_int64
_SZ = C.c_size_t


def _lib() -> C.CDLL:
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libs12.so not built ({LIB_PATH}); run __graft_entry__.build()")
        lib = C.CDLL(LIB_PATH)
        lib.s12_error_string.argtypes = [C.c_int]
        lib.s12_error_string.restype = C.c_char_p
        lib.s12_device_check.argtypes = []
        lib.s12_device_check.restype = C.c_int
        lib.s12_container_bytes.argtypes = [_I64, _I64, C.c_uint64]
        lib.s12_container_bytes.restype = C.c_uint64
        lib.s12_encode_ws_bytes.argtypes = [_I64, _I64]
        lib.s12_encode_ws_bytes.restype = _SZ
        lib.s12_encode.argtypes = [_P, _I64, _I64, _P, _SZ, C.POINTER(_SZ), _P, _SZ, _P]
        lib.s12_encode.restype = C.c_int
        lib.s12_open.argtypes = [_P, _SZ, C.POINTER(View)]
        lib.s12_open.restype = C.c_int
        lib.s12_decode.argtypes = [C.POINTER(View), _P, _P, _P]
        lib.s12_decode.restype = C.c_int
        lib.s12_gemv_ws_bytes.argtypes = [C.POINTER(View), C.c_int]
        lib.s12_gemv_ws_bytes.restype = _SZ
        lib.s12_gemv.argtypes = [C.POINTER(View), _P, C.c_int, _P, _P, _SZ, _P, _P]
        lib.s12_gemv_multi_ws_bytes.argtypes = [C.POINTER(View), C.c_int, C.c_int]
        lib.s12_gemv_multi_ws_bytes.restype = _SZ
        lib.s12_gemv_multi.argtypes = [C.POINTER(View), C.c_int, C.POINTER(_P), C.c_int, C.POINTER(_P), _P, _SZ, _P,
                                       _P]
        lib.s12_gemv_multi.restype = C.c_int
        lib.s12_gemv_noalloc.argtypes = [C.POINTER(View), _P, C.c_int, _P, _P, _P]
        lib.s12_gemv_noalloc.restype = C.c_int
        lib.s12_gemv_swiglu.argtypes = [C.POINTER(View), _P, C.c_int, _P, _P, _SZ, _P, _P]
        lib.s12_gemv_swiglu.restype = C.c_int
        lib.s12_gemv_bf16.argtypes = [C.POINTER(View), _P, C.c_int, _P, _P, _SZ, _P, _P]
        lib.s12_gemv_bf16.restype = C.c_int
        lib.s12_gemv.restype = C.c_int
        lib.s12_gemm_ws_bytes.argtypes = [C.POINTER(View), C.c_int]
        lib.s12_gemm_ws_bytes.restype = _SZ
        lib.s12_gemm_skinny.argtypes = [C.POINTER(View), _P, C.c_int, _P, _P, _SZ, _P, _P]
        lib.s12_gemm_skinny.restype = C.c_int
        lib.s12_gemm_skinny_bf16.argtypes = [C.POINTER(View), _P, C.c_int, _P, _P, _SZ, _P, _P]
        lib.s12_gemm_skinny_bf16.restype = C.c_int
        lib.s12_validate_host.argtypes = [_P, _SZ, C.POINTER(Report)]
        lib.s12_validate_host.restype = C.c_int
        lib.s12_plane_hashes_host.argtypes = [_P, _SZ, C.POINTER(C.c_uint64)]
        lib.s12_plane_hashes_host.restype = C.c_int
        for fn in ("s12_to_v2_host", "s12_from_v2_host", "s12_to_v3_host", "s12_from_v3_host"):
            getattr(lib, fn).argtypes = [_P, _SZ, _P, _SZ, C.POINTER(_SZ)]
            getattr(lib, fn).restype = C.c_int
        lib.s12_load_bf16.argtypes = [_P, _SZ, _P, _P, C.c_uint64, C.c_uint64, _P, _SZ, _P, _P,
                                      C.POINTER(LoadResult), _P]
        lib.s12_load_bf16.restype = C.c_int
        lib.s12_fnv1a64.argtypes = [_P, _SZ]
        lib.s12_fnv1a64.restype = C.c_uint64
        lib.s12_gemm_multi_ws_bytes.argtypes = [C.POINTER(View), C.c_int, C.POINTER(C.c_int)]
        lib.s12_gemm_multi_ws_bytes.restype = _SZ
        lib.s12_gemm_skinny_multi.argtypes = [C.POINTER(View), C.c_int, C.POINTER(_P), C.POINTER(C.c_int),
                                              C.POINTER(_P), _P, _SZ, _P, _P]
        lib.s12_gemm_skinny_multi.restype = C.c_int
        lib.s12_stats_ws_bytes.argtypes = []
        lib.s12_stats_ws_bytes.restype = _SZ
        lib.s12_stats.argtypes = [C.POINTER(View), C.POINTER(Stats), _P, _SZ, _P]
        lib.s12_stats.restype = C.c_int
        lib.s12_bf16_gemv.argtypes = [_P, _I64, _I64, _P, C.c_int, _P, _P]
        lib.s12_bf16_gemv.restype = C.c_int
        _LIB = lib
    return _LIB


def lib() -> C.CDLL:
    return _lib()


def _check(rc: int, what: str):
    if rc != S12_OK:
        raise S12Error(rc, what)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _dptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return C.c_void_p(t.data_ptr())


def _u16(t: torch.Tensor) -> torch.Tensor:
    """BF16 / int16 / uint16 tensors viewed as their 16-bit patterns."""
    if t.dtype in (torch.bfloat16, torch.int16, torch.float16):
        return t
    if t.dtype == torch.uint16:
        return t
    raise TypeError(f"expected a 16-bit tensor, got {t.dtype}")


class Container:
    """A Split12 container in device memory plus its opened view."""

    def __init__(self, blob: torch.Tensor):
        self.blob = blob
        self.view = s12_open(blob)

    @property
    def rows(self):
        return int(self.view.rows)

    @property
    def cols(self):
        return int(self.view.cols)

    @property
    def n_esc(self):
        return int(self.view.n_esc)

    @property
    def nbytes(self):
        return int(self.view.container_bytes)


def device_check():
    _check(_lib().s12_device_check(), "s12_device_check")


def s12_container_bytes(rows: int, cols: int, n_esc: int) -> int:
    return int(_lib().s12_container_bytes(rows, cols, n_esc))


def s12_encode(w: torch.Tensor, ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Encode a (rows, cols) BF16 CUDA tensor; returns the container as a
    uint8 CUDA tensor of exactly its size.  One library call with room for
    escapes of up to 1/256 of the weights (a view of the first bytes is
    returned); a matrix with more escapes takes a second call at the exact
    size the first one reported."""
    w = _u16(w)
    rows, cols = w.shape
    lib_ = _lib()
    need_ws = lib_.s12_encode_ws_bytes(rows, cols)
    if ws is None:
        ws = torch.empty(max(need_ws, 256), dtype=torch.uint8, device=w.device)
    st = _stream(stream)
    nbytes = _SZ(0)
    guess = int(lib_.s12_container_bytes(rows, cols, max(1024, rows * cols // 256)))
    blob = torch.empty(guess, dtype=torch.uint8, device=w.device)
    rc = lib_.s12_encode(_dptr(w), rows, cols, _dptr(blob), blob.numel(), C.byref(nbytes), _dptr(ws), ws.numel(),
                         st)
    if rc == S12_ERR_CAPACITY and nbytes.value > guess:
        blob = torch.empty(nbytes.value, dtype=torch.uint8, device=w.device)
        rc = lib_.s12_encode(_dptr(w), rows, cols, _dptr(blob), blob.numel(), C.byref(nbytes), _dptr(ws),
                             ws.numel(), st)
    _check(rc, "s12_encode")
    return blob[:nbytes.value]


def s12_open(blob: torch.Tensor) -> View:
    v = View()
    _check(_lib().s12_open(_dptr(blob), blob.numel() * blob.element_size(), C.byref(v)), "s12_open")
    v._blob = blob  # the view points into blob's memory: keep it alive as long as the view
    return v


def s12_decode(view: View, out: torch.Tensor | None = None, err_flag: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((view.rows, view.cols), dtype=torch.bfloat16, device="cuda")
    _check(_lib().s12_decode(C.byref(view), _dptr(out), _dptr(err_flag), _stream(stream)), "s12_decode")
    return out


def s12_gemv_ws_bytes(view: View, B: int = 1) -> int:
    return int(_lib().s12_gemv_ws_bytes(C.byref(view), B))


def gemv_workspace(view: View, B: int = 1, device=None) -> torch.Tensor:
    """A zero-filled workspace large enough for s12_gemv on `view`; the call
    leaves it zero-filled, so it can be reused by later calls on one stream."""
    need = max(s12_gemv_ws_bytes(view, B), 256)
    return torch.zeros(need, dtype=torch.uint8, device=device or "cuda")


def s12_gemv(view: View, x: torch.Tensor, y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
             err_flag: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    x = _u16(x)
    B = x.shape[0] if x.dim() == 2 else 1
    if y is None:
        y = torch.empty((B, view.rows), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = gemv_workspace(view, B, x.device)
    _check(_lib().s12_gemv(C.byref(view), _dptr(x), B, _dptr(y), _dptr(ws), ws.numel(), _dptr(err_flag),
                           _stream(stream)), "s12_gemv")
    return y


def s12_gemv_bf16(view: View, x: torch.Tensor, y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                  err_flag: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """s12_gemv with a BF16 output (round to nearest even), as int16 bits
    (B x rows)."""
    x = _u16(x)
    B = x.shape[0] if x.dim() == 2 else 1
    if y is None:
        y = torch.empty((B, view.rows), dtype=torch.int16, device=x.device)
    if ws is None:
        ws = gemv_workspace(view, B, x.device)
    _check(_lib().s12_gemv_bf16(C.byref(view), _dptr(x), B, _dptr(y), _dptr(ws), ws.numel(), _dptr(err_flag),
                                _stream(stream)), "s12_gemv_bf16")
    return y


def reset_workspace_if_timed_out(err_flag: torch.Tensor | None, *workspaces: torch.Tensor) -> bool:
    """After a call that was given `err_flag`: if the word shows
    S12_FLAG_TIMEOUT (a bounded wait inside a kernel gave up), zero the
    workspaces that call used, so that no stale arrival counter can reach
    the next call.  Reads the flag back (synchronises).  Returns True if it
    reset them."""
    if err_flag is None or not (int(err_flag.item()) & S12_FLAG_TIMEOUT):
        return False
    for ws in workspaces:
        ws.zero_()
    return True


def _view_array(views):
    arr = (View * len(views))()
    for i, v in enumerate(views):
        arr[i] = v
    return arr


def s12_gemv_multi_ws_bytes(views, B: int = 1) -> int:
    return int(_lib().s12_gemv_multi_ws_bytes(_view_array(views), len(views), B))


def s12_gemv_multi(views, xs, ys=None, ws: torch.Tensor | None = None, err_flag: torch.Tensor | None = None,
                   stream=None):
    """Several independent fused decode-GEMVs in one launch; returns the list
    of y tensors (allocated when `ys` is None)."""
    xs = [_u16(x) for x in xs]
    B = xs[0].shape[0] if xs[0].dim() == 2 else 1
    if ys is None:
        ys = [torch.empty((B, v.rows), dtype=torch.float32, device=xs[0].device) for v in views]
    arr = _view_array(views)
    if ws is None:
        need = max(int(_lib().s12_gemv_multi_ws_bytes(arr, len(views), B)), 256)
        ws = torch.zeros(need, dtype=torch.uint8, device=xs[0].device)
    xp = (_P * len(xs))(*[_dptr(x) for x in xs])
    yp = (_P * len(ys))(*[_dptr(y) for y in ys])
    _check(_lib().s12_gemv_multi(arr, len(views), xp, B, yp, _dptr(ws), ws.numel(), _dptr(err_flag),
                                 _stream(stream)), "s12_gemv_multi")
    return ys


def s12_gemv_noalloc(view: View, x: torch.Tensor, y: torch.Tensor | None = None,
                     err_flag: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """s12_gemv without a caller workspace (the library's static one)."""
    x = _u16(x)
    B = x.shape[0] if x.dim() == 2 else 1
    if y is None:
        y = torch.empty((B, view.rows), dtype=torch.float32, device=x.device)
    _check(_lib().s12_gemv_noalloc(C.byref(view), _dptr(x), B, _dptr(y), _dptr(err_flag), _stream(stream)),
           "s12_gemv_noalloc")
    return y


def interleave_gate_up(w_gate: torch.Tensor, w_up: torch.Tensor) -> torch.Tensor:
    """The row order s12_gemv_swiglu expects: F x K gate and up matrices
    (F a multiple of 8) into one 2F x K matrix whose rows 16i .. 16i+7 are
    gate rows 8i .. 8i+7 and rows 16i+8 .. 16i+15 the up rows with the same
    indices.  A one-time weight preparation, done before encoding."""
    if w_gate.shape != w_up.shape or w_gate.dim() != 2 or w_gate.shape[0] % 8:
        raise ValueError("gate and up must be F x K with F a multiple of 8")
    F, K = w_gate.shape
    return torch.stack([w_gate.reshape(F // 8, 8, K), w_up.reshape(F // 8, 8, K)], dim=1).reshape(2 * F, K)


def s12_gemv_swiglu(view: View, x: torch.Tensor, h: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                    err_flag: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """h = silu(W_gate x) * (W_up x) as BF16 bits (B x rows/2), from one
    container of interleaved gate/up rows (see interleave_gate_up)."""
    x = _u16(x)
    B = x.shape[0] if x.dim() == 2 else 1
    if h is None:
        h = torch.empty((B, view.rows // 2), dtype=torch.int16, device=x.device)
    if ws is None:
        ws = torch.zeros(max(s12_gemv_ws_bytes(view, B), 256), dtype=torch.uint8, device=x.device)
    _check(_lib().s12_gemv_swiglu(C.byref(view), _dptr(x), B, _dptr(h), _dptr(ws), ws.numel(), _dptr(err_flag),
                                  _stream(stream)), "s12_gemv_swiglu")
    return h


def s12_gemm_ws_bytes(view: View, M: int) -> int:
    return int(_lib().s12_gemm_ws_bytes(C.byref(view), M))


def s12_gemm_skinny(view: View, x: torch.Tensor, y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                    err_flag: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    x = _u16(x)
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, view.rows), dtype=torch.float32, device=x.device)
    need = s12_gemm_ws_bytes(view, M)
    if ws is None:
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=x.device)
    _check(_lib().s12_gemm_skinny(C.byref(view), _dptr(x), M, _dptr(y), _dptr(ws), ws.numel(), _dptr(err_flag),
                                  _stream(stream)), "s12_gemm_skinny")
    return y


def s12_gemm_skinny_bf16(view: View, x: torch.Tensor, y: torch.Tensor | None = None,
                         ws: torch.Tensor | None = None, err_flag: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """s12_gemm_skinny with the result rounded to BF16 (returned as int16 bits)."""
    x = _u16(x)
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, view.rows), dtype=torch.int16, device=x.device)
    need = s12_gemm_ws_bytes(view, M)
    if ws is None:
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=x.device)
    _check(_lib().s12_gemm_skinny_bf16(C.byref(view), _dptr(x), M, _dptr(y), _dptr(ws), ws.numel(),
                                       _dptr(err_flag), _stream(stream)), "s12_gemm_skinny_bf16")
    return y


def s12_stats(view: View, ws: torch.Tensor | None = None, stream=None) -> dict:
    lib_ = _lib()
    if ws is None:
        ws = torch.empty(lib_.s12_stats_ws_bytes(), dtype=torch.uint8, device="cuda")
    st = Stats()
    _check(lib_.s12_stats(C.byref(view), C.byref(st), _dptr(ws), ws.numel(), _stream(stream)), "s12_stats")
    d = {name: getattr(st, name) for name, _ in Stats._fields_ if name != "exp_hist"}
    d["exp_hist"] = list(st.exp_hist[:])
    return d


def s12_bf16_gemv(w: torch.Tensor, x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    w = _u16(w)
    x = _u16(x)
    rows, cols = w.shape
    B = x.shape[0] if x.dim() == 2 else 1
    if y is None:
        y = torch.empty((B, rows), dtype=torch.float32, device=x.device)
    _check(_lib().s12_bf16_gemv(_dptr(w), rows, cols, _dptr(x), B, _dptr(y), _stream(stream)), "s12_bf16_gemv")
    return y


def s12_gemm_multi_ws_bytes(views, Ms) -> int:
    ma = (C.c_int * len(Ms))(*[int(m) for m in Ms])
    return int(_lib().s12_gemm_multi_ws_bytes(_view_array(views), len(views), ma))


def s12_gemm_skinny_multi(views, xs, ys=None, ws: torch.Tensor | None = None, err_flag: torch.Tensor | None = None,
                          stream=None):
    """Several independent fused decode-skinny-GEMMs in one launch (each x_i
    is M_i x cols_i); returns the list of y tensors (allocated when `ys` is
    None)."""
    xs = [_u16(x) for x in xs]
    Ms = [int(x.shape[0]) for x in xs]
    if ys is None:
        ys = [torch.empty((m, v.rows), dtype=torch.float32, device=xs[0].device) for m, v in zip(Ms, views)]
    arr = _view_array(views)
    ma = (C.c_int * len(Ms))(*Ms)
    if ws is None:
        need = max(int(_lib().s12_gemm_multi_ws_bytes(arr, len(views), ma)), 256)
        ws = torch.zeros(need, dtype=torch.uint8, device=xs[0].device)
    xp = (_P * len(xs))(*[_dptr(x) for x in xs])
    yp = (_P * len(ys))(*[_dptr(y) for y in ys])
    _check(_lib().s12_gemm_skinny_multi(arr, len(views), xp, ma, yp, _dptr(ws), ws.numel(), _dptr(err_flag),
                                        _stream(stream)), "s12_gemm_skinny_multi")
    return ys


class Report(C.Structure):
    _fields_ = [("problem", C.c_uint32), ("notes", C.c_uint32), ("tile", C.c_uint64), ("n_esc_counted", C.c_uint64)]


S12_BAD_NAMES = {1: "header", 2: "size", 3: "offsets", 4: "tile_offsets", 5: "base", 6: "esc_count"}


def _host_bytes(container) -> np.ndarray:
    a = container.cpu().numpy() if isinstance(container, torch.Tensor) else np.asarray(container)
    return np.ascontiguousarray(a).view(np.uint8).reshape(-1)


def s12_validate_host(container):
    """Validate a container (host array or tensor, copied to host if needed).
    Returns (status, report) with report a dict of the first problem found."""
    b = _host_bytes(container)
    rep = Report()
    rc = _lib().s12_validate_host(b.ctypes.data_as(C.c_void_p), b.size, C.byref(rep))
    return rc, {"problem": S12_BAD_NAMES.get(rep.problem), "notes": int(rep.notes), "tile": int(rep.tile),
                "n_esc_counted": int(rep.n_esc_counted)}


def s12_plane_hashes_host(container):
    """FNV-1a 64-bit hashes of the raw, code, base, esc_off and esc planes."""
    b = _host_bytes(container)
    out = (C.c_uint64 * 5)()
    _check(_lib().s12_plane_hashes_host(b.ctypes.data_as(C.c_void_p), b.size, out), "s12_plane_hashes_host")
    return [int(v) for v in out]


def s12_fnv1a64(data: bytes) -> int:
    buf = C.create_string_buffer(bytes(data), len(data))
    return int(_lib().s12_fnv1a64(C.cast(buf, C.c_void_p), len(data)))


def _convert(fn_name: str, container) -> np.ndarray:
    b = _host_bytes(container)
    fn = getattr(_lib(), fn_name)
    n = _SZ(0)
    _check(fn(b.ctypes.data_as(C.c_void_p), b.size, None, 0, C.byref(n)), fn_name)
    out = np.zeros(n.value, np.uint8)
    _check(fn(b.ctypes.data_as(C.c_void_p), b.size, out.ctypes.data_as(C.c_void_p), out.size, C.byref(n)), fn_name)
    return out


class LoadResult(C.Structure):
    _fields_ = [("outcome", C.c_uint32), ("problem", C.c_uint32), ("hash_mismatch", C.c_uint32),
                ("device_flags", C.c_uint32)]


LOAD_OUTCOMES = {0: "decoded", 1: "fallback", 2: "rejected"}


def s12_load_bf16(container, rows: int, cols: int, dev_container, dev_out, dev_err, expected_hashes=None,
                  fallback=None, stream=None) -> dict:
    """Whole-tensor load with fallback (argument marshalling for the C call).
    container: host container bytes; expected_hashes: 5 ints or None;
    fallback: host uint16 array (rows x cols) or None; dev_container,
    dev_out (rows x cols 16-bit) and dev_err (one 32-bit word): device
    tensors, or plain integer addresses (a rejection never touches them).
    Returns the outcome ("decoded", "fallback" or "rejected") and the
    checks' findings."""
    b = _host_bytes(container)
    hashes = (C.c_uint64 * 5)(*expected_hashes) if expected_hashes is not None else None
    fb = None
    if fallback is not None:
        fb = np.ascontiguousarray(np.asarray(fallback).view(np.uint16))
        if fb.size != rows * cols:
            raise ValueError("fallback must hold rows x cols values")

    def addr(t):
        return t if isinstance(t, int) else _dptr(t)

    # an address given as an integer is taken to have room for the container
    cap_bytes = b.size if isinstance(dev_container, int) else dev_container.numel() * dev_container.element_size()
    st = _stream(stream) if (stream is not None or torch.cuda.is_available()) else None
    res = LoadResult()
    _check(_lib().s12_load_bf16(b.ctypes.data_as(C.c_void_p), b.size, hashes,
                                fb.ctypes.data_as(C.c_void_p) if fb is not None else None, rows, cols,
                                addr(dev_container), cap_bytes, addr(dev_out), addr(dev_err), C.byref(res), st),
           "s12_load_bf16")
    return {"outcome": LOAD_OUTCOMES[res.outcome], "problem": S12_BAD_NAMES.get(res.problem),
            "hash_mismatch": int(res.hash_mismatch), "device_flags": int(res.device_flags)}


def to_v2_host(container) -> np.ndarray:
    """A version 1 container (host array or tensor) as the compact version 2."""
    return _convert("s12_to_v2_host", container)


def to_v3_host(container) -> np.ndarray:
    """A version 1 container (host array or tensor) as version 3 (packed
    24-bit pairs)."""
    return _convert("s12_to_v3_host", container)


def from_v3_host(container) -> np.ndarray:
    """A version 3 container back to version 1."""
    return _convert("s12_from_v3_host", container)


def from_v2_host(container) -> np.ndarray:
    """A version 2 container back to version 1 (what the kernels read)."""
    return _convert("s12_from_v2_host", container)
