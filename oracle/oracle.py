"""ctypes wrapper around the C oracle (oracle/split12_oracle.c).

Test infrastructure only.  Every function here calls straight into the C
oracle; no arithmetic of the method is done in Python.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build_oracle

ORACLE_OK = 0
ORACLE_ERR_ARG = -1
ORACLE_ERR_SHAPE = -2
ORACLE_ERR_CAPACITY = -3
ORACLE_ERR_CORRUPT = -4


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} failed with code {code}")
        self.code = code


class OracleStats(C.Structure):
    _fields_ = [
        ("rows", C.c_uint64), ("cols", C.c_uint64), ("n_tiles", C.c_uint64), ("n_esc", C.c_uint64),
        ("container_bytes", C.c_uint64), ("payload_bytes", C.c_uint64),
        ("header_bytes", C.c_uint64), ("escape_bytes", C.c_uint64),
        ("escape_rate", C.c_double), ("bits_per_weight", C.c_double),
        ("ratio_vs_bf16", C.c_double), ("payload_ratio", C.c_double),
        ("exp_entropy_bits", C.c_double), ("exp_hist", C.c_uint64 * 256),
    ]


_P = C.c_void_p
_U64 = C.c_uint64
_I64 = C.c_int64


def _bind(lib: C.CDLL) -> C.CDLL:
    lib.oracle_container_bytes.argtypes = [_U64, _U64, _U64]
    lib.oracle_container_bytes.restype = _I64
    lib.oracle_tile_base.argtypes = [_P, _P, _P]
    lib.oracle_tile_base.restype = C.c_int
    lib.oracle_encode.argtypes = [_P, _U64, _U64, _P, _U64, _P]
    lib.oracle_encode.restype = C.c_int
    lib.oracle_decode.argtypes = [_P, _U64, _P]
    lib.oracle_decode.restype = C.c_int
    lib.oracle_decode_rows.argtypes = [_P, _U64, _P, _I64, _P]
    lib.oracle_decode_rows.restype = C.c_int
    lib.oracle_matmul_f64.argtypes = [_P, _U64, _U64, _P, _I64, _P, _P]
    lib.oracle_matmul_f64.restype = C.c_int
    lib.oracle_gemv_f64.argtypes = [_P, _U64, _P, _I64, _P, _P]
    lib.oracle_gemv_f64.restype = C.c_int
    lib.oracle_gemv_rows_f64.argtypes = [_P, _U64, _P, _I64, _P, _I64, _P, _P]
    lib.oracle_gemv_rows_f64.restype = C.c_int
    lib.oracle_container_bytes_v2.argtypes = [_U64, _U64, _U64]
    lib.oracle_container_bytes_v2.restype = _I64
    lib.oracle_encode_v2.argtypes = [_P, _U64, _U64, _P, _U64, _P]
    lib.oracle_encode_v2.restype = C.c_int
    lib.oracle_decode_v2.argtypes = [_P, _U64, _P]
    lib.oracle_decode_v2.restype = C.c_int
    lib.oracle_container_bytes_v3.argtypes = [_U64, _U64, _U64]
    lib.oracle_container_bytes_v3.restype = _I64
    lib.oracle_encode_v3.argtypes = [_P, _U64, _U64, _P, _U64, _P]
    lib.oracle_encode_v3.restype = C.c_int
    lib.oracle_decode_v3.argtypes = [_P, _U64, _P]
    lib.oracle_decode_v3.restype = C.c_int
    lib.oracle_container_bytes_v4.argtypes = [_U64, _U64, _U64]
    lib.oracle_container_bytes_v4.restype = _I64
    lib.oracle_encode_v4.argtypes = [_P, _U64, _U64, _P, _U64, _P]
    lib.oracle_encode_v4.restype = C.c_int
    lib.oracle_decode_v4.argtypes = [_P, _U64, _P]
    lib.oracle_decode_v4.restype = C.c_int
    lib.oracle_symbol_table.argtypes = [_P, _U64, _P]
    lib.oracle_symbol_table.restype = _U64
    lib.oracle_silu_mul_f64.argtypes = [_P, _P, _I64, _P]
    lib.oracle_silu_mul_f64.restype = C.c_int
    lib.oracle_stats.argtypes = [_P, _U64, _P]
    lib.oracle_stats.restype = C.c_int
    lib.oracle_bf16_to_double.argtypes = [C.c_uint16]
    lib.oracle_bf16_to_double.restype = C.c_double
    return lib


_LIB = None


def load(path: str | None = None) -> C.CDLL:
    """Load the oracle library (building it if needed).  A path loads a
    different build of the same source (used by the planted-mistake tests)."""
    global _LIB
    if path is not None:
        return _bind(C.CDLL(path))
    if _LIB is None:
        _LIB = _bind(C.CDLL(build_oracle.ensure_built()))
    return _LIB


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _check(rc: int, what: str):
    if rc != ORACLE_OK:
        raise OracleError(rc, what)


class Oracle:
    """Object form, so a test can bind a planted-mistake build."""

    def __init__(self, lib: C.CDLL | None = None):
        self.lib = lib if lib is not None else load()

    def container_bytes(self, rows: int, cols: int, n_esc: int) -> int:
        return int(self.lib.oracle_container_bytes(rows, cols, n_esc))

    def tile_base(self, tile: np.ndarray):
        t = np.ascontiguousarray(tile, dtype=np.uint16)
        assert t.size == 128
        base = np.zeros(1, np.uint32)
        inwin = np.zeros(1, np.uint32)
        n_esc = self.lib.oracle_tile_base(_ptr(t), _ptr(base), _ptr(inwin))
        if n_esc < 0:
            raise OracleError(n_esc, "tile_base")
        return int(base[0]), int(n_esc)

    def encode(self, w: np.ndarray) -> np.ndarray:
        w = np.ascontiguousarray(w, dtype=np.uint16)
        rows, cols = w.shape
        nbytes = C.c_uint64(0)
        _check(self.lib.oracle_encode(_ptr(w), rows, cols, None, 0, C.byref(nbytes)), "encode(size)")
        out = np.zeros(nbytes.value, np.uint8)
        _check(self.lib.oracle_encode(_ptr(w), rows, cols, _ptr(out), out.size, C.byref(nbytes)), "encode")
        return out

    def encode_size(self, w: np.ndarray) -> int:
        w = np.ascontiguousarray(w, dtype=np.uint16)
        nbytes = C.c_uint64(0)
        _check(self.lib.oracle_encode(_ptr(w), w.shape[0], w.shape[1], None, 0, C.byref(nbytes)), "encode(size)")
        return nbytes.value

    @staticmethod
    def shape_of(blob: np.ndarray):
        h = np.asarray(blob[:64], dtype=np.uint8)
        rows = int(h[8:16].view(np.uint64)[0])
        cols = int(h[16:24].view(np.uint64)[0])
        return rows, cols

    def decode(self, blob: np.ndarray) -> np.ndarray:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        rows, cols = self.shape_of(blob)
        out = np.zeros((rows, cols), np.uint16)
        _check(self.lib.oracle_decode(_ptr(blob), blob.size, _ptr(out)), "decode")
        return out

    def decode_rc(self, blob: np.ndarray) -> int:
        """Return code of a decode (for corruption tests)."""
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        rows, cols = self.shape_of(blob)
        n = rows * cols if 0 < rows * cols < (1 << 31) else 1
        out = np.zeros(n, np.uint16)
        return int(self.lib.oracle_decode(_ptr(blob), blob.size, _ptr(out)))

    def decode_rows(self, blob: np.ndarray, rows_idx) -> np.ndarray:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        _, cols = self.shape_of(blob)
        idx = np.ascontiguousarray(rows_idx, dtype=np.int64)
        out = np.zeros((idx.size, cols), np.uint16)
        _check(self.lib.oracle_decode_rows(_ptr(blob), blob.size, _ptr(idx), idx.size, _ptr(out)), "decode_rows")
        return out

    def matmul_f64(self, w: np.ndarray, x: np.ndarray):
        w = np.ascontiguousarray(w, dtype=np.uint16)
        x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
        rows, cols = w.shape
        m = x.shape[0]
        assert x.shape[1] == cols
        y = np.zeros((m, rows), np.float64)
        s = np.zeros((m, rows), np.float64)
        _check(self.lib.oracle_matmul_f64(_ptr(w), rows, cols, _ptr(x), m, _ptr(y), _ptr(s)), "matmul")
        return y, s

    def gemv_f64(self, blob: np.ndarray, x: np.ndarray):
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        rows, cols = self.shape_of(blob)
        x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
        m = x.shape[0]
        assert x.shape[1] == cols
        y = np.zeros((m, rows), np.float64)
        s = np.zeros((m, rows), np.float64)
        _check(self.lib.oracle_gemv_f64(_ptr(blob), blob.size, _ptr(x), m, _ptr(y), _ptr(s)), "gemv")
        return y, s

    def gemv_rows_f64(self, blob: np.ndarray, x: np.ndarray, rows_idx):
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        _, cols = self.shape_of(blob)
        x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.uint16)
        idx = np.ascontiguousarray(rows_idx, dtype=np.int64)
        m = x.shape[0]
        y = np.zeros((m, idx.size), np.float64)
        s = np.zeros((m, idx.size), np.float64)
        _check(self.lib.oracle_gemv_rows_f64(_ptr(blob), blob.size, _ptr(x), m, _ptr(idx), idx.size,
                                             _ptr(y), _ptr(s)), "gemv_rows")
        return y, s

    # -- container version 2 (compact tile header) --
    def container_bytes_v2(self, rows: int, cols: int, n_esc: int) -> int:
        return int(self.lib.oracle_container_bytes_v2(rows, cols, n_esc))

    def encode_v2(self, w: np.ndarray) -> np.ndarray:
        w = np.ascontiguousarray(w, dtype=np.uint16)
        rows, cols = w.shape
        nbytes = C.c_uint64(0)
        _check(self.lib.oracle_encode_v2(_ptr(w), rows, cols, None, 0, C.byref(nbytes)), "encode_v2 size")
        out = np.zeros(nbytes.value, np.uint8)
        _check(self.lib.oracle_encode_v2(_ptr(w), rows, cols, _ptr(out), out.size, C.byref(nbytes)), "encode_v2")
        return out

    def decode_v2(self, blob: np.ndarray) -> np.ndarray:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        rows, cols = self.shape_of(blob)
        out = np.zeros((rows, cols), np.uint16)
        _check(self.lib.oracle_decode_v2(_ptr(blob), blob.size, _ptr(out)), "decode_v2")
        return out

    def decode_v2_rc(self, blob: np.ndarray) -> int:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        rows, cols = self.shape_of(blob)
        out = np.zeros((rows, cols), np.uint16)
        return int(self.lib.oracle_decode_v2(_ptr(blob), blob.size, _ptr(out)))

    # -- container version 3 (packed 24-bit pairs) --
    def container_bytes_v3(self, rows: int, cols: int, n_esc: int) -> int:
        return int(self.lib.oracle_container_bytes_v3(rows, cols, n_esc))

    def encode_v3(self, w: np.ndarray) -> np.ndarray:
        w = np.ascontiguousarray(w, dtype=np.uint16)
        rows, cols = w.shape
        nbytes = C.c_uint64(0)
        _check(self.lib.oracle_encode_v3(_ptr(w), rows, cols, None, 0, C.byref(nbytes)), "encode_v3 size")
        out = np.zeros(nbytes.value, np.uint8)
        _check(self.lib.oracle_encode_v3(_ptr(w), rows, cols, _ptr(out), out.size, C.byref(nbytes)), "encode_v3")
        return out

    def decode_v3(self, blob: np.ndarray) -> np.ndarray:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        rows, cols = self.shape_of(blob)
        out = np.zeros((rows, cols), np.uint16)
        _check(self.lib.oracle_decode_v3(_ptr(blob), blob.size, _ptr(out)), "decode_v3")
        return out

    def decode_v3_rc(self, blob: np.ndarray) -> int:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        rows, cols = self.shape_of(blob)
        out = np.zeros((rows, cols), np.uint16)
        return int(self.lib.oracle_decode_v3(_ptr(blob), blob.size, _ptr(out)))
    def silu_mul_f64(self, g: np.ndarray, u: np.ndarray) -> np.ndarray:
        """h = silu(g) * u elementwise (the C oracle's gated-MLP activation)."""
        g = np.ascontiguousarray(g, dtype=np.float64)
        u = np.ascontiguousarray(u, dtype=np.float64)
        assert g.shape == u.shape
        h = np.zeros_like(g)
        _check(self.lib.oracle_silu_mul_f64(_ptr(g), _ptr(u), g.size, _ptr(h)), "silu_mul")
        return h

    # -- container version 4 (sign-and-exponent symbol codes) --
    def container_bytes_v4(self, rows: int, cols: int, n_esc: int) -> int:
        return int(self.lib.oracle_container_bytes_v4(rows, cols, n_esc))

    def symbol_table(self, w: np.ndarray):
        """(table of 32 u16, number of weights outside it)."""
        w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
        t = np.zeros(32, np.uint16)
        n_out = int(self.lib.oracle_symbol_table(_ptr(w), w.size, _ptr(t)))
        return t, n_out

    def encode_v4(self, w: np.ndarray) -> np.ndarray:
        w = np.ascontiguousarray(w, dtype=np.uint16)
        rows, cols = w.shape
        nbytes = C.c_uint64(0)
        _check(self.lib.oracle_encode_v4(_ptr(w), rows, cols, None, 0, C.byref(nbytes)), "encode_v4 size")
        out = np.zeros(nbytes.value, np.uint8)
        _check(self.lib.oracle_encode_v4(_ptr(w), rows, cols, _ptr(out), out.size, C.byref(nbytes)), "encode_v4")
        return out

    def decode_v4(self, blob: np.ndarray) -> np.ndarray:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        rows, cols = self.shape_of(blob)
        out = np.zeros((rows, cols), np.uint16)
        _check(self.lib.oracle_decode_v4(_ptr(blob), blob.size, _ptr(out)), "decode_v4")
        return out

    def decode_v4_rc(self, blob: np.ndarray) -> int:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        rows, cols = self.shape_of(blob)
        out = np.zeros((rows, cols), np.uint16)
        return int(self.lib.oracle_decode_v4(_ptr(blob), blob.size, _ptr(out)))

    def swiglu_f64(self, blob_gate: np.ndarray, blob_up: np.ndarray, x: np.ndarray):
        """Gated MLP input side: g = W_gate x, u = W_up x (FP64 GEMVs of two
        separate containers), h = silu(g) * u.  Returns h, g, u and the
        tolerance scales s_g, s_u (all m x F)."""
        g, s_g = self.gemv_f64(blob_gate, x)
        u, s_u = self.gemv_f64(blob_up, x)
        return self.silu_mul_f64(g, u), g, u, s_g, s_u

    def stats(self, blob: np.ndarray) -> dict:
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        st = OracleStats()
        _check(self.lib.oracle_stats(_ptr(blob), blob.size, C.byref(st)), "stats")
        d = {name: getattr(st, name) for name, _ in OracleStats._fields_ if name != "exp_hist"}
        d["exp_hist"] = np.array(st.exp_hist[:], dtype=np.uint64)
        return d

    def bf16_to_double(self, v: int) -> float:
        return float(self.lib.oracle_bf16_to_double(v))


def default() -> Oracle:
    return Oracle()


def lib_path() -> str:
    return os.path.abspath(build_oracle.ensure_built())
