"""CPU checks of the C ABI: the library loads, exports every entry point
include/s12.h declares, and its host-side logic (argument checks, closed
forms) behaves without touching a GPU."""
import ctypes as C
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "s12.h")


@pytest.fixture(scope="module")
def lib():
    from decode_split12_b200 import build, s12
    if not build.up_to_date():
        build.build()
    return s12.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(s12_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("s12_encode", "s12_decode", "s12_gemv", "s12_gemm_skinny", "s12_stats", "s12_open"):
        assert required in names


HELPERS = ("s12_error_string", "s12_device_check")


def declaration_comments():
    """(name, the comment block right before its declaration) for every
    function the header declares, in order."""
    text = open(HEADER).read()
    out = []
    for m in re.finditer(r"\n(?:const )?[a-z_0-9]+ \*?(s12_[a-z0-9_]+)\(", text):
        before = text[:m.start()].rstrip()
        comment = ""
        if before.endswith("*/"):
            comment = before[before.rfind("/*"):]
        elif before.endswith(";"):
            # a declaration that shares the comment of the one before it
            prev = before[:before.rfind("\n")].rstrip()
            if prev.endswith("*/"):
                comment = prev[prev.rfind("/*"):]
        out.append((m.group(1), comment))
    return out


def test_every_entry_point_cites_its_passage():
    """Every entry point except the status and device helpers and the
    workspace-size queries names the page and section it follows (a
    "Follows:" line citing [W], [M] or [T]) or states that the pages have no
    counterpart."""
    decls = declaration_comments()
    assert {n for n, _ in decls} == set(declared_functions())
    for name, comment in decls:
        if name in HELPERS or name.endswith("_ws_bytes"):
            continue
        assert comment, f"{name} has no comment"
        cited = "Follows:" in comment and re.search(r"\[(W|M|T)\]", comment)
        assert cited or "no counterpart" in comment, f"{name} cites no passage"


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in s12.h but not exported"


def test_binding_lists_every_symbol():
    from decode_split12_b200 import s12
    assert set(declared_functions()) == set(s12.EXPORTED)


def test_error_strings(lib):
    from decode_split12_b200 import s12
    for code in range(0, 8):
        assert lib.s12_error_string(code)
    assert b"CORRUPT" in lib.s12_error_string(s12.S12_ERR_CORRUPT)
    assert b"unknown" in lib.s12_error_string(99)


@pytest.mark.parametrize("rows,cols,n_esc", [(1, 128, 0), (3, 256, 7), (4096, 4096, 4000), (7, 1152, 1),
                                             (28672, 8192, 117000), (1024, 4096, 0)])
def test_container_bytes_match_oracle(lib, oracle, rows, cols, n_esc):
    assert lib.s12_container_bytes(rows, cols, n_esc) == oracle.container_bytes(rows, cols, n_esc)


def test_container_bytes_rejects_bad_shapes(lib):
    assert lib.s12_container_bytes(4, 100, 0) == 0
    assert lib.s12_container_bytes(0, 128, 0) == 0
    assert lib.s12_container_bytes(-1, 128, 0) == 0


def test_workspace_sizes(lib):
    assert lib.s12_encode_ws_bytes(4096, 4096) >= 16 + 4 * (4096 * 32 // 32)
    assert lib.s12_encode_ws_bytes(4096, 4096) % 256 == 0
    assert lib.s12_encode_ws_bytes(4, 100) == 0
    assert lib.s12_stats_ws_bytes() == 2048


def test_argument_checks_need_no_device(lib):
    from decode_split12_b200 import s12
    nbytes = C.c_size_t(0)
    # null weights / size pointer
    assert lib.s12_encode(None, 4, 128, None, 0, C.byref(nbytes), None, 0, None) == s12.S12_ERR_ARG
    # bad column count is a shape error before any device work
    fake = C.c_void_p(0x1000)
    assert lib.s12_encode(fake, 4, 100, None, 0, C.byref(nbytes), fake, 1 << 20, None) == s12.S12_ERR_SHAPE
    # misaligned pointers
    bad = C.c_void_p(0x1001)
    assert lib.s12_encode(bad, 4, 128, None, 0, C.byref(nbytes), fake, 1 << 20, None) == s12.S12_ERR_ALIGN
    # an empty view
    v = s12.View()
    assert lib.s12_decode(C.byref(v), fake, None, None) == s12.S12_ERR_ARG
    assert lib.s12_gemv(C.byref(v), fake, 1, fake, fake, 1 << 20, None, None) == s12.S12_ERR_ARG
    # batch out of range on an otherwise well-formed view
    v.rows, v.cols, v.n_tiles = 4, 128, 4
    for f in ("container", "raw", "code", "base", "esc_off", "esc"):
        setattr(v, f, 0x100000)
    v.version = 1
    assert lib.s12_gemv(C.byref(v), fake, 0, fake, fake, 1 << 20, None, None) == s12.S12_ERR_SHAPE
    assert lib.s12_gemv(C.byref(v), fake, 9, fake, fake, 1 << 20, None, None) == s12.S12_ERR_SHAPE
    # the GEMV workspace is mandatory and 16-byte aligned
    assert lib.s12_gemv(C.byref(v), fake, 1, fake, None, 0, None, None) == s12.S12_ERR_ARG
    assert lib.s12_gemv(C.byref(v), fake, 1, fake, bad, 1 << 20, None, None) == s12.S12_ERR_ALIGN
    assert lib.s12_gemv_ws_bytes(C.byref(v), 0) == 0
    assert lib.s12_gemv_ws_bytes(C.byref(v), 9) == 0
    assert lib.s12_gemm_skinny(C.byref(v), fake, 8, fake, fake, 1 << 20, None, None) == s12.S12_ERR_SHAPE
    assert lib.s12_gemm_skinny(C.byref(v), fake, 257, fake, fake, 1 << 20, None, None) == s12.S12_ERR_SHAPE
    assert lib.s12_open(None, 1024, C.byref(v)) == s12.S12_ERR_ARG
    assert lib.s12_open(bad, 1024, C.byref(v)) == s12.S12_ERR_ALIGN
    assert lib.s12_open(fake, 100, C.byref(v)) == s12.S12_ERR_CORRUPT
    assert lib.s12_bf16_gemv(fake, 4, 12, fake, 1, fake, None) == s12.S12_ERR_SHAPE


def test_swiglu_and_gemm_group_argument_checks(lib):
    """The SwiGLU and grouped-GEMM entry points reject bad arguments on the
    host, before any device work: rows not a multiple of 16 for SwiGLU, an
    odd output address, more than 16 matrices, a token count above 256."""
    from decode_split12_b200 import s12
    fake = C.c_void_p(0x100000)
    v = s12.View()
    v.rows, v.cols, v.n_tiles = 24, 128, 24
    for f in ("container", "raw", "code", "base", "esc_off", "esc"):
        setattr(v, f, 0x100000)
    v.version = 1
    assert lib.s12_gemv_swiglu(C.byref(v), fake, 1, fake, fake, 1 << 20, None, None) == s12.S12_ERR_SHAPE
    v.rows, v.n_tiles = 32, 32
    odd = C.c_void_p(0x100001)
    assert lib.s12_gemv_swiglu(C.byref(v), fake, 1, odd, fake, 1 << 20, None, None) == s12.S12_ERR_ALIGN
    assert lib.s12_gemv_swiglu(C.byref(v), fake, 9, fake, fake, 1 << 20, None, None) == s12.S12_ERR_SHAPE
    assert lib.s12_gemv_swiglu(C.byref(v), fake, 1, None, fake, 1 << 20, None, None) == s12.S12_ERR_ARG
    views = (s12.View * 17)(*([v] * 17))
    xs = (C.c_void_p * 17)(*([0x100000] * 17))
    ys = (C.c_void_p * 17)(*([0x100000] * 17))
    ms = (C.c_int * 17)(*([16] * 17))
    assert lib.s12_gemm_skinny_multi(views, 17, xs, ms, ys, fake, 1 << 20, None, None) == s12.S12_ERR_ARG
    ms[1] = 257
    assert lib.s12_gemm_skinny_multi(views, 2, xs, ms, ys, fake, 1 << 20, None, None) == s12.S12_ERR_SHAPE
    assert lib.s12_gemm_multi_ws_bytes(views, 2, ms) == 0
    ms[1] = 0
    assert lib.s12_gemm_skinny_multi(views, 2, xs, ms, ys, fake, 1 << 20, None, None) == s12.S12_ERR_SHAPE


def test_interleave_gate_up_row_order():
    """Rows 16i .. 16i+7 of the interleaved matrix are gate rows 8i .. 8i+7
    and rows 16i+8 .. 16i+15 the up rows with the same indices, which is the
    pairing the SwiGLU epilogue's lanes rely on (a lane holds rows r and
    r + 8 of each 16-row group)."""
    import torch

    from decode_split12_b200 import s12
    F, K = 24, 256
    gate = torch.arange(F * K, dtype=torch.int32).reshape(F, K).to(torch.int16)
    up = (torch.arange(F * K, dtype=torch.int32).reshape(F, K) + 30000).to(torch.int16)
    wi = s12.interleave_gate_up(gate, up)
    assert wi.shape == (2 * F, K)
    for r in range(2 * F):
        grp, within = divmod(r, 16)
        src = gate if within < 8 else up
        assert torch.equal(wi[r], src[8 * grp + within % 8]), r
    with pytest.raises(ValueError):
        s12.interleave_gate_up(gate[:20], up[:20])
    with pytest.raises(ValueError):
        s12.interleave_gate_up(gate, up[:16])
