"""Host-side checks of the C ABI that need no GPU: the library builds and loads,
exports every entry point the header declares, and rejects bad arguments on
the host before anything is enqueued."""
import ctypes
import os
import re

import pytest

import quantization_grouped_gemm_b200 as qgg
from quantization_grouped_gemm_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8qgg.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w ]*?[\s\*]+(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return qgg.lib()


def test_header_declares_the_three_entry_points():
    names = declared_functions()
    for n in ("fp8_quant_rowwise", "fp8_quant_colwise_jagged", "fp8_scaled_grouped_gemm"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    # and the binding knows the signature of each
    assert set(names) <= set(qgg._SIGNATURES)


def test_library_is_built_for_sm100a():
    qbuild.build()
    assert "arch=compute_100a,code=sm_100a" in qbuild.ARCH
    assert os.path.exists(qbuild.LIB)


def test_unit_wait_test_hook_checks_its_limit(lib):
    """The failure-detection hook never allows a wait longer than the normal
    2 s limit, and (0, 0) restores normal calls."""
    assert lib.fp8qgg_test_unit_wait(1, 3_000_000_000) == -4
    assert lib.fp8qgg_test_unit_wait(0, 0) == 0


def test_native_format_and_error_strings(lib):
    assert lib.fp8_native_format() == qgg.E4M3FN
    for rc in (0, -1, -2, -3, -4, -5):
        assert lib.fp8qgg_error_string(rc)
    assert lib.fp8qgg_error_string(-99) == b"unknown error"


FAKE = ctypes.c_void_p(1 << 20)  # 16-byte-aligned non-null value, never dereferenced on these paths
ODD = ctypes.c_void_p((1 << 20) + 4)


def test_rowwise_argument_checks(lib):
    f = lib.fp8_quant_rowwise
    assert f(None, 4, 64, 64, FAKE, 64, FAKE, 0, 0.0, None, None) == -1
    assert f(FAKE, 4, 0, 64, FAKE, 64, FAKE, 0, 0.0, None, None) == -2
    assert f(FAKE, 4, 64, 32, FAKE, 64, FAKE, 0, 0.0, None, None) == -2
    assert f(FAKE, 4, 40000, 40000, FAKE, 40000, FAKE, 0, 0.0, None, None) == -2
    assert f(FAKE, 4, 60, 64, FAKE, 64, FAKE, 0, 0.0, None, None) == -3
    assert f(ODD, 4, 64, 64, FAKE, 64, FAKE, 0, 0.0, None, None) == -3
    assert f(FAKE, 4, 64, 64, FAKE, 64, FAKE, 7, 0.0, None, None) == -4
    assert f(FAKE, 4, 64, 64, FAKE, 64, FAKE, 0, -1.0, None, None) == -4
    assert f(FAKE, 0, 64, 64, FAKE, 64, FAKE, 0, 0.0, None, None) == 0  # empty: no-op


def test_colwise_noalloc_refuses_problems_beyond_its_scratch(lib):
    # the size check runs on the host before any device access
    f = lib.fp8_quant_colwise_jagged_noalloc
    big = (98304, 8192, 64)
    assert lib.fp8_quant_colwise_jagged_workspace_size(*big) > 2 * 1024 * 1024
    assert f(FAKE, big[0], big[1], big[1], FAKE, big[2], FAKE, big[1], 0, FAKE, 0, 0.0, None,
             None, None) == -2


def test_colwise_argument_checks(lib):
    f = lib.fp8_quant_colwise_jagged
    ws = lib.fp8_quant_colwise_jagged_workspace_size(100, 64, 4)
    assert ws > 0 and ws % 256 == 0
    # the larger of the two kernels' needs.  Plain layouts: tall units (over
    # 448 rows) each need an arrival counter and 64 absmax words; at most
    # min(groups, rows / 432) groups can be that tall.  Padded layout: one
    # arrival counter per (group, 256-column panel) and one absmax word per
    # (group, column).  Each part is rounded up to 256 bytes.
    g = lib.fp8_quant_colwise_jagged_workspace_size

    def r256(b):
        return (b + 255) // 256 * 256

    def plain(rows, cols, e):
        units = min(e, rows // 432) * ((cols + 63) // 64)
        return 256 + r256(4 * units) + 256 * units

    def padded(rows, cols, e):
        return 256 + r256(4 * e * ((cols + 255) // 256)) + r256(4 * e * cols)

    for args in ((431, 64, 4), (432, 64, 4), (98304, 2048, 64), (98304, 2048, 1000),
                 (98304, 1408, 64), (5, 8, 1)):
        assert g(*args) == max(plain(*args), padded(*args)), args
    assert g(98304, 2048, 64) == 256 + 2048 * 4 + 2048 * 256  # the plain kernel's need
    assert g(431, 64, 4) == 256 + 256 + 4 * 4 * 64          # the padded kernel's need
    d = lib.fp8_quant_dual_jagged_workspace_size
    assert d(98304, 1408, 64) == padded(98304, 1408, 64) + r256(4 * 98304)

    def call(**kw):
        a = dict(x=FAKE, rows=100, cols=64, ld_x=64, off=FAKE, e=4, q=FAKE, ld_q=64, layout=0,
                 s=FAKE, fmt=0, smax=0.0, sat=None, st=None, ws=FAKE, wsb=ws)
        a.update(kw)
        return f(a["x"], a["rows"], a["cols"], a["ld_x"], a["off"], a["e"], a["q"], a["ld_q"],
                 a["layout"], a["s"], a["fmt"], a["smax"], a["sat"], a["st"], a["ws"], a["wsb"],
                 None)

    assert call(x=None) == -1
    assert call(off=None) == -1
    assert call(ws=None) == -1
    assert call(e=0) == -2
    assert call(e=2000) == -2
    assert call(wsb=ws - 1) == -2
    assert call(layout=1, ld_q=64) == -2       # transposed needs ld_q >= rows_total
    assert call(layout=1, ld_q=104) == -3      # and ld_q % 16 == 0
    assert call(cols=60, ld_x=64) == -3
    # padded transposed: room for every group rounded up to 128 tokens
    assert call(layout=2, ld_q=112) == -2
    assert call(layout=2, ld_q=100 + 128 * 4 - 16) == -2
    assert call(layout=2, ld_q=100 + 128 * 4 + 8) == -3
    assert call(layout=5) == -4
    assert call(fmt=3) == -4


def test_gemm_argument_checks(lib):
    f = lib.fp8_scaled_grouped_gemm

    def call(**kw):
        a = dict(mode=0, a=FAKE, lda=64, sa=FAKE, sas=0, b=FAKE, ldb=64, bgs=64 * 32, sb=FAKE,
                 sbs=32, off=FAKE, e=2, m=100, n=32, k=64, out=FAKE, ldo=32, ogs=0, odt=0, fmt=0)
        a.update(kw)
        return f(a["mode"], a["a"], a["lda"], a["sa"], a["sas"], a["b"], a["ldb"], a["bgs"],
                 a["sb"], a["sbs"], a["off"], a["e"], a["m"], a["n"], a["k"], a["out"], a["ldo"],
                 a["ogs"], a["odt"], a["fmt"], None, None)

    assert call(fmt=1) == -4           # no e4m3fnuz input on the tensor cores
    assert call(mode=3) == -4
    assert call(odt=3) == -4
    assert call(e=0) == -2
    assert call(e=1025) == -2
    assert call(lda=32) == -2
    assert call(bgs=64) == -2          # groups of B overlap
    assert call(a=None) == -1
    assert call(lda=72) == -3          # leading dimension not a multiple of 16
    assert call(n=30, ldo=32, sbs=32) == -3
    assert call(a=ODD) == -3
    # K-jagged: token axis is the leading dimension of both operands
    assert call(mode=1, lda=64, ldb=64, m=100, sas=32, sbs=64, ldo=64, ogs=32 * 64) == -2
    assert call(mode=1, lda=112, ldb=112, m=100, sas=32, sbs=64, ldo=64, ogs=16) == -2
    # padded operands: the token axis holds up to 128 more columns per group
    assert call(mode=2, lda=112, ldb=112, m=100, sas=32, sbs=64, ldo=64, ogs=32 * 64) == -2
    assert call(mode=2, lda=352, ldb=368, m=100, sas=32, sbs=64, ldo=64, ogs=32 * 64) == -2


def test_cast_argument_checks(lib):
    f = lib.fp8_cast_f32
    assert f(FAKE, -1, FAKE, 0, None) == -2
    assert f(FAKE, 4, FAKE, 2, None) == -4
    assert f(None, 4, FAKE, 0, None) == -1
    assert f(FAKE, 0, FAKE, 0, None) == 0


def test_binding_refuses_host_tensors_instead_of_computing_on_the_cpu():
    """There is no CPU or torch fallback: every entry point of the binding
    raises on host tensors before anything is computed."""
    import torch
    x = torch.zeros((4, 8), dtype=torch.bfloat16)
    off = torch.tensor([4], dtype=torch.int32)
    q8 = torch.zeros((4, 8), dtype=torch.uint8)
    s = torch.ones(4, dtype=torch.float32)
    calls = [
        lambda: qgg.fp8_quant_rowwise(x),
        lambda: qgg.fp8_quant_colwise_jagged(x, off),
        lambda: qgg.fp8_quant_colwise_jagged(x, off, qgg.LAYOUT_TRANSPOSED_PADDED),
        lambda: qgg.fp8_scaled_grouped_gemm(qgg.M_JAGGED, q8, s, q8.view(1, 4, 8),
                                            s.view(1, 4), off),
        lambda: qgg.fp8_scaled_grouped_gemm(qgg.K_JAGGED_PADDED, q8, s.view(1, 4), q8,
                                            s.view(1, 4), off, m_total=4),
        lambda: qgg.fp8_cast_f32(torch.zeros(8)),
        lambda: qgg.fp8_mx_quant_rowwise(torch.zeros((4, 32), dtype=torch.bfloat16)),
        lambda: qgg.fp8_mx_quant_colwise_padded(x, off),
        lambda: qgg.fp8_mx_quant_dual_padded(torch.zeros((4, 32), dtype=torch.bfloat16), off),
        lambda: qgg.fp8_mx_grouped_gemm(qgg.M_JAGGED, q8, q8, q8.view(1, 4, 8),
                                        q8.view(1, 4, 8), off),
    ]
    for f in calls:
        with pytest.raises(ValueError, match="CUDA tensors only"):
            f()


def test_mx_quant_argument_checks(lib):
    r = lib.fp8_mx_quant_rowwise

    def row(**kw):
        a = dict(x=FAKE, rows=10, cols=64, ldx=64, q=FAKE, ldq=64, s=FAKE, ldsw=10)
        a.update(kw)
        return r(a["x"], a["rows"], a["cols"], a["ldx"], a["q"], a["ldq"], a["s"], a["ldsw"],
                 None)

    assert row(cols=48, ldx=48, ldq=48) == -2   # not whole 32-element blocks
    assert row(ldsw=9) == -2                    # one scale word per row and group
    assert row(ldx=32) == -2
    assert row(x=None) == -1
    assert row(s=None) == -1
    assert row(ldx=68) == -3                    # 16-byte rows
    assert row(q=ODD) == -3
    assert row(s=ctypes.c_void_p((1 << 20) + 2)) == -3
    assert row(rows=0) == 0                     # nothing to do
    c = lib.fp8_mx_quant_colwise_padded

    def col(**kw):
        a = dict(x=FAKE, rows=100, cols=64, ldx=64, off=FAKE, e=2, q=FAKE, ldq=368, s=FAKE,
                 ldsw=64)
        a.update(kw)
        return c(a["x"], a["rows"], a["cols"], a["ldx"], a["off"], a["e"], a["q"], a["ldq"],
                 a["s"], a["ldsw"], None, None)

    assert col(ldq=352) == -2                   # rows + 128 per group = 356 tokens
    assert col(ldsw=63) == -2                   # one word per column and token group
    assert col(ldq=360) == -3                   # 16-byte token rows
    assert col(e=0) == -2
    assert col(e=1025) == -2
    assert col(cols=60, ldx=64, ldsw=64) == -3
    assert col(off=None) == -1
    assert col(s=ctypes.c_void_p((1 << 20) + 2)) == -3


def test_mx_gemm_argument_checks(lib):
    f = lib.fp8_mx_grouped_gemm

    def call(**kw):
        a = dict(mode=0, a=FAKE, lda=256, sa=FAKE, ldsa=100, b=FAKE, ldb=256, bgs=256 * 32,
                 sb=FAKE, ldsb=64, sbgs=32, off=FAKE, e=2, m=100, n=32, k=256, out=FAKE, ldo=32,
                 ogs=0, odt=0)
        a.update(kw)
        return f(a["mode"], a["a"], a["lda"], a["sa"], a["ldsa"], a["b"], a["ldb"], a["bgs"],
                 a["sb"], a["ldsb"], a["sbgs"], a["off"], a["e"], a["m"], a["n"], a["k"],
                 a["out"], a["ldo"], a["ogs"], a["odt"], None, None)

    assert call(mode=1) == -4          # plain contraction-jagged: blocks could hold two groups
    assert call(odt=3) == -4
    assert call(k=240, lda=256, ldb=256) == -2   # whole 32-element blocks only
    assert call(ldsa=99) == -2         # one scale word per row of A and group
    assert call(sbgs=31) == -2         # the experts' scale rows of B overlap
    assert call(ldsb=63) == -2         # two experts of 32 rows
    assert call(bgs=256 * 31) == -2
    assert call(e=0) == -2
    assert call(sa=None) == -1
    assert call(sa=ctypes.c_void_p((1 << 20) + 2)) == -3
    assert call(m=0) == 0              # token-jagged with no rows: nothing to write
    # padded contraction-jagged: tokens + 128 per group on both operands
    kw = dict(mode=2, lda=368, ldb=368, ldsa=32, ldsb=64, n=32, k=64, ldo=64, ogs=32 * 64)
    assert call(**dict(kw, lda=352)) == -2
    assert call(**dict(kw, ldsa=31)) == -2
    assert call(**dict(kw, ldsb=63)) == -2
    assert call(**dict(kw, ogs=16)) == -2


def test_mx_dual_argument_checks(lib):
    f = lib.fp8_mx_quant_dual_padded

    def call(**kw):
        a = dict(x=FAKE, rows=100, cols=64, ldx=64, off=FAKE, e=2, qr=FAKE, ldqr=64, sr=FAKE,
                 ldswr=100, qc=FAKE, ldqc=368, sc=FAKE, ldswc=64)
        a.update(kw)
        return f(a["x"], a["rows"], a["cols"], a["ldx"], a["off"], a["e"], a["qr"], a["ldqr"],
                 a["sr"], a["ldswr"], a["qc"], a["ldqc"], a["sc"], a["ldswc"], None, None)

    assert call(qr=None) == -1
    assert call(sr=None) == -1
    assert call(cols=48, ldx=48, ldqr=48, ldswc=48) == -2   # rowwise blocks of 32 columns
    assert call(ldswr=99) == -2                              # one scale word per row
    assert call(ldqr=56) == -2
    assert call(ldqr=68) == -3
    assert call(qr=ctypes.c_void_p((1 << 20) + 4)) == -3
    assert call(ldqc=352) == -2                              # as the column-wise call
    assert call(rows=0, ldswr=0) == 0
