"""ctypes wrapper around the plain C oracle (``fp8_oracle.c``).

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never does, and this package never touches it.

Every array crosses as numpy; bf16 tensors are passed as their raw 16-bit
patterns (``uint16``).  Each function states the passage it follows in the C
source it calls.
"""
import ctypes
import os

import numpy as np

from . import build as _build

E4M3FN = 0
E4M3FNUZ = 1
SAME = 0
TRANSPOSED = 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        i32 = ctypes.c_int32
        ci = ctypes.c_int
        f32 = ctypes.c_float
        L.oracle_fp8_decode.restype = ctypes.c_double
        L.oracle_fp8_decode.argtypes = [ctypes.c_uint8, ci]
        L.oracle_fp8_encode.restype = ctypes.c_uint8
        L.oracle_fp8_encode.argtypes = [f32, ci]
        L.oracle_fp8_encode_array.restype = None
        L.oracle_fp8_encode_array.argtypes = [P, i64, P, ci]
        L.oracle_fp8_max.restype = ctypes.c_double
        L.oracle_fp8_max.argtypes = [ci]
        L.oracle_group_bounds.restype = None
        L.oracle_group_bounds.argtypes = [P, i32, i64, P, P]
        L.oracle_quant_rowwise.restype = None
        L.oracle_quant_rowwise.argtypes = [P, i64, i64, i64, P, i64, P, ci, f32, P]
        L.oracle_quant_colwise_jagged.restype = None
        L.oracle_quant_colwise_jagged.argtypes = [P, i64, i64, i64, P, i32, P, i64, ci, P, ci,
                                                  f32, P, P, P]
        L.oracle_gemm_m_jagged_sample.restype = None
        L.oracle_gemm_m_jagged_sample.argtypes = [P, i64, P, P, i64, i64, P, i64, P, i32, i64,
                                                  i64, ci, P, P, i64, P, P, P, P]
        L.oracle_gemm_k_jagged_sample.restype = None
        L.oracle_gemm_k_jagged_sample.argtypes = [P, i64, P, i64, P, i64, P, i64, P, i32, i64,
                                                  ci, P, P, P, i64, P, P, P, P]
        L.oracle_mx_quant_rowwise.restype = None
        L.oracle_mx_quant_rowwise.argtypes = [P, i64, i64, i64, P, i64, P, i64]
        L.oracle_mx_quant_colwise_padded.restype = None
        L.oracle_mx_quant_colwise_padded.argtypes = [P, i64, i64, i64, P, i32, P, i64, P, i64,
                                                     P, P, P]
        L.oracle_mx_gemm_m_jagged_sample.restype = None
        L.oracle_mx_gemm_m_jagged_sample.argtypes = [P, i64, P, i64, P, i64, i64, P, i64, i64,
                                                     P, i32, i64, i64, P, P, i64, P, P, P, P]
        L.oracle_mx_gemm_k_jagged_padded_sample.restype = None
        L.oracle_mx_gemm_k_jagged_padded_sample.argtypes = [P, i64, P, i64, P, i64, P, i64, P,
                                                            i32, i64, P, P, P, i64, P, P, P, P,
                                                            P]
        _lib = L
    return _lib


def _p(a):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def fp8_max(fmt: int) -> float:
    return lib().oracle_fp8_max(fmt)


def decode(code: int, fmt: int) -> float:
    """Value of one e4m3 code (format definitions; NaN codes give NaN)."""
    return lib().oracle_fp8_decode(int(code), fmt)


def decode_table(fmt: int) -> np.ndarray:
    return np.array([decode(c, fmt) for c in range(256)], dtype=np.float64)


def encode(y: float, fmt: int) -> int:
    """RNE single-rounding encode of one fp32 value, saturating."""
    return int(lib().oracle_fp8_encode(float(np.float32(y)), fmt))


def encode_array(y, fmt: int) -> np.ndarray:
    """Encode every element of an fp32 array (the C encoder in a plain loop)."""
    flat = np.ascontiguousarray(np.asarray(y, dtype=np.float32).ravel())
    out = np.empty(flat.shape, dtype=np.uint8)
    lib().oracle_fp8_encode_array(_p(flat), flat.size, _p(out), fmt)
    return out.reshape(np.shape(y))


def group_bounds(offsets, rows_total: int):
    off = _c(offsets, np.int32)
    e = off.shape[0]
    start = np.zeros(e, np.int64)
    end = np.zeros(e, np.int64)
    lib().oracle_group_bounds(_p(off), e, rows_total, _p(start), _p(end))
    return start, end


def quant_rowwise(x_bits, fmt: int = E4M3FN, scale_max: float = 0.0):
    """Rowwise absmax -> scale -> clamp -> RNE cast.  x_bits: uint16 [rows, cols].

    Returns (codes uint8 [rows, cols], scales fp32 [rows], saturated count)."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    q = np.zeros((rows, cols), np.uint8)
    s = np.zeros(rows, np.float32)
    sat = np.zeros(1, np.uint64)
    lib().oracle_quant_rowwise(_p(x), rows, cols, cols, _p(q), cols, _p(s), fmt,
                               float(scale_max), _p(sat))
    return q, s, int(sat[0])


def quant_colwise_jagged(x_bits, offsets, layout: int = SAME, fmt: int = E4M3FN,
                         scale_max: float = 0.0, ld_q: int = None, fill: int = 0):
    """Per-(group, column) absmax -> scale -> clamp -> RNE cast.

    x_bits: uint16 [rows_total, cols]; offsets: int32 cumulative group ends.
    Returns (codes, scales fp32 [E, cols], saturated count).  codes is
    [rows_total, cols] for SAME and [cols, ld_q] for TRANSPOSED; entries that
    no group covers keep ``fill``."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    off = _c(offsets, np.int32)
    e = off.shape[0]
    if layout == TRANSPOSED:
        ld = rows if ld_q is None else ld_q
        q = np.full((cols, ld), fill, np.uint8)
    else:
        ld = cols if ld_q is None else ld_q
        q = np.full((rows, ld), fill, np.uint8)
    s = np.zeros((e, cols), np.float32)
    sat = np.zeros(1, np.uint64)
    start = np.zeros(max(e, 1), np.int64)
    end = np.zeros(max(e, 1), np.int64)
    lib().oracle_quant_colwise_jagged(_p(x), rows, cols, cols, _p(off), e, _p(q), ld, layout,
                                      _p(s), fmt, float(scale_max), _p(sat), _p(start), _p(end))
    return q, s, int(sat[0])


def gemm_m_jagged_sample(qa, sa, qb, sb, offsets, rows, cols, fmt: int = E4M3FN):
    """Sampled fp64 reference of the token-jagged grouped GEMM.

    qa: uint8 [m_total, k]; sa: fp32 [m_total]; qb: uint8 [E, n, k];
    sb: fp32 [E, n].  Returns (c_ref, bound) at (rows[i], cols[i])."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sa = _c(sa, np.float32)
    sb = _c(sb, np.float32)
    off = _c(offsets, np.int32)
    m_total, k = qa.shape
    e, n, k2 = qb.shape
    assert k2 == k and sb.shape == (e, n)
    rows = _c(rows, np.int64)
    cols = _c(cols, np.int64)
    ns = rows.shape[0]
    c = np.zeros(ns, np.float64)
    b = np.zeros(ns, np.float64)
    start = np.zeros(max(e, 1), np.int64)
    end = np.zeros(max(e, 1), np.int64)
    lib().oracle_gemm_m_jagged_sample(_p(qa), k, _p(sa), _p(qb), k, n * k, _p(sb), n, _p(off),
                                      off.shape[0], m_total, k, fmt, _p(rows), _p(cols), ns,
                                      _p(c), _p(b), _p(start), _p(end))
    return c, b


def gemm_k_jagged_sample(qa_t, sa, qb_t, sb, offsets, m_total, grp, rows, cols,
                         fmt: int = E4M3FN):
    """Sampled fp64 reference of the contraction-jagged grouped GEMM (dW).

    qa_t: uint8 [n, ld_a]; sa: fp32 [E, n]; qb_t: uint8 [k, ld_b];
    sb: fp32 [E, k].  Returns (c_ref, bound) at (grp[i], rows[i], cols[i])."""
    qa_t = _c(qa_t, np.uint8)
    qb_t = _c(qb_t, np.uint8)
    sa = _c(sa, np.float32)
    sb = _c(sb, np.float32)
    off = _c(offsets, np.int32)
    n, ld_a = qa_t.shape
    k, ld_b = qb_t.shape
    e = off.shape[0]
    grp = _c(grp, np.int64)
    rows = _c(rows, np.int64)
    cols = _c(cols, np.int64)
    ns = rows.shape[0]
    c = np.zeros(ns, np.float64)
    b = np.zeros(ns, np.float64)
    start = np.zeros(max(e, 1), np.int64)
    end = np.zeros(max(e, 1), np.int64)
    lib().oracle_gemm_k_jagged_sample(_p(qa_t), ld_a, _p(sa), n, _p(qb_t), ld_b, _p(sb), k,
                                      _p(off), e, m_total, fmt, _p(grp), _p(rows), _p(cols), ns,
                                      _p(c), _p(b), _p(start), _p(end))
    return c, b


# ---------------------------------------------------------------- MXFP8
# The OCP MX v1.0 reading of MXFP8 (32-element blocks, E8M0 scale
# 2^(floor(log2 amax) - 8), e4m3fn elements); see the MX section of
# fp8_oracle.c.


def padded_len(sizes) -> int:
    """Tokens of the padded transposed layout: sum of round_up(size, 128)."""
    return int(sum((int(s) + 127) // 128 * 128 for s in sizes))


def mx_quant_rowwise(x_bits):
    """MX quantisation along rows.  x_bits: uint16 [rows, cols], cols % 32 == 0.

    Returns (codes uint8 [rows, cols], scales uint8 [rows, cols // 32])."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    assert cols % 32 == 0
    q = np.zeros((rows, cols), np.uint8)
    s = np.zeros((rows, cols // 32), np.uint8)
    lib().oracle_mx_quant_rowwise(_p(x), rows, cols, cols, _p(q), cols, _p(s), cols // 32)
    return q, s


def mx_quant_colwise_padded(x_bits, offsets, ld_q: int = None, fill: int = 0,
                            scale_fill: int = 0):
    """MX quantisation along each group's tokens, transposed into the padded
    layout.  x_bits: uint16 [rows_total, cols]; offsets: int32 group ends.

    Returns (codes uint8 [cols, ld_q], scales uint8 [cols, ld_q // 32]);
    entries past the last padded group keep ``fill`` / ``scale_fill``."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    off = _c(offsets, np.int32)
    e = off.shape[0]
    start, end = group_bounds(off, rows) if e else (np.zeros(0, np.int64),) * 2
    need = padded_len(end - start)
    ld = need if ld_q is None else ld_q
    assert ld >= need and ld % 32 == 0
    q = np.full((cols, ld), fill, np.uint8)
    s = np.full((cols, ld // 32), scale_fill, np.uint8)
    st = np.zeros(max(e, 1), np.int64)
    en = np.zeros(max(e, 1), np.int64)
    ps = np.zeros(max(e, 1), np.int64)
    lib().oracle_mx_quant_colwise_padded(_p(x), rows, cols, cols, _p(off), e, _p(q), ld, _p(s),
                                         ld // 32, _p(st), _p(en), _p(ps))
    return q, s


def mx_gemm_m_jagged_sample(qa, sa, qb, sb, offsets, rows, cols):
    """Sampled fp64 reference of the MX token-jagged grouped GEMM.

    qa: uint8 [m_total, k]; sa: uint8 [m_total, k // 32]; qb: uint8 [E, n, k];
    sb: uint8 [E, n, k // 32].  Returns (c_ref, bound)."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sa = _c(sa, np.uint8)
    sb = _c(sb, np.uint8)
    off = _c(offsets, np.int32)
    m_total, k = qa.shape
    e, n, k2 = qb.shape
    assert k2 == k and sa.shape == (m_total, k // 32) and sb.shape == (e, n, k // 32)
    rows = _c(rows, np.int64)
    cols = _c(cols, np.int64)
    ns = rows.shape[0]
    c = np.zeros(ns, np.float64)
    b = np.zeros(ns, np.float64)
    start = np.zeros(max(e, 1), np.int64)
    end = np.zeros(max(e, 1), np.int64)
    lib().oracle_mx_gemm_m_jagged_sample(_p(qa), k, _p(sa), k // 32, _p(qb), k, n * k, _p(sb),
                                         k // 32, n * (k // 32), _p(off), off.shape[0], m_total,
                                         k, _p(rows), _p(cols), ns, _p(c), _p(b), _p(start),
                                         _p(end))
    return c, b


def mx_gemm_k_jagged_padded_sample(qa_t, sa_t, qb_t, sb_t, offsets, m_total, grp, rows, cols):
    """Sampled fp64 reference of the MX contraction-jagged grouped GEMM on
    the padded transposed layout.  qa_t: uint8 [n, ld_a]; sa_t: uint8
    [n, ld_a // 32]; qb_t / sb_t likewise for the second operand.
    Returns (c_ref, bound) at (grp[i], rows[i], cols[i])."""
    qa_t = _c(qa_t, np.uint8)
    qb_t = _c(qb_t, np.uint8)
    sa_t = _c(sa_t, np.uint8)
    sb_t = _c(sb_t, np.uint8)
    off = _c(offsets, np.int32)
    e = off.shape[0]
    grp = _c(grp, np.int64)
    rows = _c(rows, np.int64)
    cols = _c(cols, np.int64)
    ns = rows.shape[0]
    c = np.zeros(ns, np.float64)
    b = np.zeros(ns, np.float64)
    st = np.zeros(max(e, 1), np.int64)
    en = np.zeros(max(e, 1), np.int64)
    ps = np.zeros(max(e, 1), np.int64)
    lib().oracle_mx_gemm_k_jagged_padded_sample(
        _p(qa_t), qa_t.shape[1], _p(sa_t), sa_t.shape[1], _p(qb_t), qb_t.shape[1], _p(sb_t),
        sb_t.shape[1], _p(off), e, m_total, _p(grp), _p(rows), _p(cols), ns, _p(c), _p(b),
        _p(st), _p(en), _p(ps))
    return c, b
