"""B200-native FP8 quantisation and FP8 scaled grouped GEMM for MoE training.

Thin Python binding over the C ABI in ``include/fp8qgg.h`` (``libfp8qgg.so``,
built in-tree for sm_100a).  This module only marshals arguments: it turns
torch CUDA tensors into device pointers, allocates outputs with torch and
passes torch's current stream.  Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback.  A missing or
unloadable library raises ``RuntimeError``.
"""
import ctypes
import os
import threading

import torch

E4M3FN = 0
E4M3FNUZ = 1
LAYOUT_SAME = 0
LAYOUT_TRANSPOSED = 1
LAYOUT_TRANSPOSED_PADDED = 2
M_JAGGED = 0
K_JAGGED = 1
K_JAGGED_PADDED = 2
OUT_F32 = 0
OUT_BF16 = 1
STATUS_BAD_OFFSETS = 1
STATUS_TIMEOUT = 2

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8qgg.so")
_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_INT = ctypes.c_int
_F32 = ctypes.c_float
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "fp8_native_format": (_INT, []),
    "fp8qgg_error_string": (ctypes.c_char_p, [_INT]),
    "fp8_quant_rowwise": (_INT, [_P, _I64, _I64, _I64, _P, _I64, _P, _INT, _F32, _P, _P]),
    "fp8_quant_colwise_jagged_workspace_size": (_SZ, [_I64, _I64, _I32]),
    "fp8_quant_colwise_jagged": (_INT, [_P, _I64, _I64, _I64, _P, _I32, _P, _I64, _INT, _P,
                                        _INT, _F32, _P, _P, _P, _SZ, _P]),
    "fp8_scaled_grouped_gemm": (_INT, [_INT, _P, _I64, _P, _I64, _P, _I64, _I64, _P, _I64, _P,
                                       _I32, _I64, _I64, _I64, _P, _I64, _I64, _INT, _INT, _P,
                                       _P]),
    "fp8_cast_f32": (_INT, [_P, _I64, _P, _INT, _P]),
    "fp8_quant_colwise_jagged_noalloc": (_INT, [_P, _I64, _I64, _I64, _P, _I32, _P, _I64, _INT,
                                                _P, _INT, _F32, _P, _P, _P]),
    "fp8qgg_test_unit_wait": (_INT, [ctypes.c_uint32, ctypes.c_uint64]),
    "fp8_quant_dual_jagged_workspace_size": (_SZ, [_I64, _I64, _I32]),
    "fp8_quant_dual_jagged": (_INT, [_P, _I64, _I64, _I64, _P, _I32, _P, _I64, _P, _P, _I64, _P,
                                     _INT, _F32, _P, _P, _P, _SZ, _P]),
    "fp8_mx_quant_rowwise": (_INT, [_P, _I64, _I64, _I64, _P, _I64, _P, _I64, _P]),
    "fp8_mx_quant_colwise_padded": (_INT, [_P, _I64, _I64, _I64, _P, _I32, _P, _I64, _P, _I64,
                                           _P, _P]),
    "fp8_mx_grouped_gemm": (_INT, [_INT, _P, _I64, _P, _I64, _P, _I64, _I64, _P, _I64, _I64, _P,
                                   _I32, _I64, _I64, _I64, _P, _I64, _I64, _INT, _P, _P]),
    "fp8_mx_quant_dual_padded": (_INT, [_P, _I64, _I64, _I64, _P, _I32, _P, _I64, _P, _I64, _P,
                                        _I64, _P, _I64, _P, _P]),
}


def lib():
    """The loaded C library (built in-tree on first use if absent)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    from . import build as _build
                    _build.build()
                try:
                    L = ctypes.CDLL(LIB_PATH)
                except OSError as e:
                    raise RuntimeError(f"fp8qgg CUDA library could not be loaded: {e}") from e
                for name, (res, args) in _SIGNATURES.items():
                    f = getattr(L, name)
                    f.restype = res
                    f.argtypes = args
                _lib = L
    return _lib


class Fp8qggError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != 0:
        msg = lib().fp8qgg_error_string(rc).decode()
        raise Fp8qggError(f"{what} failed with status {rc}: {msg}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ld(t):
    """Leading dimension (elements between rows) of a row-major 2-D tensor; for a
    tensor with at most one row the row stride is irrelevant and the width is used."""
    if t.shape[0] <= 1:
        return t.shape[1]
    assert t.stride(1) == 1 or t.shape[1] <= 1, "rows must be contiguous"
    return t.stride(0)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("fp8qgg operates on CUDA tensors only")


def native_format() -> int:
    return lib().fp8_native_format()


def fp8_quant_rowwise(x, fmt=E4M3FN, scale_max=0.0, q=None, scales=None, sat_count=None,
                      stream=None):
    """Rowwise quantisation of a bf16 [rows, cols] CUDA tensor (row stride may exceed cols).

    Returns (q uint8 [rows, cols], scales fp32 [rows])."""
    _need_cuda(x)
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    rows, cols = x.shape
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows,), dtype=torch.float32, device=x.device)
    _need_cuda(q, scales, sat_count)
    rc = lib().fp8_quant_rowwise(_ptr(x), rows, cols, _ld(x), _ptr(q), _ld(q),
                                 _ptr(scales), fmt, float(scale_max), _ptr(sat_count),
                                 _stream(stream))
    _check(rc, "fp8_quant_rowwise")
    return q, scales


def colwise_workspace_bytes(rows_total, cols, num_groups) -> int:
    return int(lib().fp8_quant_colwise_jagged_workspace_size(rows_total, cols, num_groups))


def fp8_quant_colwise_jagged(x, offsets, layout=LAYOUT_SAME, fmt=E4M3FN, scale_max=0.0,
                             q=None, ld_q=None, scales=None, workspace=None, sat_count=None,
                             status=None, stream=None):
    """Per-(group, column) quantisation of a bf16 [rows_total, cols] CUDA tensor.

    offsets: int32 CUDA tensor of cumulative group ends.  Returns (q, scales)
    with q [rows_total, cols] (SAME) or [cols, ld_q] (TRANSPOSED and
    TRANSPOSED_PADDED), scales fp32 [num_groups, cols]."""
    _need_cuda(x, offsets)
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    assert offsets.dtype == torch.int32
    rows, cols = x.shape
    e = offsets.numel()
    if q is None:
        if layout == LAYOUT_TRANSPOSED:
            # default row pitch: a multiple of 128 tokens, so that every
            # 128-token block the contraction-jagged GEMM copies is aligned
            ld = ld_q if ld_q is not None else (rows + 127) // 128 * 128
            q = torch.empty((cols, ld), dtype=torch.uint8, device=x.device)
        elif layout == LAYOUT_TRANSPOSED_PADDED:
            # room for every group rounded up to 128 tokens
            ld = ld_q if ld_q is not None else (rows + 128 * e + 127) // 128 * 128
            q = torch.empty((cols, ld), dtype=torch.uint8, device=x.device)
        else:
            q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((e, cols), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(colwise_workspace_bytes(rows, cols, e), dtype=torch.uint8,
                                device=x.device)
    _need_cuda(q, scales, workspace, sat_count, status)
    rc = lib().fp8_quant_colwise_jagged(
        _ptr(x), rows, cols, _ld(x), _ptr(offsets), e, _ptr(q), _ld(q), layout,
        _ptr(scales), fmt, float(scale_max), _ptr(sat_count), _ptr(status), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "fp8_quant_colwise_jagged")
    return q, scales


def dual_workspace_bytes(rows_total, cols, num_groups) -> int:
    return int(lib().fp8_quant_dual_jagged_workspace_size(rows_total, cols, num_groups))


def fp8_quant_dual_jagged(x, offsets, fmt=E4M3FN, scale_max=0.0, q_row=None, scales_row=None,
                          q_col=None, ld_qc=None, scales_col=None, workspace=None,
                          sat_count=None, status=None, stream=None):
    """One read of a bf16 [rows_total, cols] CUDA tensor gives its rowwise
    quantisation (q_row [rows_total, cols], scales_row [rows_total], rows of the
    groups) and its jagged column-wise quantisation in LAYOUT_TRANSPOSED_PADDED
    (q_col [cols, ld_qc], scales_col [num_groups, cols]).

    Returns (q_row, scales_row, q_col, scales_col)."""
    _need_cuda(x, offsets)
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    assert offsets.dtype == torch.int32
    rows, cols = x.shape
    e = offsets.numel()
    if q_row is None:
        q_row = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales_row is None:
        scales_row = torch.empty((rows,), dtype=torch.float32, device=x.device)
    if q_col is None:
        ld = ld_qc if ld_qc is not None else (rows + 128 * e + 127) // 128 * 128
        q_col = torch.empty((cols, ld), dtype=torch.uint8, device=x.device)
    if scales_col is None:
        scales_col = torch.empty((e, cols), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(dual_workspace_bytes(rows, cols, e), dtype=torch.uint8,
                                device=x.device)
    _need_cuda(q_row, scales_row, q_col, scales_col, workspace, sat_count, status)
    rc = lib().fp8_quant_dual_jagged(
        _ptr(x), rows, cols, _ld(x), _ptr(offsets), e, _ptr(q_row), _ld(q_row),
        _ptr(scales_row), _ptr(q_col), _ld(q_col), _ptr(scales_col), fmt, float(scale_max),
        _ptr(sat_count), _ptr(status), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "fp8_quant_dual_jagged")
    return q_row, scales_row, q_col, scales_col


def fp8_scaled_grouped_gemm(mode, a, scale_a, b, scale_b, offsets, m_total=None, n=None, k=None,
                            out=None, out_dtype=torch.float32, status=None, b_group_stride=None,
                            stream=None):
    """FP8 scaled grouped GEMM (see the C header for the two modes).

    M_JAGGED: a uint8 [m_total, K], scale_a [m_total], b uint8 [E, N, K] (or any
    layout with b_group_stride), scale_b [E, N] -> out [m_total, N].
    K_JAGGED: a uint8 [N, ld_a], b uint8 [K, ld_b] (token axis contiguous),
    scale_a [E, N], scale_b [E, K], m_total tokens -> out [E, N, K].
    K_JAGGED_PADDED: as K_JAGGED, on operands in LAYOUT_TRANSPOSED_PADDED;
    m_total is the unpadded token count."""
    _need_cuda(a, scale_a, b, scale_b, offsets)
    assert a.dtype == torch.uint8 and b.dtype == torch.uint8 and offsets.dtype == torch.int32
    e = offsets.numel()
    if out is not None:
        out_dtype = out.dtype
    assert out_dtype in (torch.float32, torch.bfloat16)
    odt = OUT_F32 if out_dtype == torch.float32 else OUT_BF16
    if mode == M_JAGGED:
        m_total = a.shape[0] if m_total is None else m_total
        k = a.shape[1] if k is None else k
        if b.dim() == 3:
            n = b.shape[1] if n is None else n
            ld_b = b.stride(1)
            bgs = b.stride(0) if b_group_stride is None else b_group_stride
        else:
            n = b.shape[0] // e if n is None else n
            ld_b = b.stride(0)
            bgs = n * ld_b if b_group_stride is None else b_group_stride
        sbs = scale_b.shape[-1] if scale_b.dim() == 2 else n
        if out is None:
            out = torch.empty((m_total, n), dtype=out_dtype, device=a.device)
        ld_out, ogs, sas, ld_a = _ld(out), 0, 0, _ld(a)
    else:
        n = a.shape[0] if n is None else n
        k = b.shape[0] if k is None else k
        assert m_total is not None
        ld_a, ld_b, bgs = _ld(a), _ld(b), 0
        sas = scale_a.shape[-1]
        sbs = scale_b.shape[-1]
        if out is None:
            out = torch.empty((e, n, k), dtype=out_dtype, device=a.device)
        ld_out, ogs = out.stride(-2), out.stride(0)
    _need_cuda(out, status)
    rc = lib().fp8_scaled_grouped_gemm(
        mode, _ptr(a), ld_a, _ptr(scale_a), sas, _ptr(b), ld_b, bgs, _ptr(scale_b), sbs,
        _ptr(offsets), e, m_total, n, k, _ptr(out), ld_out, ogs, odt, E4M3FN, _ptr(status),
        _stream(stream))
    _check(rc, "fp8_scaled_grouped_gemm")
    return out


def fp8_cast_f32(y, fmt=E4M3FN, q=None, sat_count=None, stream=None):
    """Round-to-nearest-even saturating cast of an fp32 CUDA tensor to e4m3 codes."""
    _need_cuda(y)
    assert y.dtype == torch.float32 and y.is_contiguous()
    if q is None:
        q = torch.empty(y.shape, dtype=torch.uint8, device=y.device)
    rc = lib().fp8_cast_f32(_ptr(y), y.numel(), _ptr(q), fmt, _stream(stream))
    _check(rc, "fp8_cast_f32")
    return q


# ------------------------------------------------------------------ MXFP8
def mx_scale_groups(length: int) -> int:
    """Scale words per row: one per 128 elements of the contraction axis."""
    return (length + 127) // 128


def mx_scales_to_blocks(words, nblocks: int):
    """The packed scale words [groups, ld_sw] (torch int32 / uint32 storage)
    as plain E8M0 bytes [rows, nblocks] for the first ld_sw rows: byte j of
    word (g, r) is the scale of block 4g + j of row r.  (A view change and a
    transpose, for reading results; the kernels never need it.)"""
    w = words.contiguous().view(torch.uint8).view(words.shape[0], words.shape[1], 4)
    return w.permute(1, 0, 2).reshape(words.shape[1], -1)[:, :nblocks]


def fp8_mx_quant_rowwise(x, q=None, scales=None, stream=None):
    """MXFP8 quantisation along the rows of a bf16 [rows, cols] CUDA tensor
    (cols % 32 == 0): one E8M0 scale byte per 32 consecutive columns, packed
    four to a word per 128 columns.

    Returns (q uint8 [rows, cols], scales int32 [ceil(cols / 128), rows])."""
    _need_cuda(x)
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    rows, cols = x.shape
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((mx_scale_groups(cols), rows), dtype=torch.int32, device=x.device)
    _need_cuda(q, scales)
    assert scales.dtype == torch.int32
    rc = lib().fp8_mx_quant_rowwise(_ptr(x), rows, cols, _ld(x), _ptr(q), _ld(q), _ptr(scales),
                                    _ld(scales), _stream(stream))
    _check(rc, "fp8_mx_quant_rowwise")
    return q, scales


def fp8_mx_quant_colwise_padded(x, offsets, q=None, ld_q=None, scales=None, status=None,
                                stream=None):
    """MXFP8 quantisation along each expert group's tokens of a bf16
    [rows_total, cols] CUDA tensor, written transposed in the padded layout
    (group e from token P_e, zero codes up to a 128-token boundary).

    Returns (q uint8 [cols, ld_q], scales int32 [ld_q // 128, cols])."""
    _need_cuda(x, offsets)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and offsets.dtype == torch.int32
    rows, cols = x.shape
    e = offsets.numel()
    if q is None:
        ld = ld_q if ld_q is not None else (rows + 128 * e + 127) // 128 * 128
        q = torch.empty((cols, ld), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((mx_scale_groups(q.shape[1]), cols), dtype=torch.int32,
                             device=x.device)
    _need_cuda(q, scales, status)
    assert scales.dtype == torch.int32
    rc = lib().fp8_mx_quant_colwise_padded(_ptr(x), rows, cols, _ld(x), _ptr(offsets), e,
                                           _ptr(q), _ld(q), _ptr(scales), _ld(scales),
                                           _ptr(status), _stream(stream))
    _check(rc, "fp8_mx_quant_colwise_padded")
    return q, scales


def fp8_mx_quant_dual_padded(x, offsets, q_row=None, scales_row=None, q_col=None, ld_qc=None,
                             scales_col=None, status=None, stream=None):
    """One read of a bf16 [rows_total, cols] CUDA tensor (cols % 32 == 0) gives
    its MX rowwise quantisation (rows of the groups) and its MX column-wise
    quantisation in the padded transposed layout.

    Returns (q_row [rows_total, cols], scales_row int32 [cols/128, rows_total],
    q_col [cols, ld_qc], scales_col int32 [ld_qc/128, cols])."""
    _need_cuda(x, offsets)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and offsets.dtype == torch.int32
    rows, cols = x.shape
    e = offsets.numel()
    if q_row is None:
        q_row = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales_row is None:
        scales_row = torch.empty((mx_scale_groups(cols), rows), dtype=torch.int32,
                                 device=x.device)
    if q_col is None:
        ld = ld_qc if ld_qc is not None else (rows + 128 * e + 127) // 128 * 128
        q_col = torch.empty((cols, ld), dtype=torch.uint8, device=x.device)
    if scales_col is None:
        scales_col = torch.empty((mx_scale_groups(q_col.shape[1]), cols), dtype=torch.int32,
                                 device=x.device)
    _need_cuda(q_row, scales_row, q_col, scales_col, status)
    rc = lib().fp8_mx_quant_dual_padded(
        _ptr(x), rows, cols, _ld(x), _ptr(offsets), e, _ptr(q_row), _ld(q_row), _ptr(scales_row),
        _ld(scales_row), _ptr(q_col), _ld(q_col), _ptr(scales_col), _ld(scales_col),
        _ptr(status), _stream(stream))
    _check(rc, "fp8_mx_quant_dual_padded")
    return q_row, scales_row, q_col, scales_col


def fp8_mx_grouped_gemm(mode, a, scale_a, b, scale_b, offsets, m_total=None, n=None, k=None,
                        out=None, out_dtype=torch.float32, status=None, b_group_stride=None,
                        scale_b_group_stride=None, stream=None):
    """MXFP8 grouped GEMM (see the C header); scales as returned by the MX
    quantisation calls (int32 words [groups, rows]).

    M_JAGGED: a uint8 [m_total, K], scale_a [K/128, m_total], b uint8 [E, N, K]
    (or [E*N, K]), scale_b [K/128, E*N] -> out [m_total, N].
    K_JAGGED_PADDED: a uint8 [N, ld_a], scale_a [ld_a/128, N], b uint8 [K, ld_b],
    scale_b [ld_b/128, K] (outputs of fp8_mx_quant_colwise_padded), m_total
    unpadded tokens -> out [E, N, K]."""
    _need_cuda(a, scale_a, b, scale_b, offsets)
    assert a.dtype == torch.uint8 and b.dtype == torch.uint8 and offsets.dtype == torch.int32
    assert scale_a.dtype == torch.int32 and scale_b.dtype == torch.int32
    e = offsets.numel()
    if out is not None:
        out_dtype = out.dtype
    assert out_dtype in (torch.float32, torch.bfloat16)
    odt = OUT_F32 if out_dtype == torch.float32 else OUT_BF16
    if mode == M_JAGGED:
        m_total = a.shape[0] if m_total is None else m_total
        k = a.shape[1] if k is None else k
        if b.dim() == 3:
            n = b.shape[1] if n is None else n
            ld_b = b.stride(1)
            bgs = b.stride(0) if b_group_stride is None else b_group_stride
        else:
            n = b.shape[0] // e if n is None else n
            ld_b = b.stride(0)
            bgs = n * ld_b if b_group_stride is None else b_group_stride
        sbgs = n if scale_b_group_stride is None else scale_b_group_stride
        if out is None:
            out = torch.empty((m_total, n), dtype=out_dtype, device=a.device)
        ld_out, ogs = _ld(out), 0
    else:
        n = a.shape[0] if n is None else n
        k = b.shape[0] if k is None else k
        assert m_total is not None
        ld_b, bgs, sbgs = _ld(b), 0, 0
        if out is None:
            out = torch.empty((e, n, k), dtype=out_dtype, device=a.device)
        ld_out, ogs = out.stride(-2), out.stride(0)
    _need_cuda(out, status)
    rc = lib().fp8_mx_grouped_gemm(
        mode, _ptr(a), _ld(a), _ptr(scale_a), _ld(scale_a), _ptr(b), ld_b, bgs, _ptr(scale_b),
        _ld(scale_b), sbgs, _ptr(offsets), e, m_total, n, k, _ptr(out), ld_out, ogs, odt,
        _ptr(status), _stream(stream))
    _check(rc, "fp8_mx_grouped_gemm")
    return out


class Fp8WeightCache:
    """FP8 codes and scales of weights kept between calls.

    Expert weights change only at optimizer steps, while the forward and
    backward passes of every micro-batch in between need their FP8 copies
    ("AMD Primus adds FP8/MXFP8 kernels ...", "What Primus adds for MoE
    training on MI355X": FP8 weight caching).  A cached copy is reused while
    the weight is the same tensor (storage, shape, strides) at the same
    in-place version (torch bumps ``tensor._version`` on every in-place
    update, which is how optimizers write parameters), and the quantisation
    is re-run, into the same buffers, when it changed.  This class only
    decides whether to call the library; every code and scale comes from the
    library's kernels.

    ``quantize`` is the function that fills (q, scales); it defaults to the
    library call and can be replaced (for instance by a counting wrapper).
    """

    def __init__(self, quantize=None):
        self._quantize = quantize
        self._entries = {}
        self.hits = 0
        self.misses = 0

    def _key(self, w, kind, args):
        return (kind, w.data_ptr(), tuple(w.shape), tuple(w.stride()), w.dtype, args)

    def rowwise(self, w, fmt=E4M3FN, scale_max=0.0):
        """(q, scales) of fp8_quant_rowwise(w), reused while w is unchanged."""
        q_fn = self._quantize or fp8_quant_rowwise
        key = self._key(w, "rowwise", (fmt, float(scale_max)))
        ent = self._entries.get(key)
        if ent is not None and ent[0] == w._version:
            self.hits += 1
            return ent[1], ent[2]
        self.misses += 1
        if ent is None:
            q, s = q_fn(w, fmt=fmt, scale_max=scale_max)
        else:
            q, s = q_fn(w, fmt=fmt, scale_max=scale_max, q=ent[1], scales=ent[2])
        self._entries[key] = (w._version, q, s)
        return q, s

    def colwise_jagged(self, w, offsets, layout=LAYOUT_SAME, fmt=E4M3FN, scale_max=0.0):
        """(q, scales) of fp8_quant_colwise_jagged(w, offsets, layout), reused
        while w and offsets are unchanged."""
        q_fn = self._quantize or fp8_quant_colwise_jagged
        key = self._key(w, "colwise", (layout, fmt, float(scale_max), offsets.data_ptr(),
                                       offsets.numel()))
        ent = self._entries.get(key)
        ver = (w._version, offsets._version)
        if ent is not None and ent[0] == ver:
            self.hits += 1
            return ent[1], ent[2]
        self.misses += 1
        if ent is None:
            q, s = q_fn(w, offsets, layout, fmt=fmt, scale_max=scale_max)
        else:
            q, s = q_fn(w, offsets, layout, fmt=fmt, scale_max=scale_max, q=ent[1],
                        scales=ent[2])
        self._entries[key] = (ver, q, s)
        return q, s

    def mx_rowwise(self, w):
        """(q, scales) of fp8_mx_quant_rowwise(w) (MXFP8, the forward's B),
        reused while w is unchanged."""
        q_fn = self._quantize or fp8_mx_quant_rowwise
        key = self._key(w, "mx_rowwise", ())
        ent = self._entries.get(key)
        if ent is not None and ent[0] == w._version:
            self.hits += 1
            return ent[1], ent[2]
        self.misses += 1
        if ent is None:
            q, s = q_fn(w)
        else:
            q, s = q_fn(w, q=ent[1], scales=ent[2])
        self._entries[key] = (w._version, q, s)
        return q, s

    def mx_colwise_padded(self, w, offsets):
        """(q, scales) of fp8_mx_quant_colwise_padded(w, offsets) (MXFP8,
        W^T for the input gradient with groups of each expert's rows), reused
        while w and offsets are unchanged."""
        q_fn = self._quantize or fp8_mx_quant_colwise_padded
        key = self._key(w, "mx_colwise", (offsets.data_ptr(), offsets.numel()))
        ent = self._entries.get(key)
        ver = (w._version, offsets._version)
        if ent is not None and ent[0] == ver:
            self.hits += 1
            return ent[1], ent[2]
        self.misses += 1
        if ent is None:
            q, s = q_fn(w, offsets)
        else:
            q, s = q_fn(w, offsets, q=ent[1], scales=ent[2])
        self._entries[key] = (ver, q, s)
        return q, s

    def clear(self):
        self._entries.clear()
