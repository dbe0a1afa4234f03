"""The no-allocation variant of the jagged column-wise quantisation.

Callers such as runtimes that fix their device-memory budget at start-up (and
forbid cudaMalloc afterwards) or plugin interfaces that hand over tensors but
no scratch buffer cannot pass a workspace.  fp8_quant_colwise_jagged_noalloc
serves them from a fixed scratch array inside the library.  These checks call
it through the C ABI and require the same codes and scales as the regular
entry point, on two calls in a row (the second call must not see the first
call's leftovers in the shared scratch).

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import quantization_grouped_gemm_b200 as qgg
from quantization_grouped_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def call_noalloc(x, off, layout, q, scales, fmt=qgg.E4M3FN, status=None):
    lib = qgg.lib()
    rows, cols = x.shape
    ld_q = q.stride(0) if q.shape[0] > 1 else q.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.fp8_quant_colwise_jagged_noalloc(
        _p(x), rows, cols, x.stride(0), _p(off), off.numel(), _p(q), ld_q, layout, _p(scales),
        fmt, 0.0, None, _p(status), stream)


def make_case(seed, sizes, cols):
    m = int(sum(sizes))
    g = np.random.default_rng(seed)
    a = g.standard_normal((m, cols)).astype(np.float32)
    a.reshape(-1)[g.integers(0, a.size, max(1, a.size // 500))] *= 50
    x = wl.to_bf16(a).cuda()
    off = torch.from_numpy(wl.offsets_from_sizes(sizes)).cuda()
    return x, off


@pytest.mark.parametrize("layout", [qgg.LAYOUT_SAME, qgg.LAYOUT_TRANSPOSED])
def test_noalloc_matches_regular_entry_point_on_two_calls_in_a_row(layout):
    # two different problems back to back: both use the shared scratch for
    # groups taller than one block's chunk
    cases = [make_case(1, [2500, 0, 17, 1300, 5], 200), make_case(2, [700, 4100, 3], 136)]
    outs = []
    for x, off in cases:
        m, cols = x.shape
        ld = (m + 15) // 16 * 16
        shape = (cols, ld) if layout == qgg.LAYOUT_TRANSPOSED else (m, cols)
        q = torch.full(shape, 0xAB, dtype=torch.uint8, device="cuda")
        s = torch.full((off.numel(), cols), -1.0, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert call_noalloc(x, off, layout, q, s, status=st) == 0
        outs.append((q, s, st))
    torch.cuda.synchronize()
    for (x, off), (q, s, st) in zip(cases, outs):
        m = x.shape[0]
        q_ref, s_ref = qgg.fp8_quant_colwise_jagged(x, off, layout,
                                                    ld_q=q.shape[1] if layout else None)
        torch.cuda.synchronize()
        if layout == qgg.LAYOUT_TRANSPOSED:
            assert torch.equal(q[:, :m], q_ref[:, :m])
        else:
            assert torch.equal(q, q_ref)
        assert torch.equal(s, s_ref)
        assert int(st.item()) == 0


def test_noalloc_rejects_problems_beyond_its_scratch_and_accepts_the_rest():
    """Problems whose workspace exceeds the fixed array are refused with
    FP8QGG_ERR_SHAPE before anything runs; one just inside the limit runs."""
    limit = 2 * 1024 * 1024
    big = (98304, 8192, 64)
    assert qgg.colwise_workspace_bytes(*big) > limit
    assert 0 < qgg.colwise_workspace_bytes(98304, 2048, 64) <= limit
    # a small stand-in with the big problem's sizes is enough for the check,
    # which happens on the host before any device access
    x, off = make_case(3, [800, 900], 64)
    q = torch.empty((1700, 64), dtype=torch.uint8, device="cuda")
    s = torch.empty((2, 64), device="cuda")
    lib = qgg.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.fp8_quant_colwise_jagged_noalloc(
        _p(x), big[0], big[1], big[1], _p(off), big[2], _p(q), big[1], qgg.LAYOUT_SAME, _p(s),
        qgg.E4M3FN, 0.0, None, None, stream)
    assert rc == -2
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert call_noalloc(x, off, qgg.LAYOUT_SAME, q, s, status=st) == 0
    q_ref, s_ref = qgg.fp8_quant_colwise_jagged(x, off, qgg.LAYOUT_SAME)
    torch.cuda.synchronize()
    assert torch.equal(q, q_ref) and torch.equal(s, s_ref) and int(st.item()) == 0
