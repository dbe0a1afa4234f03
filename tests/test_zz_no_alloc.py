"""The no-allocation variant of the jagged column-wise quantisation.

Callers such as runtimes that fix their device-memory budget at start-up (and
forbid cudaMalloc afterwards) or plugin interfaces that hand over tensors but
no scratch buffer cannot pass a workspace.  fp8_quant_colwise_jagged_noalloc
serves them from a fixed scratch array inside the library.  These checks call
it through the C ABI and require the same codes and scales as the regular
entry point and as the oracle, on two calls in a row (the second call must not
see the first call's leftovers in the shared scratch), in all three layouts.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as orc
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


def padded_positions(sizes):
    """First token of each group in the padded transposed layout and its end."""
    sizes = np.asarray(sizes, np.int64)
    padded = (sizes + 127) // 128 * 128
    p_start = np.concatenate([[0], np.cumsum(padded)[:-1]])
    return p_start, int(p_start[-1] + padded[-1])


@pytest.mark.parametrize("layout", [qgg.LAYOUT_SAME, qgg.LAYOUT_TRANSPOSED,
                                    qgg.LAYOUT_TRANSPOSED_PADDED])
def test_noalloc_matches_regular_entry_point_on_two_calls_in_a_row(layout):
    # two different problems back to back: both use the shared scratch for
    # groups taller than one block's chunk
    size_sets = [[2500, 0, 17, 1300, 5], [700, 4100, 3]]
    cases = [make_case(1, size_sets[0], 200), make_case(2, size_sets[1], 136)]
    outs = []
    for x, off in cases:
        m, cols = x.shape
        e = off.numel()
        if layout == qgg.LAYOUT_TRANSPOSED:
            shape = (cols, (m + 15) // 16 * 16)
        elif layout == qgg.LAYOUT_TRANSPOSED_PADDED:
            shape = (cols, (m + 128 * e + 15) // 16 * 16)
        else:
            shape = (m, cols)
        q = torch.full(shape, 0xAB, dtype=torch.uint8, device="cuda")
        s = torch.full((e, cols), -1.0, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert call_noalloc(x, off, layout, q, s, status=st) == 0
        outs.append((q, s, st))
    torch.cuda.synchronize()
    for sizes, (x, off), (q, s, st) in zip(size_sets, cases, outs):
        m = x.shape[0]
        # the regular entry point, on a buffer with the same starting contents
        q_reg = torch.full(q.shape, 0xAB, dtype=torch.uint8, device="cuda")
        q_reg, s_reg = qgg.fp8_quant_colwise_jagged(x, off, layout, q=q_reg)
        torch.cuda.synchronize()
        if layout == qgg.LAYOUT_TRANSPOSED:
            assert torch.equal(q[:, :m], q_reg[:, :m])
        elif layout == qgg.LAYOUT_TRANSPOSED_PADDED:
            p_start, p_end = padded_positions(sizes)
            assert torch.equal(q[:, :p_end], q_reg[:, :p_end])  # codes and zero gaps
        else:
            assert torch.equal(q, q_reg)
        assert torch.equal(s, s_reg)
        assert int(st.item()) == 0
        # and directly against the oracle
        xb = wl.bf16_bits(x.cpu())
        olay = orc.SAME if layout == qgg.LAYOUT_SAME else orc.TRANSPOSED
        q_ref, s_ref, _ = orc.quant_colwise_jagged(xb, off.cpu().numpy(), olay)
        qn = q.cpu().numpy()
        if layout == qgg.LAYOUT_SAME:
            assert (qn == q_ref).all()
        elif layout == qgg.LAYOUT_TRANSPOSED:
            assert (qn[:, :m] == q_ref).all()
        else:
            starts = np.concatenate([[0], np.cumsum(sizes)[:-1]])
            expect = np.zeros((qn.shape[0], p_end), np.uint8)
            for g, sz in enumerate(sizes):
                expect[:, p_start[g]:p_start[g] + sz] = q_ref[:, starts[g]:starts[g] + sz]
            assert (qn[:, :p_end] == expect).all()
        assert (s.cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()


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
