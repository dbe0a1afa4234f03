"""Parity at the full sizes of the benchmarked workloads, in the launch
configuration the benchmark times (its step classes and arguments).

The oracle cannot redo a whole step in seconds, so outputs are sampled where
the method makes samples independent:
  - rowwise: sampled rows (a row's scale and codes depend on that row only);
  - jagged colwise: sampled columns over all rows (a column's scales and codes
    depend on that column only), with the same offsets;
  - grouped GEMM: sampled outputs, computed by the oracle from its OWN
    quantisation of the rows and columns they need (never from the kernels'
    codes), within the bound 1e-3 * sum |a||b| per element.
Inputs are the seeded synthetic workloads the benchmark uses.
"""
import os
import sys

import numpy as np
import pytest
import torch

import oracle as orc
import quantization_grouped_gemm_b200 as qgg
from quantization_grouped_gemm_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402  (the step classes the benchmark times)

pytestmark = pytest.mark.gpu


def run_step(step):
    for f in step.kernels():
        f()
    torch.cuda.synchronize()


def sample(g, n, count, must=()):
    return np.unique(np.concatenate([np.asarray(must, np.int64),
                                     g.integers(0, n, count)])).astype(np.int64)


def check_forward(w, seed, n_rows=40, n_cols=40, n_out=2000):
    """Rowwise X and W on sampled rows, and the token-jagged GEMM on sampled
    outputs, for a ForwardStep run at full size."""
    st = bench.ForwardStep(w)
    run_step(st)
    g = np.random.default_rng(seed)
    m, k = w.x.shape
    e, n = w.w.shape[0], w.w.shape[1]
    off = np.asarray(w.offsets, np.int64)
    end = int(off[-1])
    # activations: sampled rows inside the groups (group starts and ends included)
    starts = np.concatenate([[0], off[:-1]])
    edges = np.concatenate([starts[off > starts], off[off > starts] - 1])
    rows = sample(g, end, n_rows, must=edges[:8])
    qa_ref, sa_ref, _ = orc.quant_rowwise(wl.bf16_bits(w.x[torch.from_numpy(rows)]))
    assert (st.qa[torch.from_numpy(rows).cuda()].cpu().numpy() == qa_ref).all()
    assert (st.sa.cpu().numpy()[rows].view(np.uint32) == sa_ref.view(np.uint32)).all()
    # weights: every expert's sampled output channels (quantised as [E*N, K] rows)
    cols = sample(g, n, n_cols, must=[0, n - 1])
    wsel = w.w[:, torch.from_numpy(cols), :].reshape(e * len(cols), k)
    qb_ref, sb_ref, _ = orc.quant_rowwise(wl.bf16_bits(wsel))
    qb = st.qb.view(e, n, k)[:, torch.from_numpy(cols).cuda(), :].reshape(e * len(cols), k)
    assert (qb.cpu().numpy() == qb_ref).all()
    sb = st.sb.view(e, n)[:, torch.from_numpy(cols).cuda()].reshape(-1)
    assert (sb.cpu().numpy().view(np.uint32) == sb_ref.view(np.uint32)).all()
    # GEMM: outputs (rows[i], cols[j]) from the oracle's operands, with the
    # sampled rows regrouped into compact offsets (a row keeps its group)
    grp = np.searchsorted(off, rows, side="right")
    off_c = np.array([(grp <= ge).sum() for ge in range(e)], np.int32)
    li = g.integers(0, len(rows), n_out)
    lj = g.integers(0, len(cols), n_out)
    c, b = orc.gemm_m_jagged_sample(qa_ref, sa_ref, qb_ref.reshape(e, len(cols), k),
                                    sb_ref.reshape(e, len(cols)), off_c, li, lj)
    out = st.out[torch.from_numpy(rows[li]).cuda(), torch.from_numpy(cols[lj]).cuda()]
    got = out.cpu().numpy().astype(np.float64)
    bad = np.nonzero(~(np.abs(got - c) <= b))[0]
    assert bad.size == 0, (bad.size, got[bad[:4]], c[bad[:4]], b[bad[:4]])


def test_llama3_8b_up_projection_full_size_sampled():
    check_forward(wl.llama3_8b_up_proj(), 11)


def test_deepseek_v3_local_experts_full_size_sampled():
    check_forward(wl.deepseek_v3_local_experts(), 12)


SWEEP = [(m, loads) for m in (4096, 8192, 16384, 32768, 65536, 131072)
         for loads in ("uniform", "zipf")]


def check_fnuz(w, seed, exact_mismatch):
    """The Llama-4 sweep's quantisation under e4m3fnuz (largest finite 240):
    rowwise X and W on sampled rows, jagged column-wise X (same layout and
    transposed) on sampled columns, all bit-exact against the oracle, with the
    saturation count on.  With the matching maximum nothing may saturate (the
    count is exactly 0, outliers of +-1e4 and zero rows and columns
    included).  With exact_mismatch, the 448 scaling maximum is also used with
    the 240 encoding (the silent-clipping mistake of "FP8 su GPU AMD: ..."
    (ai-radar.it), "La correttezza del formato viene prima del tuning") and
    the saturation count must equal a plain numpy fp32 count over the whole
    tensor."""
    import quantization_grouped_gemm_b200 as qgg
    from tests import numpy_sat
    FNUZ = qgg.E4M3FNUZ
    g = np.random.default_rng(seed)
    m, k = w.x.shape
    e, n = w.w.shape[0], w.w.shape[1]
    xd = w.x.cuda()
    wd = w.w.reshape(e * n, k).cuda()
    off = torch.from_numpy(w.offsets).cuda()
    sat = torch.zeros(1, dtype=torch.int64, device="cuda")

    def rowwise_rows(src_cpu, src_dev, rows, smax):
        sat.zero_()
        q, s = qgg.fp8_quant_rowwise(src_dev, FNUZ, scale_max=smax, sat_count=sat)
        q_ref, s_ref, _ = orc.quant_rowwise(wl.bf16_bits(src_cpu[torch.from_numpy(rows)]), FNUZ,
                                            scale_max=smax)
        assert (q[torch.from_numpy(rows).cuda()].cpu().numpy() == q_ref).all()
        assert (s.cpu().numpy()[rows].view(np.uint32) == s_ref.view(np.uint32)).all()
        return int(sat.item())

    xrows = sample(g, m, 40, must=[0, m - 1])
    wrows = sample(g, e * n, 40, must=[0, e * n - 1])
    assert rowwise_rows(w.x, xd, xrows, 0.0) == 0
    assert rowwise_rows(w.w.reshape(e * n, k), wd, wrows, 0.0) == 0
    cols = sample(g, k, 16, must=[0, k - 1])
    xcols = wl.bf16_bits(w.x[:, torch.from_numpy(cols)])
    colsd = torch.from_numpy(cols).cuda()
    for smax in ([0.0, 448.0] if exact_mismatch else [0.0]):
        expect = 0 if smax == 0.0 else numpy_sat.colwise_jagged(wl.bf16_bits(w.x), w.offsets,
                                                                  FNUZ, smax)
        for layout, olay in ((qgg.LAYOUT_SAME, orc.SAME), (qgg.LAYOUT_TRANSPOSED, orc.TRANSPOSED)):
            sat.zero_()
            q, s = qgg.fp8_quant_colwise_jagged(xd, off, layout, FNUZ, scale_max=smax,
                                                sat_count=sat)
            q_ref, s_ref, _ = orc.quant_colwise_jagged(xcols, w.offsets, olay, FNUZ,
                                                       scale_max=smax)
            got = q[:, colsd] if layout == qgg.LAYOUT_SAME else q[colsd, :m]
            assert (got.cpu().numpy() == q_ref).all()
            assert (s[:, colsd].cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()
            assert int(sat.item()) == expect
            if smax:
                assert expect > 0
    if exact_mismatch:
        got_x = rowwise_rows(w.x, xd, xrows, 448.0)
        assert got_x == numpy_sat.rowwise(wl.bf16_bits(w.x), FNUZ, 448.0) > 0
        got_w = rowwise_rows(w.w.reshape(e * n, k), wd, wrows, 448.0)
        assert got_w == numpy_sat.rowwise(wl.bf16_bits(w.w.reshape(e * n, k)), FNUZ, 448.0) > 0


@pytest.mark.parametrize("m,loads", SWEEP)
def test_llama4_sweep_full_size_sampled(m, loads):
    """Every point of the Llama-4-style sweep at full size: the forward step
    (e4m3fn) on samples, then the quantisation under e4m3fnuz (exact
    saturation counts of the 448-on-240 mismatch at the smallest and largest
    points of each load shape)."""
    w = wl.llama4_sweep(m, loads)
    check_forward(w, 13 + m + (loads == "zipf"))
    check_fnuz(w, m + 7, exact_mismatch=m in (4096, 131072))


def test_deepseek_moe16b_backward_full_size_sampled():
    """Jagged colwise + transpose of grad_out and X on sampled columns (all
    98304 rows, 64 Zipf groups), then the contraction-jagged dW on sampled
    (expert, row, column) outputs."""
    w = wl.deepseek_moe_16b_backward()
    st = bench.BackwardDwStep(w)
    run_step(st)
    g = np.random.default_rng(14)
    m = st.m
    ld = st.qg.shape[1]
    checked = []
    # the step writes the padded transposed layout: group e at tokens
    # [P_e, P_e + size_e), P_e the earlier sizes rounded up to 128, zero codes
    # up to the next multiple of 128
    starts = np.concatenate([[0], w.offsets[:-1]]).astype(np.int64)
    sizes = w.offsets.astype(np.int64) - starts
    padded = (sizes + 127) // 128 * 128
    p_start = np.concatenate([[0], np.cumsum(padded)[:-1]])
    p_end = int(p_start[-1] + padded[-1])
    assert ld >= p_end
    for src, q_dev, s_dev in ((w.grad_out, st.qg, st.sg), (w.x, st.qx, st.sx)):
        cols = sample(g, src.shape[1], 24, must=[0, src.shape[1] - 1])
        xb = wl.bf16_bits(src[:, torch.from_numpy(cols)])
        q_ref, s_ref, _ = orc.quant_colwise_jagged(xb, w.offsets, orc.TRANSPOSED)
        expect = np.zeros((len(cols), p_end), np.uint8)
        for e in range(len(sizes)):
            expect[:, p_start[e]:p_start[e] + sizes[e]] = q_ref[:, starts[e]:starts[e] + sizes[e]]
        got_q = q_dev[torch.from_numpy(cols).cuda(), :p_end].cpu().numpy()
        assert (got_q == expect).all()
        got_s = s_dev[:, torch.from_numpy(cols).cuda()].cpu().numpy()
        assert (got_s.view(np.uint32) == s_ref.view(np.uint32)).all()
        checked.append((cols, q_ref, s_ref))
    (ci, qa_t, sa), (cj, qb_t, sb) = checked
    ns = 3000
    grp = g.integers(0, st.e, ns)
    li = g.integers(0, len(ci), ns)
    lj = g.integers(0, len(cj), ns)
    c, b = orc.gemm_k_jagged_sample(qa_t, sa, qb_t, sb, w.offsets, m, grp, li, lj)
    out = st.out[torch.from_numpy(grp).cuda(), torch.from_numpy(ci[li]).cuda(),
                 torch.from_numpy(cj[lj]).cuda()]
    got = out.cpu().numpy().astype(np.float64)
    bad = np.nonzero(~(np.abs(got - c) <= b))[0]
    assert bad.size == 0, (bad.size, got[bad[:4]], c[bad[:4]], b[bad[:4]])


def test_deepseek_moe16b_dual_output_full_size():
    """The dual-output quantisation of grad_out [98304, 1408] (64 Zipf groups)
    in the benchmark's launch configuration: identical, byte for byte, to the
    two separate calls it replaces, and equal to the oracle on sampled rows
    (rowwise) and sampled columns over all rows (padded column-wise)."""
    w = wl.deepseek_moe_16b_backward(with_x=False)
    st = bench.DualCompareStep(w)
    run_step(st)
    m, n = st.m, st.n
    assert torch.equal(st.qr2, st.qr) and torch.equal(st.sr2, st.sr)
    starts = np.concatenate([[0], w.offsets[:-1]]).astype(np.int64)
    sizes = w.offsets.astype(np.int64) - starts
    padded = (sizes + 127) // 128 * 128
    p_start = np.concatenate([[0], np.cumsum(padded)[:-1]])
    p_end = int(p_start[-1] + padded[-1])
    assert torch.equal(st.qc2[:, :p_end], st.qc[:, :p_end]) and torch.equal(st.sc2, st.sc)
    g = np.random.default_rng(15)
    rows = sample(g, m, 40, must=[0, m - 1])
    q_ref, s_ref, _ = orc.quant_rowwise(wl.bf16_bits(w.grad_out[torch.from_numpy(rows)]))
    assert (st.qr2[torch.from_numpy(rows).cuda()].cpu().numpy() == q_ref).all()
    assert (st.sr2.cpu().numpy()[rows].view(np.uint32) == s_ref.view(np.uint32)).all()
    cols = sample(g, n, 16, must=[0, n - 1])
    c_ref, cs_ref, _ = orc.quant_colwise_jagged(wl.bf16_bits(w.grad_out[:, torch.from_numpy(cols)]),
                                                w.offsets, orc.TRANSPOSED)
    expect = np.zeros((len(cols), p_end), np.uint8)
    for e in range(len(sizes)):
        expect[:, p_start[e]:p_start[e] + sizes[e]] = c_ref[:, starts[e]:starts[e] + sizes[e]]
    got = st.qc2[torch.from_numpy(cols).cuda(), :p_end].cpu().numpy()
    assert (got == expect).all()
    got_s = st.sc2[:, torch.from_numpy(cols).cuda()].cpu().numpy()
    assert (got_s.view(np.uint32) == cs_ref.view(np.uint32)).all()


def test_llama3_8b_up_projection_mxfp8_full_size_sampled():
    """MXFP8 forward at full size (the benchmark's MxForwardStep): MX rowwise X
    and W on sampled rows, bit-exact with every block scale; the block-scaled
    GEMM on sampled outputs from the oracle's own MX quantisation."""
    w = wl.llama3_8b_up_proj()
    st = bench.MxForwardStep(w)
    run_step(st)
    g = np.random.default_rng(21)
    m, k = w.x.shape
    e, n = w.w.shape[0], w.w.shape[1]
    rows = sample(g, m, 32, must=[0, m - 1])
    qa_ref, sa_ref = orc.mx_quant_rowwise(wl.bf16_bits(w.x[torch.from_numpy(rows)]))
    assert (st.qa[torch.from_numpy(rows).cuda()].cpu().numpy() == qa_ref).all()
    sa_blocks = qgg.mx_scales_to_blocks(st.sa, k // 32)
    assert (sa_blocks[torch.from_numpy(rows).cuda()].cpu().numpy() == sa_ref).all()
    cols = sample(g, n, 32, must=[0, n - 1])
    wsel = w.w[:, torch.from_numpy(cols), :].reshape(e * len(cols), k)
    qb_ref, sb_ref = orc.mx_quant_rowwise(wl.bf16_bits(wsel))
    qb = st.qb.view(e, n, k)[:, torch.from_numpy(cols).cuda(), :].reshape(e * len(cols), k)
    assert (qb.cpu().numpy() == qb_ref).all()
    sb = qgg.mx_scales_to_blocks(st.sb, k // 32).view(e, n, -1)[:, torch.from_numpy(cols).cuda()]
    assert (sb.reshape(e * len(cols), -1).cpu().numpy() == sb_ref).all()
    ns = 2000
    li = g.integers(0, len(rows), ns)
    lj = g.integers(0, len(cols), ns)
    c, b = orc.mx_gemm_m_jagged_sample(qa_ref, sa_ref, qb_ref.reshape(e, len(cols), k),
                                       sb_ref.reshape(e, len(cols), k // 32),
                                       np.array([len(rows)], np.int32), li, lj)
    out = st.out[torch.from_numpy(rows[li]).cuda(), torch.from_numpy(cols[lj]).cuda()]
    got = out.cpu().numpy().astype(np.float64)
    bad = np.nonzero(~(np.abs(got - c) <= b))[0]
    assert bad.size == 0, (bad.size, got[bad[:4]], c[bad[:4]], b[bad[:4]])


def test_deepseek_moe16b_backward_mxfp8_full_size_sampled():
    """MXFP8 weight gradient at full size (the benchmark's MxBackwardDwStep):
    MX quantisation of grad_out and X along each group's tokens on sampled
    columns over all 98304 rows (codes of the whole padded range, gaps
    included, and every scale byte), then the block-scaled contraction-jagged
    dW on sampled (expert, row, column) outputs."""
    w = wl.deepseek_moe_16b_backward()
    st = bench.MxBackwardDwStep(w)
    run_step(st)
    g = np.random.default_rng(22)
    m = st.m
    p_end = orc.padded_len(np.diff(np.concatenate([[0], w.offsets])))
    checked = []
    for src, q_dev, s_dev in ((w.grad_out, st.qg, st.sg), (w.x, st.qx, st.sx)):
        cols = sample(g, src.shape[1], 16, must=[0, src.shape[1] - 1])
        q_ref, s_ref = orc.mx_quant_colwise_padded(wl.bf16_bits(src[:, torch.from_numpy(cols)]),
                                                   w.offsets)
        assert q_ref.shape[1] == p_end
        got_q = q_dev[torch.from_numpy(cols).cuda(), :p_end].cpu().numpy()
        assert (got_q == q_ref).all()
        blocks = qgg.mx_scales_to_blocks(s_dev, p_end // 32)
        got_s = blocks[torch.from_numpy(cols).cuda()].cpu().numpy()
        assert (got_s == s_ref).all()
        checked.append((cols, q_ref, s_ref))
    (ci, qa_t, sa_t), (cj, qb_t, sb_t) = checked
    ns = 3000
    grp = g.integers(0, st.e, ns)
    li = g.integers(0, len(ci), ns)
    lj = g.integers(0, len(cj), ns)
    c, b = orc.mx_gemm_k_jagged_padded_sample(qa_t, sa_t, qb_t, sb_t, w.offsets, m, grp, li, lj)
    out = st.out[torch.from_numpy(grp).cuda(), torch.from_numpy(ci[li]).cuda(),
                 torch.from_numpy(cj[lj]).cuda()]
    got = out.cpu().numpy().astype(np.float64)
    bad = np.nonzero(~(np.abs(got - c) <= b))[0]
    assert bad.size == 0, (bad.size, got[bad[:4]], c[bad[:4]], b[bad[:4]])
