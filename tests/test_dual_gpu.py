"""GPU parity of the dual-output backward quantisation (fp8_quant_dual_jagged):
one read of x gives the rowwise quantisation of every grouped row and the
jagged column-wise quantisation in the padded transposed layout.  Both are
compared bit for bit with the oracle's rowwise and (plain transposed, moved to
the padded positions) column-wise quantisation of the same bf16 input, and
the saturation count with the sum of the oracle's two counts."""
import numpy as np
import pytest
import torch

import oracle as orc
import quantization_grouped_gemm_b200 as qgg
from quantization_grouped_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def rand_bf16(seed, m, cols, outliers=0.0):
    g = np.random.default_rng(seed)
    a = g.standard_normal((m, cols)).astype(np.float32)
    if outliers and a.size:
        idx = g.integers(0, a.size, max(1, int(a.size * outliers)))
        a.reshape(-1)[idx] *= 100
    return wl.to_bf16(a)


def padded_placement(q_t, sizes, width, fill):
    out = np.full((q_t.shape[0], width), fill, np.uint8)
    start, p = 0, 0
    for sz in sizes:
        out[:, p:p + sz] = q_t[:, start:start + sz]
        r = (sz + 127) // 128 * 128
        out[:, p + sz:p + r] = 0
        start, p = start + sz, p + r
    return out


def run_dual(x, sizes, fmt=qgg.E4M3FN, scale_max=0.0, count=False, extra_rows=0):
    """Runs the dual quantisation on x (with `extra_rows` rows past the last
    group) into canary-filled buffers; returns the device results and the
    oracle's."""
    m, cols = x.shape
    e = len(sizes)
    off = wl.offsets_from_sizes(sizes)
    ld_qc = (m + 128 * e + 16 + 15) // 16 * 16
    q_row = torch.full((m, cols), 0xAB, dtype=torch.uint8, device="cuda")
    s_row = torch.full((m,), -7.0, device="cuda")
    q_col = torch.full((cols, ld_qc), 0xAB, dtype=torch.uint8, device="cuda")
    sat = torch.zeros(1, dtype=torch.int64, device="cuda") if count else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qgg.fp8_quant_dual_jagged(x.cuda(), torch.from_numpy(off).cuda(), fmt, scale_max,
                              q_row=q_row, scales_row=s_row, q_col=q_col, sat_count=sat,
                              status=st)
    torch.cuda.synchronize()
    grouped = int(sum(sizes))
    xb = wl.bf16_bits(x)
    r_q, r_s, r_sat = orc.quant_rowwise(xb[:grouped], fmt, scale_max)
    c_q, c_s, c_sat = orc.quant_colwise_jagged(xb, off, orc.TRANSPOSED, fmt, scale_max)
    return dict(q_row=q_row.cpu().numpy(), s_row=s_row.cpu().numpy(), q_col=q_col.cpu().numpy(),
                sat=None if sat is None else int(sat.item()), status=int(st.item()),
                r_q=r_q, r_s=r_s, r_sat=r_sat, c_q=padded_placement(c_q, sizes, ld_qc, 0xAB),
                c_s=c_s, c_sat=c_sat, grouped=grouped)


def check(res, s_col):
    g = res["grouped"]
    assert (res["q_row"][:g] == res["r_q"]).all()
    assert (res["s_row"][:g].view(np.uint32) == res["r_s"].view(np.uint32)).all()
    # rows past the last group end are not written
    assert (res["q_row"][g:] == 0xAB).all() and (res["s_row"][g:] == -7.0).all()
    bad = np.argwhere(res["q_col"] != res["c_q"])
    assert bad.size == 0, (bad.shape, bad[:8])
    assert (s_col.view(np.uint32) == res["c_s"].view(np.uint32)).all()
    assert res["status"] == 0


@pytest.mark.parametrize("sizes,cols,fmt", [
    ([5, 0, 19, 8], 16, qgg.E4M3FN),
    ([0, 1, 15, 17, 0, 33, 128, 129, 255], 72, qgg.E4M3FNUZ),
    ([3000, 70, 700], 1408, qgg.E4M3FN),
    ([20011, 3, 9000, 0, 385], 136, qgg.E4M3FN),
    ([256, 128, 384], 264, qgg.E4M3FN),
    ([1] * 17, 512, qgg.E4M3FNUZ),
    ([0, 0, 0], 64, qgg.E4M3FN),
])
def test_dual_matches_rowwise_and_padded_colwise(sizes, cols, fmt):
    m = int(sum(sizes))
    x = rand_bf16(11 * m + cols, m, cols, outliers=0.002)
    e = len(sizes)
    # the column scales come back through the binding's default buffer
    off = torch.from_numpy(wl.offsets_from_sizes(sizes)).cuda()
    _, _, _, s_col = qgg.fp8_quant_dual_jagged(x.cuda(), off, fmt)
    torch.cuda.synchronize()
    res = run_dual(x, sizes, fmt)
    check(res, s_col.cpu().numpy())
    assert s_col.shape == (e, cols)


def test_dual_rows_past_the_last_group_are_not_written():
    sizes = [300, 0, 41]
    x = rand_bf16(5, sum(sizes) + 77, 96)
    res = run_dual(x, sizes)
    g = res["grouped"]
    assert (res["q_row"][g:] == 0xAB).all() and (res["s_row"][g:] == -7.0).all()
    assert (res["q_row"][:g] == res["r_q"]).all()


@pytest.mark.parametrize("fmt,smax", [(qgg.E4M3FNUZ, 448.0), (qgg.E4M3FN, 0.0),
                                      (qgg.E4M3FNUZ, 0.0)])
def test_dual_saturation_count_is_the_sum_of_both(fmt, smax):
    """With the counter on (and the 448-on-240 mismatch that the counter is
    there to expose) the codes stay bit-exact and the count equals the
    oracle's rowwise count plus its column-wise count."""
    sizes = [700, 3, 0, 260]
    x = rand_bf16(9, sum(sizes), 200, outliers=0.01)
    res = run_dual(x, sizes, fmt, smax, count=True)
    g = res["grouped"]
    assert (res["q_row"][:g] == res["r_q"]).all()
    assert (res["q_col"] == res["c_q"]).all()
    assert res["sat"] == res["r_sat"] + res["c_sat"]
    if smax:
        assert res["sat"] > 0
    else:
        assert res["sat"] == 0
