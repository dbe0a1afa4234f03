"""GPU parity of the MXFP8 path (OCP MX v1.0 reading of the MXFP8 format that
"AMD Primus adds FP8/MXFP8 kernels ..." names in "What Primus adds for MoE
training on MI355X") through the C ABI: the MX quantisation kernels bit for
bit against the oracle, the MX grouped GEMM on every element within
1e-3 * sum |a||b| of the oracle's fp64 sum over the oracle's own
quantisation of the same bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle as orc
import quantization_grouped_gemm_b200 as qgg
from quantization_grouped_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def spread_bf16(seed, shape, block_axis=-1, spread=12.0, outliers=0.0):
    """N(0,1) values whose 32-element blocks along block_axis carry magnitudes
    2^U(-spread, spread): a block scale applied to the wrong block shows."""
    g = np.random.default_rng(seed)
    a = g.standard_normal(shape)
    n = shape[block_axis]
    nb = (n + 31) // 32
    mag_shape = list(shape)
    mag_shape[block_axis] = nb
    mags = np.exp2(g.uniform(-spread, spread, mag_shape))
    mags = np.repeat(mags, 32, axis=block_axis)
    idx = [slice(None)] * len(shape)
    idx[block_axis] = slice(0, n)
    a = a * mags[tuple(idx)]
    if outliers:
        k = max(1, int(a.size * outliers))
        pos = g.integers(0, a.size, k)
        a.reshape(-1)[pos] *= 300.0
    return wl.to_bf16(a.astype(np.float32))


CANARY = -842150451  # 0xCDCDCDCD


def bits(x):
    return wl.bf16_bits(x)


# --------------------------------------------------------------------------- rowwise
@pytest.mark.parametrize("rows,cols", [(1, 32), (7, 64), (33, 96), (130, 256), (5, 288),
                                       (300, 1024), (3, 4096), (1000, 160)])
def test_mx_rowwise_bit_exact(rows, cols):
    x = spread_bf16(rows * 7 + cols, (rows, cols), outliers=0.01)
    q, s = qgg.fp8_mx_quant_rowwise(x.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = orc.mx_quant_rowwise(bits(x))
    assert (q.cpu().numpy() == q_ref).all()
    blocks = qgg.mx_scales_to_blocks(s, 4 * s.shape[0]).cpu().numpy()
    assert (blocks[:, :cols // 32] == s_ref).all()
    assert (blocks[:, cols // 32:] == 0).all()  # bytes past the row's last block


def test_mx_rowwise_special_values():
    """Zero blocks, bf16 subnormals, huge magnitudes, infinities and NaN."""
    g = np.random.default_rng(3)
    rows = []
    for mag in [1.0, 1e-39, 1e-30, 1e30, 3e38]:
        rows.append(g.standard_normal(64) * mag)
    r = np.zeros(64)
    r[40] = 1.0
    rows.append(r)
    r = g.standard_normal(64)
    r[3] = np.inf
    r[40] = -np.inf
    rows.append(r)
    r = g.standard_normal(64)
    r[7] = np.nan
    r[32:] = np.nan
    rows.append(r)
    with np.errstate(over="ignore"):
        x = wl.to_bf16(np.stack(rows).astype(np.float32))
    q, s = qgg.fp8_mx_quant_rowwise(x.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = orc.mx_quant_rowwise(bits(x))
    qd = q.cpu().numpy()
    nan = np.isnan(x.float().numpy())
    assert (qgg.mx_scales_to_blocks(s, 2).cpu().numpy() == s_ref).all()
    assert (qd[~nan] == q_ref[~nan]).all()
    # a NaN input gives a NaN code (0x7F or 0xFF)
    assert ((qd[nan] & 0x7F) == 0x7F).all()


def test_mx_rowwise_strided_input_and_untouched_padding():
    base = spread_bf16(5, (40, 200))
    x = base[:, 8:168]  # 160 columns, row stride 200
    q = torch.full((40, 168), 0xAB, dtype=torch.uint8, device="cuda")
    s = torch.full((3, 44), CANARY, dtype=torch.int32, device="cuda")  # 2 groups, ld_sw 44
    qgg.fp8_mx_quant_rowwise(x.cuda(), q=q[:, :160], scales=s[:2])
    torch.cuda.synchronize()
    q_ref, s_ref = orc.mx_quant_rowwise(bits(x.contiguous()))
    assert (q.cpu().numpy()[:, :160] == q_ref).all()
    assert (q.cpu().numpy()[:, 160:] == 0xAB).all()
    assert (qgg.mx_scales_to_blocks(s[:2, :40], 5).cpu().numpy() == s_ref).all()
    assert (s[:2, 40:] == CANARY).all() and (s[2] == CANARY).all()


# --------------------------------------------------------------------------- colwise
@pytest.mark.parametrize("sizes,cols", [
    ([5, 0, 19, 8], 16),
    ([0, 1, 31, 32, 33, 0, 129, 255, 256], 72),
    ([3000, 70, 700], 264),
    ([20011, 3, 385], 136),
    ([1] * 17, 512),
    ([0, 0, 0], 64),
    ([128, 256], 8),
])
def test_mx_colwise_padded_bit_exact(sizes, cols):
    m = int(sum(sizes))
    extra = 37
    x = spread_bf16(m + cols, (m + extra, cols), block_axis=0, outliers=0.002)
    off = wl.offsets_from_sizes(sizes)
    e = len(sizes)
    ld_q = (m + extra + 128 * e + 127) // 128 * 128
    q = torch.full((cols, ld_q), 0xAB, dtype=torch.uint8, device="cuda")
    s = torch.full((ld_q // 128, cols), CANARY, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qgg.fp8_mx_quant_colwise_padded(x.cuda(), torch.from_numpy(off).cuda(), q=q, scales=s,
                                    status=st)
    torch.cuda.synchronize()
    q_ref, s_ref = orc.mx_quant_colwise_padded(bits(x), off, ld_q=ld_q, fill=0xAB,
                                               scale_fill=0xCD)
    bad = np.argwhere(q.cpu().numpy() != q_ref)
    assert bad.size == 0, (bad.shape, bad[:8])
    assert (qgg.mx_scales_to_blocks(s, ld_q // 32).cpu().numpy() == s_ref).all()
    assert int(st.item()) == 0


# --------------------------------------------------------------------------- GEMM
def mx_operands_m_jagged(seed, sizes, n, k):
    m = int(sum(sizes))
    e = len(sizes)
    x = spread_bf16(seed, (m, k), spread=10.0)
    w = spread_bf16(seed + 1, (e * n, k), spread=10.0)
    return x, w


def check_m_jagged(sizes, n, k, out_dtype=torch.float32, seed=1, full=True):
    e = len(sizes)
    x, w = mx_operands_m_jagged(seed, sizes, n, k)
    m = x.shape[0]
    off = wl.offsets_from_sizes(sizes)
    qa, sa = qgg.fp8_mx_quant_rowwise(x.cuda())
    qb, sb = qgg.fp8_mx_quant_rowwise(w.cuda())
    out = torch.full((m + 5, n), float("nan"), dtype=out_dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qgg.fp8_mx_grouped_gemm(qgg.M_JAGGED, qa, sa, qb.view(e, n, k), sb,
                            torch.from_numpy(off).cuda(), out=out[:m], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    oqa, osa = orc.mx_quant_rowwise(bits(x))
    oqb, osb = orc.mx_quant_rowwise(bits(w))
    if full:
        rows = np.repeat(np.arange(m), n)
        cols = np.tile(np.arange(n), m)
    else:
        g = np.random.default_rng(seed)
        rows = g.integers(0, m, 3000)
        cols = g.integers(0, n, 3000)
    ref, bound = orc.mx_gemm_m_jagged_sample(oqa, osa, oqb.reshape(e, n, k),
                                             osb.reshape(e, n, k // 32), off, rows, cols)
    got = out.float().cpu().numpy()
    val = got[rows, cols].astype(np.float64)
    if out_dtype == torch.bfloat16:
        bound = bound + np.abs(ref) * 2.0 ** -8
    err = np.abs(val - ref)
    assert (err <= bound).all(), (err.max(), bound[np.argmax(err - bound)])
    # rows past the group ends are not written
    assert np.isnan(got[m:]).all()
    return err, bound


@pytest.mark.parametrize("sizes,n,k", [
    ([5, 0, 19, 8], 32, 64),
    ([300, 1, 129], 96, 160),        # K tail: 160 = 128 + 32
    ([0, 257, 0, 64], 224, 256),
    ([200, 200], 448, 128),          # two full 224-column tiles
    ([130, 7], 200, 96),             # N tail inside the tile (a 208-column tile)
    ([1000], 64, 512),
    ([260, 0, 33], 240, 128),        # one 240-column tile: its last 16 columns loaded alone
    ([64, 200], 480, 96),            # two 240-column tiles
])
def test_mx_gemm_m_jagged_every_element(sizes, n, k):
    check_m_jagged(sizes, n, k)


def test_mx_gemm_m_jagged_bf16_output():
    check_m_jagged([70, 0, 300], 96, 256, out_dtype=torch.bfloat16)


def test_mx_gemm_m_jagged_many_tiles_wraps_the_persistent_grid():
    # 64 groups x 2 M tiles x 5 N tiles = 640 tiles > one per SM
    check_m_jagged([200] * 64, 1120, 128, seed=5, full=False)


def check_k_jagged(sizes, n1, n2, out_dtype=torch.float32, seed=3):
    m = int(sum(sizes))
    e = len(sizes)
    go = spread_bf16(seed, (m, n1), block_axis=0, spread=8.0)
    xx = spread_bf16(seed + 1, (m, n2), block_axis=0, spread=8.0)
    off = wl.offsets_from_sizes(sizes)
    offd = torch.from_numpy(off).cuda()
    qa, sa = qgg.fp8_mx_quant_colwise_padded(go.cuda(), offd)
    qb, sb = qgg.fp8_mx_quant_colwise_padded(xx.cuda(), offd)
    out = torch.full((e, n1, n2), float("nan"), dtype=out_dtype, device="cuda")
    qgg.fp8_mx_grouped_gemm(qgg.K_JAGGED_PADDED, qa, sa, qb, sb, offd, m_total=m, out=out)
    torch.cuda.synchronize()
    oqa, osa = orc.mx_quant_colwise_padded(bits(go), off)
    oqb, osb = orc.mx_quant_colwise_padded(bits(xx), off)
    grp, rows, cols = np.meshgrid(np.arange(e), np.arange(n1), np.arange(n2), indexing="ij")
    ref, bound = orc.mx_gemm_k_jagged_padded_sample(oqa, osa, oqb, osb, off, m, grp.ravel(),
                                                    rows.ravel(), cols.ravel())
    got = out.float().cpu().numpy().ravel().astype(np.float64)
    if out_dtype == torch.bfloat16:
        bound = bound + np.abs(ref) * 2.0 ** -8
    err = np.abs(got - ref)
    assert (err <= bound).all(), (err.max(), np.argmax(err - bound))
    for g_, sz in enumerate(sizes):
        if sz == 0:
            assert (out[g_] == 0).all()


@pytest.mark.parametrize("sizes,n1,n2", [
    ([5, 0, 19, 8], 32, 64),
    ([0, 1, 31, 32, 33, 129, 255], 128, 96),
    ([700, 3000], 136, 224),
    ([300, 300], 256, 448),
    ([300, 0, 129], 96, 200),        # a 208-column tile: its last 16 columns loaded alone
    ([200, 70], 128, 464),           # two 240-column tiles, the second cut at the edge
])
def test_mx_gemm_k_jagged_padded_every_element(sizes, n1, n2):
    check_k_jagged(sizes, n1, n2)


def test_mx_gemm_k_jagged_padded_bf16_output():
    check_k_jagged([100, 0, 257], 64, 128, out_dtype=torch.bfloat16)


@pytest.mark.parametrize("sizes,n_w,k_w", [([70, 0, 200], 256, 192), ([33, 300], 128, 96)])
def test_mx_input_gradient_path(sizes, n_w, k_w):
    """dX = grad_out W_e in MXFP8: grad_out quantised along its N columns
    (rowwise), W [E*N, K] quantised along each expert's N rows by the
    column-wise kernel with groups of N rows (W_e^T codes, experts side by
    side in every row, scale words of expert e from group e*N/128), then the
    token-jagged block-scaled GEMM with B interleaved."""
    e = len(sizes)
    m = int(sum(sizes))
    go = spread_bf16(17 + m, (m, n_w), spread=8.0)
    wt = spread_bf16(19 + m, (e * n_w, k_w), block_axis=0, spread=8.0)
    off = wl.offsets_from_sizes(sizes)
    off_w = wl.offsets_from_sizes([n_w] * e)
    qg, sg = qgg.fp8_mx_quant_rowwise(go.cuda())
    qwt, swt = qgg.fp8_mx_quant_colwise_padded(wt.cuda(), torch.from_numpy(off_w).cuda())
    ld_q = qwt.shape[1]
    b = qwt.as_strided((e, k_w, n_w), (n_w, ld_q, 1))
    out = torch.full((m, k_w), float("nan"), device="cuda")
    qgg.fp8_mx_grouped_gemm(qgg.M_JAGGED, qg, sg, b, swt, torch.from_numpy(off).cuda(), out=out,
                            scale_b_group_stride=(n_w // 128) * swt.stride(0))
    torch.cuda.synchronize()
    oqg, osg = orc.mx_quant_rowwise(bits(go))
    oqw, osw = orc.mx_quant_colwise_padded(bits(wt), off_w)
    qb = np.stack([oqw[:, i * n_w:(i + 1) * n_w] for i in range(e)])               # [E, K, N]
    sb = np.stack([osw[:, i * n_w // 32:(i + 1) * n_w // 32] for i in range(e)])   # [E, K, N/32]
    rows = np.repeat(np.arange(m), k_w)
    cols = np.tile(np.arange(k_w), m)
    ref, bound = orc.mx_gemm_m_jagged_sample(oqg, osg, qb, sb, off, rows, cols)
    got = out.cpu().numpy()[rows, cols].astype(np.float64)
    err = np.abs(got - ref)
    assert (err <= bound).all(), (err.max(), np.argmax(err - bound))


@pytest.mark.parametrize("sizes,cols", [
    ([5, 0, 19, 8], 32),
    ([0, 1, 31, 32, 33, 0, 129, 255, 256], 96),
    ([3000, 70, 700], 288),
    ([20011, 3, 385], 128),
    ([0, 0, 0], 64),
])
def test_mx_dual_matches_rowwise_and_padded_colwise(sizes, cols):
    """One read gives the MX rowwise codes of every grouped row and the MX
    padded column-wise codes, each bit-exact against the oracle; rows past
    the last group are not written."""
    m = int(sum(sizes))
    extra = 21
    x = spread_bf16(7 * m + cols, (m + extra, cols), block_axis=0, outliers=0.002)
    off = wl.offsets_from_sizes(sizes)
    e = len(sizes)
    ld_q = (m + extra + 128 * e + 127) // 128 * 128
    q_row = torch.full((m + extra, cols), 0xAB, dtype=torch.uint8, device="cuda")
    s_row = torch.full(((cols + 127) // 128, m + extra), CANARY, dtype=torch.int32, device="cuda")
    q_col = torch.full((cols, ld_q), 0xAB, dtype=torch.uint8, device="cuda")
    s_col = torch.full((ld_q // 128, cols), CANARY, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qgg.fp8_mx_quant_dual_padded(x.cuda(), torch.from_numpy(off).cuda(), q_row=q_row,
                                 scales_row=s_row, q_col=q_col, scales_col=s_col, status=st)
    torch.cuda.synchronize()
    xb = bits(x)
    r_q, r_s = orc.mx_quant_rowwise(xb[:m])
    c_q, c_s = orc.mx_quant_colwise_padded(xb, off, ld_q=ld_q, fill=0xAB, scale_fill=0xCD)
    qr = q_row.cpu().numpy()
    assert (qr[:m] == r_q).all()
    assert (qr[m:] == 0xAB).all()
    blocks = qgg.mx_scales_to_blocks(s_row, 4 * s_row.shape[0]).cpu().numpy()
    assert (blocks[:m, :cols // 32] == r_s).all()
    assert (s_row[:, m:] == CANARY).all()
    assert (q_col.cpu().numpy() == c_q).all()
    assert (qgg.mx_scales_to_blocks(s_col, ld_q // 32).cpu().numpy() == c_s).all()
    assert int(st.item()) == 0
