"""GPU parity of the quantisation kernels against the CPU oracle.

Codes, scales and saturation counts must be bit-exact.  Every call goes
through the C ABI (via the thin binding); expected values come only from the
oracle."""
import numpy as np
import pytest
import torch

import oracle as orc
import quantization_grouped_gemm_b200 as qgg
from quantization_grouped_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
FMTS = [qgg.E4M3FN, qgg.E4M3FNUZ]


def dev(t):
    return t.cuda()


def canon(codes, fmt):
    """Codes with the two e4m3fn NaN codes (0x7F, 0xFF) made one: the sign of a
    NaN is not defined, so either is a correct result where the oracle has 0x7F."""
    c = np.asarray(codes).copy()
    if fmt == qgg.E4M3FN:
        c[c == 0xFF] = 0x7F
    return c


def bits(t):
    return wl.bf16_bits(t.cpu())


def rand_bf16(seed, rows, cols, outliers=0.01, zero_rows=(), zero_cols=()):
    g = np.random.default_rng(seed)
    a = g.standard_normal((rows, cols)).astype(np.float32)
    if outliers and a.size:
        idx = g.integers(0, a.size, max(1, int(a.size * outliers)))
        a.reshape(-1)[idx] *= 100
    for r in zero_rows:
        a[r, :] = 0
    for c in zero_cols:
        a[:, c] = 0
    return wl.to_bf16(a)


# ----------------------------------------------------------------- encoder sweep
@pytest.mark.parametrize("fmt", FMTS)
def test_device_encoder_exhaustive_over_the_active_binades(fmt):
    """Every fp32 bit pattern whose magnitude lies in [2^-12, 2^9) (both signs),
    through fp8_cast_f32, equals the oracle's encode; a sample of the rest too."""
    mant = torch.arange(1 << 23, dtype=torch.int32, device="cuda")
    for exp_field in range(127 - 12, 127 + 9):
        for sign in (0, 1):
            pat = mant | ((sign << 31) | (exp_field << 23))
            y = pat.view(torch.float32)
            q = qgg.fp8_cast_f32(y, fmt).cpu().numpy()
            ref = orc.encode_array(y.cpu().numpy(), fmt)
            bad = np.nonzero(q != ref)[0]
            assert bad.size == 0, (exp_field, sign, [(hex(int(pat[i])), hex(q[i]), hex(ref[i]))
                                                     for i in bad[:5]])
    g = np.random.default_rng(5)
    pats = g.integers(0, 1 << 32, 1 << 22, dtype=np.uint64).astype(np.uint32)
    pats = pats[(pats & 0x7F800000) != 0x7F800000]  # no NaN/Inf
    y = pats.view(np.float32)
    q = qgg.fp8_cast_f32(torch.from_numpy(y).cuda(), fmt).cpu().numpy()
    assert (q == orc.encode_array(y, fmt)).all()
    special = np.array([0.0, -0.0, np.inf, -np.inf, 448.0, -448.0, 240.0, 232.0, -232.0, 464.0,
                        np.nan, -np.nan], np.float32)
    special = np.concatenate([special, np.array([0x7F800001, 0xFFC00001], np.uint32)
                              .view(np.float32)])
    q = qgg.fp8_cast_f32(torch.from_numpy(special).cuda(), fmt).cpu().numpy()
    assert (canon(q, fmt) == orc.encode_array(special, fmt)).all()


@pytest.mark.parametrize("n", [1, 7, 8, 9, 1000, 4099])
def test_cast_ragged_lengths(n):
    g = np.random.default_rng(n)
    y = (g.standard_normal(n) * 50).astype(np.float32)
    for fmt in FMTS:
        q = qgg.fp8_cast_f32(torch.from_numpy(y).cuda(), fmt).cpu().numpy()
        assert (q == orc.encode_array(y, fmt)).all()


# ----------------------------------------------------------------- rowwise
ROW_SHAPES = [(1, 8), (3, 256), (17, 1408), (64, 4096), (33, 7168), (5, 5120), (2, 32768),
              (300, 72), (1000, 2048), (9, 16384)]


@pytest.mark.parametrize("rows,cols", ROW_SHAPES)
@pytest.mark.parametrize("fmt", FMTS)
def test_rowwise_parity(rows, cols, fmt):
    x = rand_bf16(rows * 7 + cols, rows, cols, zero_rows=[0] if rows > 2 else [])
    xb = bits(x)
    q_ref, s_ref, sat_ref = orc.quant_rowwise(xb, fmt)
    sat = torch.zeros(1, dtype=torch.int64, device="cuda")
    q, s = qgg.fp8_quant_rowwise(dev(x), fmt, sat_count=sat)
    torch.cuda.synchronize()
    assert (q.cpu().numpy() == q_ref).all()
    assert (s.cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()
    assert int(sat.item()) == sat_ref == 0


def test_rowwise_strided_input_and_output_leave_padding_untouched():
    rows, cols, ldx, ldq = 37, 1408, 1408 + 64, 1408 + 24
    full = rand_bf16(3, rows, ldx)
    x = dev(full)[:, :cols]
    qbuf = torch.full((rows, ldq), 0xAB, dtype=torch.uint8, device="cuda")
    q, s = qgg.fp8_quant_rowwise(x, q=qbuf[:, :cols],
                                 scales=torch.empty(rows, device="cuda"))
    q_ref, s_ref, _ = orc.quant_rowwise(bits(full)[:, :cols])
    qb = qbuf.cpu().numpy()
    assert (qb[:, :cols] == q_ref).all()
    assert (qb[:, cols:] == 0xAB).all()
    assert (s.cpu().numpy() == s_ref).all()


@pytest.mark.parametrize("fmt", FMTS)
def test_rowwise_every_bf16_value_at_unit_scale(fmt):
    """All finite bf16 values within +-fmax, with fmax itself in every row so that
    s = fmax / fmax = 1: the codes are the encoder applied to x."""
    fmax = orc.fp8_max(fmt)
    pats = np.arange(65536, dtype=np.uint32)
    vals = (pats << 16).view(np.float32)
    keep = np.isfinite(vals) & (np.abs(vals) <= fmax)
    p16 = pats[keep].astype(np.uint16)
    per = 255
    nrows = (p16.size + per - 1) // per
    grid = np.full((nrows, per + 1), 0, np.uint16)
    body = np.zeros(nrows * per, np.uint16)
    body[: p16.size] = p16
    grid[:, :per] = body.reshape(nrows, per)
    grid[:, per] = (np.array([fmax], np.float32).view(np.uint32) >> 16).astype(np.uint16)
    x = torch.from_numpy(grid.view(np.int16)).view(torch.bfloat16)
    q_ref, s_ref, _ = orc.quant_rowwise(grid, fmt)
    assert (s_ref == 1.0).all()
    q, s = qgg.fp8_quant_rowwise(dev(x), fmt)
    assert (q.cpu().numpy() == q_ref).all()
    assert (s.cpu().numpy() == 1.0).all()


@pytest.mark.parametrize("fmt", FMTS)
def test_rowwise_special_values_match_the_oracle(fmt):
    """Rows holding NaNs (ignored by the absmax, like the oracle's comparison),
    all-NaN rows, infinities (scale 0), signed zeros and subnormal-only rows."""
    rows, cols = 12, 1408
    g = np.random.default_rng(21 + fmt)
    a = wl.bf16_bits(rand_bf16(6, rows, cols)).copy()
    a[0, ::97] = 0x7FC1
    a[1, 5::89] = 0xFFC0
    a[2, :] = 0x7F81                                   # all NaN
    a[3, 17] = 0x7F80                                  # +inf
    a[4, 99] = 0xFF80                                  # -inf
    a[5, :] = 0x8000                                   # -0
    a[6, :] = g.integers(1, 0x80, cols).astype(np.uint16)          # subnormals
    a[7, :] = g.integers(1, 0x80, cols).astype(np.uint16) | 0x8000
    a[8, :] = 0x0001
    a[9, ::2] = 0x7FC0
    a[9, 1::2] = 0x0003
    x = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    q_ref, s_ref, _ = orc.quant_rowwise(a, fmt)
    q, s = qgg.fp8_quant_rowwise(dev(x), fmt)
    assert (canon(q.cpu().numpy(), fmt) == q_ref).all()
    assert (s.cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()
    sat = torch.zeros(1, dtype=torch.int64, device="cuda")  # the clamping (slow) kernel too
    q2, s2 = qgg.fp8_quant_rowwise(dev(x), fmt, sat_count=sat)
    assert (canon(q2.cpu().numpy(), fmt) == q_ref).all()
    assert (s2.cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()


@pytest.mark.parametrize("fmt,smax", [(qgg.E4M3FNUZ, 448.0), (qgg.E4M3FN, 240.0)])
def test_rowwise_format_mismatch_is_counted_like_the_oracle(fmt, smax):
    x = rand_bf16(77, 64, 512, outliers=0.0)
    q_ref, s_ref, sat_ref = orc.quant_rowwise(bits(x), fmt, scale_max=smax)
    sat = torch.zeros(1, dtype=torch.int64, device="cuda")
    q, s = qgg.fp8_quant_rowwise(dev(x), fmt, scale_max=smax, sat_count=sat)
    assert (q.cpu().numpy() == q_ref).all()
    assert (s.cpu().numpy() == s_ref).all()
    assert int(sat.item()) == sat_ref
    if fmt == qgg.E4M3FNUZ:
        assert sat_ref > 0
    else:
        assert sat_ref == 0


def test_rowwise_zero_rows_is_a_no_op():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q, s = qgg.fp8_quant_rowwise(x)
    assert q.shape == (0, 64) and s.shape == (0,)


# ----------------------------------------------------------------- jagged colwise
COL_CASES = [
    ([5, 0, 19, 8], 16),
    ([0, 1, 15, 17, 0, 33], 72),
    ([511, 512, 513], 64),
    ([1500, 0, 3], 200),
    ([2000], 8),
    ([0, 0, 0], 64),
    ([1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1], 128),
    ([3000, 70, 700], 1408),
]


@pytest.mark.parametrize("sizes,cols", COL_CASES)
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("layout", [qgg.LAYOUT_SAME, qgg.LAYOUT_TRANSPOSED])
def test_colwise_parity(sizes, cols, fmt, layout):
    m = int(sum(sizes))
    x = rand_bf16(m + cols + len(sizes), m, cols, zero_cols=[cols // 2] if cols > 2 else [])
    off = wl.offsets_from_sizes(sizes)
    ld = (m + 16 + 15) // 16 * 16 if layout == qgg.LAYOUT_TRANSPOSED else cols
    q_ref, s_ref, sat_ref = orc.quant_colwise_jagged(bits(x), off, layout, fmt, ld_q=ld,
                                                     fill=0xAB)
    if layout == qgg.LAYOUT_TRANSPOSED:
        qbuf = torch.full((cols, ld), 0xAB, dtype=torch.uint8, device="cuda")
    else:
        qbuf = torch.full((m, cols), 0xAB, dtype=torch.uint8, device="cuda")
    sat = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, s = qgg.fp8_quant_colwise_jagged(dev(x), torch.from_numpy(off).cuda(), layout, fmt,
                                        q=qbuf, sat_count=sat, status=st)
    torch.cuda.synchronize()
    qn = q.cpu().numpy()
    bad = np.argwhere(qn != q_ref)
    assert bad.size == 0, bad[:10]
    assert (s.cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()
    assert int(sat.item()) == sat_ref == 0
    assert int(st.item()) == 0


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("layout", [qgg.LAYOUT_SAME, qgg.LAYOUT_TRANSPOSED])
@pytest.mark.parametrize("sizes", [[100, 0, 150, 50], [900, 20]])
def test_colwise_special_values_match_the_oracle(sizes, layout, fmt):
    """Columns whose group absmax is a subnormal, signed zeros, infinities and
    NaNs with several payloads: the absmax and the codes follow the oracle
    bit for bit (the second size list takes the path that merges chunks)."""
    m, cols = sum(sizes), 64
    g = np.random.default_rng(sum(sizes) + layout + 7 * fmt)
    a = wl.bf16_bits(rand_bf16(5, m, cols)).copy()
    sub = g.integers(1, 0x80, (m, 8)).astype(np.uint16)           # positive subnormals
    a[:, 0:8] = sub | (g.integers(0, 2, (m, 8)).astype(np.uint16) << 15)
    a[:, 8] = 0x8000                                                # -0 everywhere
    a[:, 9] = 0x0000
    a[::37, 10] = 0x7F80                                            # +inf
    a[5::41, 11] = 0xFF80                                           # -inf
    a[::53, 12] = 0x7FC1                                            # NaN payloads
    a[7::59, 13] = 0xFFC0
    a[3::61, 14] = 0x7F81
    a[:, 15] = 0x7F7F                                               # largest finite
    a[1::2, 15] = 0x0001
    x = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    off = wl.offsets_from_sizes(sizes)
    ld = (m + 15) // 16 * 16 if layout == qgg.LAYOUT_TRANSPOSED else cols
    q_ref, s_ref, _ = orc.quant_colwise_jagged(a, off, layout, fmt, ld_q=ld, fill=0xAB)
    shape = (cols, ld) if layout == qgg.LAYOUT_TRANSPOSED else (m, cols)
    qbuf = torch.full(shape, 0xAB, dtype=torch.uint8, device="cuda")
    for sat in (None, torch.zeros(1, dtype=torch.int64, device="cuda")):
        qbuf.fill_(0xAB)
        q, s = qgg.fp8_quant_colwise_jagged(dev(x), torch.from_numpy(off).cuda(), layout, fmt,
                                            q=qbuf, sat_count=sat)
        torch.cuda.synchronize()
        bad = np.argwhere(canon(q.cpu().numpy(), fmt) != q_ref)
        assert bad.size == 0, bad[:10]
        assert (s.cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()


def test_colwise_transposed_equals_transpose_of_same_layout():
    sizes = [700, 1, 0, 1200, 45]
    m, cols = sum(sizes), 136
    x = dev(rand_bf16(9, m, cols))
    off = torch.from_numpy(wl.offsets_from_sizes(sizes)).cuda()
    q1, s1 = qgg.fp8_quant_colwise_jagged(x, off, qgg.LAYOUT_SAME)
    q2, s2 = qgg.fp8_quant_colwise_jagged(x, off, qgg.LAYOUT_TRANSPOSED)
    assert torch.equal(q2[:, :m], q1.t())
    assert torch.equal(s1, s2)


def test_colwise_malformed_offsets_are_clamped_and_reported():
    m, cols = 100, 64
    x = rand_bf16(11, m, cols)
    off = np.array([5, 3, 200, -1], np.int32)
    q_ref, s_ref, _ = orc.quant_colwise_jagged(bits(x), off, orc.SAME)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, s = qgg.fp8_quant_colwise_jagged(dev(x), torch.from_numpy(off).cuda(), status=st)
    assert (q.cpu().numpy() == q_ref).all()
    assert (s.cpu().numpy() == s_ref).all()
    assert int(st.item()) & qgg.STATUS_BAD_OFFSETS


def test_colwise_rows_past_last_offset_are_not_written():
    m, cols = 300, 64
    x = rand_bf16(12, m, cols)
    off = np.array([100, 250], np.int32)
    qbuf = torch.full((m, cols), 0xAB, dtype=torch.uint8, device="cuda")
    q, _ = qgg.fp8_quant_colwise_jagged(dev(x), torch.from_numpy(off).cuda(), q=qbuf)
    q_ref, _, _ = orc.quant_colwise_jagged(bits(x), off, orc.SAME, fill=0xAB)
    assert (q.cpu().numpy() == q_ref).all()
    assert (q.cpu().numpy()[250:] == 0xAB).all()


def test_colwise_workspace_is_reusable_across_calls():
    sizes = [2500, 10, 1800]
    m, cols = sum(sizes), 256
    off = torch.from_numpy(wl.offsets_from_sizes(sizes)).cuda()
    ws = torch.full((qgg.colwise_workspace_bytes(m, cols, 3),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    outs = []
    for seed in (1, 2, 1):
        x = dev(rand_bf16(seed, m, cols))
        outs.append(qgg.fp8_quant_colwise_jagged(x, off, qgg.LAYOUT_TRANSPOSED, workspace=ws))
    assert torch.equal(outs[0][0][:, :m], outs[2][0][:, :m])
    assert torch.equal(outs[0][1], outs[2][1])
    x = rand_bf16(2, m, cols)
    q_ref, s_ref, _ = orc.quant_colwise_jagged(bits(x), off.cpu().numpy(), orc.TRANSPOSED,
                                               ld_q=outs[1][0].shape[1])
    assert (outs[1][0].cpu().numpy()[:, :m] == q_ref[:, :m]).all()
    assert (outs[1][1].cpu().numpy() == s_ref).all()


@pytest.mark.parametrize("fmt,smax", [(qgg.E4M3FNUZ, 448.0), (qgg.E4M3FN, 240.0)])
def test_colwise_format_mismatch_is_counted_like_the_oracle(fmt, smax):
    sizes = [600, 0, 90]
    x = rand_bf16(13, sum(sizes), 64, outliers=0.0)
    off = wl.offsets_from_sizes(sizes)
    q_ref, s_ref, sat_ref = orc.quant_colwise_jagged(bits(x), off, orc.SAME, fmt,
                                                     scale_max=smax)
    sat = torch.zeros(1, dtype=torch.int64, device="cuda")
    q, s = qgg.fp8_quant_colwise_jagged(dev(x), torch.from_numpy(off).cuda(), fmt=fmt,
                                        scale_max=smax, sat_count=sat)
    assert (q.cpu().numpy() == q_ref).all()
    assert (s.cpu().numpy() == s_ref).all()
    assert int(sat.item()) == sat_ref


def padded_placement(q_t, off, ld_p, fill):
    """The oracle's transposed codes at the padded layout's positions: group e
    at tokens [P_e, P_e + size_e) with P_e the sum of the earlier sizes rounded
    up to 128, zero codes up to P_e + round_up(size_e, 128), `fill` after."""
    out = np.full((q_t.shape[0], ld_p), fill, np.uint8)
    start, p = 0, 0
    for end in np.asarray(off, np.int64):
        sz = int(end) - start
        out[:, p:p + sz] = q_t[:, start:int(end)]
        r = (sz + 127) // 128 * 128
        out[:, p + sz:p + r] = 0
        start, p = int(end), p + r
    return out


@pytest.mark.parametrize("sizes,cols,fmt", [
    ([5, 0, 19, 8], 16, qgg.E4M3FN),
    ([0, 1, 15, 17, 0, 33, 128, 129, 255], 72, qgg.E4M3FNUZ),
    ([20011, 3, 9000, 0, 385], 136, qgg.E4M3FN),
    ([3000, 70, 700], 1408, qgg.E4M3FN),
    ([1] * 17, 128, qgg.E4M3FN),
    ([0, 0, 0], 64, qgg.E4M3FN),
])
def test_colwise_padded_transposed_layout(sizes, cols, fmt):
    """Every group at a 128-token boundary, zero codes to the next boundary and
    nothing written past the last group; codes and scales bit-exact with the
    oracle's plain transposed layout moved to those positions.  The tall groups
    go through the chunked path, whose rows then start at the group's first row."""
    m = int(sum(sizes))
    e = len(sizes)
    x = rand_bf16(7 * m + cols, m, cols, outliers=0.002)
    off = wl.offsets_from_sizes(sizes)
    ld = (m + 128 * e + 16 + 15) // 16 * 16
    q_t, s_ref, _ = orc.quant_colwise_jagged(bits(x), off, orc.TRANSPOSED, fmt)
    expect = padded_placement(q_t, off, ld, 0xAB)
    qbuf = torch.full((cols, ld), 0xAB, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, s = qgg.fp8_quant_colwise_jagged(dev(x), torch.from_numpy(off).cuda(),
                                        qgg.LAYOUT_TRANSPOSED_PADDED, fmt, q=qbuf, status=st)
    qn = q.cpu().numpy()
    bad = np.argwhere(qn != expect)
    assert bad.size == 0, (bad.shape, bad[:10])
    assert (s.cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()
    assert int(st.item()) == 0


@pytest.mark.parametrize("layout", [qgg.LAYOUT_SAME, qgg.LAYOUT_TRANSPOSED])
def test_colwise_tall_groups_split_over_many_blocks(layout):
    """Groups of 20k and 9k rows: cut into 45 and 21 chunks per 64-column tile,
    spread over the blocks, which merge their partial absmax in the workspace."""
    sizes = [20011, 3, 9000, 0, 385]
    m, cols = sum(sizes), 136
    x = rand_bf16(31, m, cols, outliers=0.001)
    off = wl.offsets_from_sizes(sizes)
    ld = (m + 15) // 16 * 16
    q_ref, s_ref, _ = orc.quant_colwise_jagged(bits(x), off, layout, ld_q=ld if layout else None)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, s = qgg.fp8_quant_colwise_jagged(dev(x), torch.from_numpy(off).cuda(), layout,
                                        ld_q=ld, status=st)
    qn = q.cpu().numpy()
    if layout == qgg.LAYOUT_TRANSPOSED:
        qn, q_ref = qn[:, :m], q_ref[:, :m]
    assert (qn == q_ref).all()
    assert (s.cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()
    assert int(st.item()) == 0


@pytest.mark.parametrize("layout", [qgg.LAYOUT_SAME, qgg.LAYOUT_TRANSPOSED])
def test_colwise_single_group_of_seventy_thousand_rows(layout):
    """No group-height limit: one 70,003-row group (157 chunks per column tile,
    each read once for its absmax and once, from L2, for its cast)."""
    m, cols = 70003, 40
    x = rand_bf16(41, m, cols, outliers=0.0005)
    off = np.array([m], np.int32)
    ld = (m + 15) // 16 * 16
    q_ref, s_ref, _ = orc.quant_colwise_jagged(bits(x), off, layout, ld_q=ld if layout else None)
    q, s = qgg.fp8_quant_colwise_jagged(dev(x), torch.from_numpy(off).cuda(), layout, ld_q=ld)
    qn = q.cpu().numpy()
    if layout == qgg.LAYOUT_TRANSPOSED:
        qn, q_ref = qn[:, :m], q_ref[:, :m]
    assert (qn == q_ref).all()
    assert (s.cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()
