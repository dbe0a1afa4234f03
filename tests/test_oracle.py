"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: every expected value comes from
a hand-worked fixture (tests/golden), from an independent library (torch's
float8 dtypes, numpy fp64 matmul), from a closed form or from an invariant.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from quantization_grouped_gemm_b200 import workloads as wl
from tests import golden_io as gio

FN, FNUZ = orc.E4M3FN, orc.E4M3FNUZ
TORCH_FP8 = {FN: torch.float8_e4m3fn, FNUZ: torch.float8_e4m3fnuz}


def torch_decode(codes, fmt):
    t = torch.from_numpy(np.asarray(codes, np.uint8)).view(TORCH_FP8[fmt])
    return t.to(torch.float64).numpy()


def torch_encode(y, fmt):
    t = torch.from_numpy(np.ascontiguousarray(y, np.float32))
    return t.to(TORCH_FP8[fmt]).view(torch.uint8).numpy()


def bits_of(values):
    return wl.bf16_bits(torch.tensor(values, dtype=torch.float32).to(torch.bfloat16))


# --------------------------------------------------------------------------- decode
@pytest.mark.parametrize("fmt", [FN, FNUZ])
def test_decode_table_matches_torch_float8(fmt):
    ours = orc.decode_table(fmt)
    ref = torch_decode(np.arange(256), fmt)
    nan_o, nan_r = np.isnan(ours), np.isnan(ref)
    assert (nan_o == nan_r).all()
    assert (ours[~nan_o] == ref[~nan_r]).all()
    # signed zero is part of the format definition
    assert (np.signbit(ours[~nan_o]) == np.signbit(ref[~nan_r])).all()


def test_decode_facts_fixture():
    for r in gio.rows("format_facts.txt"):
        if r[0] == "count_finite":
            fmt = gio.FMT[r[1]]
            assert int(np.isfinite(orc.decode_table(fmt)).sum()) == int(r[2])
            continue
        fmt, code = gio.FMT[r[0]], int(r[1], 16)
        v = orc.decode(code, fmt)
        if r[2] == "nan":
            assert math.isnan(v), (r, v)
        else:
            assert v == float(r[2]) and math.copysign(1, v) == math.copysign(1, float(r[2])), (r, v)


def test_fnuz_has_single_nan_and_no_negative_zero():
    t = orc.decode_table(FNUZ)
    assert [c for c in range(256) if math.isnan(t[c])] == [0x80]
    assert not any(t[c] == 0 and math.copysign(1, t[c]) < 0 for c in range(256))
    assert np.nanmax(t) == 240.0 and np.nanmin(t) == -240.0


def test_fn_nan_codes_and_extremes():
    t = orc.decode_table(FN)
    assert [c for c in range(256) if math.isnan(t[c])] == [0x7F, 0xFF]
    assert np.nanmax(t) == 448.0 and np.nanmin(t) == -448.0


# --------------------------------------------------------------------------- encode
def test_encode_special_cases_fixture():
    for r in gio.rows("encode_special_cases.txt"):
        fmt, y, code = gio.FMT[r[0]], float(r[1]), int(r[2], 16)
        assert orc.encode(y, fmt) == code, r


@pytest.mark.parametrize("fmt", [FN, FNUZ])
def test_encode_roundtrips_every_finite_code(fmt):
    t = orc.decode_table(fmt)
    for c in range(256):
        if math.isnan(t[c]):
            continue
        expect = c
        if fmt == FN and c == 0x80:
            expect = 0x80
        assert orc.encode(t[c], fmt) == expect, hex(c)


@pytest.mark.parametrize("fmt", [FN, FNUZ])
def test_encode_all_bf16_patterns_match_torch(fmt):
    """Every bf16 value within +-fmax (s = 1) encodes as torch's cast does."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    keep = np.isfinite(vals) & (np.abs(vals) <= orc.fp8_max(fmt))
    vals = vals[keep]
    ours = orc.encode_array(vals, fmt)
    ref = torch_encode(vals, fmt)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(vals[i]), hex(ours[i]), hex(ref[i])) for i in bad[:8]]


@pytest.mark.parametrize("fmt", [FN, FNUZ])
def test_encode_midpoints_and_neighbours_match_torch(fmt):
    """Exact ties between neighbouring codes, and one fp32 ulp either side."""
    t = orc.decode_table(fmt)
    pos = np.unique(t[np.isfinite(t) & (t >= 0)])
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    assert (mids.astype(np.float64) == (pos[:-1] + pos[1:]) / 2).all()  # exact in fp32
    pts = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)),
                          np.nextafter(mids, np.float32(0)), pos.astype(np.float32)])
    pts = np.concatenate([pts, -pts]).astype(np.float32)
    pts = pts[np.abs(pts) <= orc.fp8_max(fmt)]
    ours = orc.encode_array(pts, fmt)
    ref = torch_encode(pts, fmt)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(pts[i]), hex(ours[i]), hex(ref[i])) for i in bad[:8]]


@pytest.mark.parametrize("fmt", [FN, FNUZ])
def test_encode_random_fp32_match_torch(fmt):
    g = np.random.default_rng(7)
    m = orc.fp8_max(fmt)
    y = np.concatenate([
        g.uniform(-m, m, 40000),
        np.sign(g.standard_normal(40000)) * np.exp2(g.uniform(-14, np.log2(m), 40000)),
    ]).astype(np.float32)
    y = y[np.abs(y) <= m]
    ours = orc.encode_array(y, fmt)
    ref = torch_encode(y, fmt)
    assert (ours == ref).all()


def test_encode_is_nearest_grid_point_brute_force():
    """Brute force over the whole grid: the chosen code is a nearest finite value."""
    g = np.random.default_rng(3)
    for fmt in (FN, FNUZ):
        t = orc.decode_table(fmt)
        grid = t[np.isfinite(t)]
        for y in g.uniform(-orc.fp8_max(fmt), orc.fp8_max(fmt), 3000).astype(np.float32):
            v = orc.decode(orc.encode(y, fmt), fmt)
            assert abs(v - float(y)) == np.min(np.abs(grid - float(y)))


# --------------------------------------------------------------------------- rowwise
def test_rowwise_worked_examples_fixture():
    for r in gio.rows("rowwise_worked_examples.txt"):
        fmt = gio.FMT[r[0]]
        vals = gio.floats(r[1])
        x = bits_of(vals)
        assert (x.astype(np.uint32) << 16).view(np.float32).tolist() == vals  # bf16-exact
        q, s, sat = orc.quant_rowwise(x[None, :], fmt)
        assert int(s.view(np.uint32)[0]) == int(r[2], 16), (r, hex(int(s.view(np.uint32)[0])))
        assert q[0].tolist() == gio.hexbytes(r[3]), (r, [hex(v) for v in q[0]])
        assert sat == 0


def _random_rows(seed, rows, cols, outliers=True):
    x = wl.random_jagged(seed, [rows], cols, outlier_frac=0.01 if outliers else 0.0).x
    return wl.bf16_bits(x)


@pytest.mark.parametrize("fmt", [FN, FNUZ])
def test_rowwise_invariants(fmt):
    """No saturation with the matching maximum; the absmax element lands on +-fmax;
    round-trip error within half an e4m3 spacing; no NaN codes."""
    xb = _random_rows(11, 64, 96)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    xb[5, :] = 0  # an all-zero row
    xf[5, :] = 0
    q, s, sat = orc.quant_rowwise(xb, fmt)
    fmax = orc.fp8_max(fmt)
    table = torch_decode(np.arange(256), fmt)  # independent decode
    dq = table[q]
    assert sat == 0
    assert not np.isnan(dq).any()
    if fmt == FNUZ:
        assert not (q == 0x80).any()
    for r in range(xb.shape[0]):
        amax = np.abs(xf[r]).max()
        if amax == 0:
            assert (dq[r] == 0).all()
            continue
        j = int(np.argmax(np.abs(xf[r])))
        assert abs(dq[r, j]) == fmax
        # round-trip: |decode(q)/s - x| <= half the e4m3 spacing at |x*s|, divided by s
        y = np.abs(xf[r] * float(s[r]))
        e = np.floor(np.log2(np.maximum(y, 1e-30)))
        min_norm_exp = -6 if fmt == FN else -7
        spacing = np.exp2(np.maximum(e, min_norm_exp) - 3)
        err = np.abs(dq[r] / float(s[r]) - xf[r])
        assert (err <= spacing / 2 / float(s[r]) * (1 + 1e-6) + 1e-300).all()


def test_rowwise_scale_is_ieee_fp32_division():
    """s = RN32(fmax / max(absmax, 1e-12)), checked against numpy's fp32 divide."""
    xb = _random_rows(12, 200, 40)
    xb[7, :] = 0
    xb[9, :] = 1  # subnormal bf16 row (absmax < 1e-12)
    xf = (xb.astype(np.uint32) << 16).view(np.float32)
    for fmt in (FN, FNUZ):
        _, s, _ = orc.quant_rowwise(xb, fmt)
        amax = np.abs(xf).max(axis=1)
        expect = np.float32(orc.fp8_max(fmt)) / np.maximum(amax, np.float32(1e-12))
        assert (s.view(np.uint32) == expect.astype(np.float32).view(np.uint32)).all()


@pytest.mark.parametrize("fmt", [FN, FNUZ])
def test_encode_nan_gives_a_nan_code_and_infinity_saturates(fmt):
    """A NaN of either sign and any payload goes to a code that decodes to NaN
    (for a positive NaN the very code torch's float8 cast gives); an infinity
    saturates at the largest finite value like every magnitude above it (the
    saturating-encode reading)."""
    nans = (np.array([0x7FC00000, 0xFFC00000, 0x7F800001, 0x7FFFFFFF, 0xFF800001], np.uint32)
            .view(np.float32))
    for y in nans:
        assert np.isnan(orc.decode(orc.encode(float(y), fmt), fmt))
    pos = nans[~np.signbit(nans)]
    assert (orc.encode_array(pos, fmt) == torch_encode(pos, fmt)).all()
    t = orc.decode_table(fmt)
    top = int(np.nanargmax(np.where(np.isfinite(t), t, -np.inf)))
    low = int(np.nanargmin(np.where(np.isfinite(t), t, np.inf)))
    assert orc.encode(float("inf"), fmt) == top and t[top] == orc.fp8_max(fmt)
    assert orc.encode(float("-inf"), fmt) == low and t[low] == -orc.fp8_max(fmt)


def test_absmax_skips_nan_and_keeps_infinity():
    """A NaN in a row never decides its scale: [NaN, 2, -1] scales like [2, -1];
    an infinite absmax gives scale fmax / inf = 0, and x * 0 of the infinity is
    NaN, encoded as NaN."""
    nan, inf = float("nan"), float("inf")
    for fmt in (FN, FNUZ):
        fmax = np.float32(orc.fp8_max(fmt))
        _, s, _ = orc.quant_rowwise(bits_of([[nan, 2.0, -1.0, nan]]), fmt)
        assert s[0] == fmax / np.float32(2.0)
        _, s2, _ = orc.quant_rowwise(bits_of([[nan, nan]]), fmt)
        assert s2[0] == fmax / np.float32(1e-12)
        q3, s3, _ = orc.quant_rowwise(bits_of([[inf, 3.0, -5.0]]), fmt)
        assert s3[0] == 0.0
        nan_code = 0x80 if fmt == FNUZ else 0x7F
        zero_neg = 0x00 if fmt == FNUZ else 0x80
        assert list(q3[0]) == [nan_code, 0x00, zero_neg]
        qc, sc, _ = orc.quant_colwise_jagged(bits_of([[nan, 1.0], [4.0, nan], [-8.0, 2.0]]),
                                             np.array([3], np.int32), orc.SAME, fmt)
        assert sc[0, 0] == fmax / np.float32(8.0) and sc[0, 1] == fmax / np.float32(2.0)


def test_rowwise_codes_match_torch_cast_of_clamped_product():
    """Codes equal torch's cast of clamp(fp32(x * s)) (single rounding from fp32)."""
    xb = _random_rows(13, 128, 64)
    xf = (xb.astype(np.uint32) << 16).view(np.float32)
    for fmt in (FN, FNUZ):
        q, s, _ = orc.quant_rowwise(xb, fmt)
        fmax = np.float32(orc.fp8_max(fmt))
        y = np.clip(xf * s[:, None], -fmax, fmax).astype(np.float32)
        ref = torch_encode(y, fmt)
        if fmt == FNUZ:
            ref = np.where(ref == 0x80, 0, ref)  # unsigned zero, as the format defines
        assert (q == ref).all()


def test_format_mismatch_is_detected_both_ways():
    """Scaling against 448 while encoding e4m3fnuz saturates (counted), and the absmax
    element decodes to 240; scaling against 240 with e4m3fn never uses the top binade."""
    xb = _random_rows(14, 32, 64, outliers=False)
    q, s, sat = orc.quant_rowwise(xb, FNUZ, scale_max=448.0)
    assert sat > 0
    t = torch_decode(np.arange(256), FNUZ)
    xf = (xb.astype(np.uint32) << 16).view(np.float32)
    j = np.argmax(np.abs(xf), axis=1)
    assert (np.abs(t[q[np.arange(32), j]]) == 240).all()
    q2, s2, sat2 = orc.quant_rowwise(xb, FN, scale_max=240.0)
    t2 = torch_decode(np.arange(256), FN)
    assert sat2 == 0
    assert (np.abs(t2[q2]) <= 240).all()
    assert (np.abs(t2[q2[np.arange(32), j]]) == 240).all()
    assert not (np.abs(t2[q2]) == 448).any()


@pytest.mark.parametrize("fmt,smax", [(FNUZ, 448.0), (FN, 500.0), (FN, 0.0), (FNUZ, 0.0),
                                      (FN, 240.0), (FNUZ, 300.0)])
def test_saturation_count_is_exact(fmt, smax):
    """The oracle's saturation count equals a plain numpy fp32 count of
    |fp32(x * s)| above the next fp32 value after the encoding's maximum, for
    rowwise and jagged column-wise calls (outliers, ragged and empty groups),
    with the matching maximum (count 0) and with mismatched ones (count > 0)."""
    from tests import numpy_sat
    xb = _random_rows(15, 300, 72)
    got = orc.quant_rowwise(xb, fmt, scale_max=smax)[2]
    assert got == numpy_sat.rowwise(xb, fmt, smax)
    off = wl.offsets_from_sizes([40, 0, 1, 150, 109])
    gotc = orc.quant_colwise_jagged(xb, off, orc.SAME, fmt, scale_max=smax)[2]
    assert gotc == numpy_sat.colwise_jagged(xb, off, fmt, smax)
    if smax == 0.0 or smax <= orc.fp8_max(fmt):
        assert got == 0 and gotc == 0
    else:
        assert got > 0 and gotc > 0


# --------------------------------------------------------------------------- jagged colwise
def test_jagged_example_fixture():
    d = {r[0]: r for r in gio.rows("jagged_example.txt") if r[0] != "scales"}
    scale_rows = [r for r in gio.rows("jagged_example.txt") if r[0] == "scales"]
    x = np.array(gio.matrix(d["x"][1], gio.floats), np.float32)
    off = np.array([int(v) for v in d["offsets"][1].split()], np.int32)
    xb = bits_of(x.tolist())
    q, s, sat = orc.quant_colwise_jagged(xb, off, orc.SAME, FN)
    expect_s = np.array([gio.hexbytes(r[1]) for r in scale_rows], np.uint32)
    assert (s.view(np.uint32) == expect_s).all(), [hex(v) for v in s.view(np.uint32).ravel()]
    assert q.tolist() == gio.matrix(d["codes"][1], gio.hexbytes)
    qt, st, _ = orc.quant_colwise_jagged(xb, off, orc.TRANSPOSED, FN)
    assert (qt == q.T).all() and (st == s).all()


@pytest.mark.parametrize("fmt", [FN, FNUZ])
def test_jagged_equals_rowwise_on_each_group_transpose(fmt):
    """Per-(group, column) quantisation of X equals rowwise quantisation of each
    group's transpose: an independent route through the oracle's other entry."""
    sizes = [0, 17, 1, 40, 0, 15, 33]
    w = wl.random_jagged(21, sizes, 24, outlier_frac=0.02, zero_cols=2)
    xb = wl.bf16_bits(w.x)
    q, s, _ = orc.quant_colwise_jagged(xb, w.offsets, orc.SAME, fmt)
    start = 0
    for e, sz in enumerate(sizes):
        blk = xb[start:start + sz]
        if sz:
            qr, sr, _ = orc.quant_rowwise(np.ascontiguousarray(blk.T), fmt)
            assert (qr.T == q[start:start + sz]).all()
            assert (sr.view(np.uint32) == s[e].view(np.uint32)).all()
        else:
            expect = np.float32(orc.fp8_max(fmt)) / np.float32(1e-12)
            assert (s[e] == expect).all()
        start += sz


def test_jagged_transposed_is_bitwise_transpose_and_untouched_outside_groups():
    sizes = [5, 0, 19, 8]
    w = wl.random_jagged(22, sizes, 16)
    xb = wl.bf16_bits(w.x)
    m = sum(sizes)
    q, s, _ = orc.quant_colwise_jagged(xb, w.offsets, orc.SAME, FN)
    ld = 48
    qt, st, _ = orc.quant_colwise_jagged(xb, w.offsets, orc.TRANSPOSED, FN, ld_q=ld, fill=0xAB)
    assert (qt[:, :m] == q.T).all()
    assert (qt[:, m:] == 0xAB).all()
    assert (st == s).all()


def test_group_bounds_clamp_malformed_offsets():
    start, end = orc.group_bounds(np.array([3, 1, 9, -2, 7, 12], np.int32), 10)
    assert start.tolist() == [0, 3, 3, 9, 9, 9]
    assert end.tolist() == [3, 3, 9, 9, 9, 10]


# --------------------------------------------------------------------------- GEMM
def _quantised_moe(seed, sizes, n, k, fmt=FN):
    g = np.random.default_rng(seed)
    m = int(sum(sizes))
    e = len(sizes)
    x = wl.to_bf16(g.standard_normal((m, k)).astype(np.float32))
    w = wl.to_bf16((g.standard_normal((e * n, k)) * 0.05).astype(np.float32))
    qa, sa, _ = orc.quant_rowwise(wl.bf16_bits(x), fmt)
    qb, sb, _ = orc.quant_rowwise(wl.bf16_bits(w), fmt)
    return qa, sa, qb.reshape(e, n, k), sb.reshape(e, n), wl.offsets_from_sizes(sizes)


def test_gemm_m_jagged_matches_numpy_fp64_on_every_element():
    sizes = [3, 0, 17, 1, 9]
    n, k = 12, 40
    qa, sa, qb, sb, off = _quantised_moe(31, sizes, n, k)
    m = sum(sizes)
    rr, cc = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    c, b = orc.gemm_m_jagged_sample(qa, sa, qb, sb, off, rr.ravel(), cc.ravel())
    c = c.reshape(m, n)
    b = b.reshape(m, n)
    ta = torch_decode(qa, FN) / sa[:, None].astype(np.float64)
    tb = torch_decode(qb, FN) / sb[:, :, None].astype(np.float64)
    start = 0
    for e, sz in enumerate(sizes):
        ref = ta[start:start + sz] @ tb[e].T
        mag = np.abs(ta[start:start + sz]) @ np.abs(tb[e]).T
        assert np.allclose(c[start:start + sz], ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(b[start:start + sz], 1e-3 * mag, rtol=1e-12, atol=0)
        start += sz


def test_gemm_m_jagged_rows_outside_groups_are_nan():
    qa, sa, qb, sb, off = _quantised_moe(32, [4, 4], 8, 16)
    off = np.array([3, 5], np.int32)  # rows 5..7 belong to no group
    c, _ = orc.gemm_m_jagged_sample(qa, sa, qb, sb, off, [0, 4, 5, 7], [1, 1, 1, 1])
    assert np.isfinite(c[:2]).all() and np.isnan(c[2:]).all()


def test_gemm_k_jagged_matches_numpy_fp64_per_group():
    sizes = [7, 0, 30, 1, 12]
    n, k = 10, 14
    m = sum(sizes)
    g = np.random.default_rng(41)
    dh = wl.to_bf16(g.standard_normal((m, n)).astype(np.float32) * 1e-3)
    x = wl.to_bf16(g.standard_normal((m, k)).astype(np.float32))
    off = wl.offsets_from_sizes(sizes)
    ld = 64
    qa_t, sa, _ = orc.quant_colwise_jagged(wl.bf16_bits(dh), off, orc.TRANSPOSED, FN, ld_q=ld)
    qb_t, sb, _ = orc.quant_colwise_jagged(wl.bf16_bits(x), off, orc.TRANSPOSED, FN, ld_q=ld)
    ee, ii, jj = np.meshgrid(np.arange(len(sizes)), np.arange(n), np.arange(k), indexing="ij")
    c, b = orc.gemm_k_jagged_sample(qa_t, sa, qb_t, sb, off, m, ee.ravel(), ii.ravel(), jj.ravel())
    c = c.reshape(len(sizes), n, k)
    b = b.reshape(len(sizes), n, k)
    da = torch_decode(qa_t[:, :m], FN)  # [n, m]
    db = torch_decode(qb_t[:, :m], FN)  # [k, m]
    start = 0
    for e, sz in enumerate(sizes):
        a_e = da[:, start:start + sz] / sa[e][:, None].astype(np.float64)
        b_e = db[:, start:start + sz] / sb[e][:, None].astype(np.float64)
        ref = a_e @ b_e.T
        assert np.allclose(c[e], ref, rtol=1e-12, atol=1e-15)
        assert np.allclose(b[e], 1e-3 * (np.abs(a_e) @ np.abs(b_e).T), rtol=1e-12, atol=0)
        if sz == 0:
            assert (c[e] == 0).all()
        start += sz


def test_gemm_reference_tracks_the_bf16_product():
    """Closed-form sanity: with per-row / per-channel scaling the dequantised product
    stays close to the bf16 product it approximates (FP8 relative step 2^-4)."""
    g = np.random.default_rng(51)
    m, n, k = 16, 8, 64
    x = wl.to_bf16(g.standard_normal((m, k)).astype(np.float32))
    w = wl.to_bf16(g.standard_normal((n, k)).astype(np.float32))
    qa, sa, _ = orc.quant_rowwise(wl.bf16_bits(x), FN)
    qb, sb, _ = orc.quant_rowwise(wl.bf16_bits(w), FN)
    rr, cc = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    c, _ = orc.gemm_m_jagged_sample(qa, sa, qb[None], sb[None], np.array([m], np.int32),
                                    rr.ravel(), cc.ravel())
    exact = x.double().numpy() @ w.double().numpy().T
    mag = np.abs(x.double().numpy()) @ np.abs(w.double().numpy()).T
    assert (np.abs(c.reshape(m, n) - exact) <= 2 * 2 ** -4 * mag).all()
