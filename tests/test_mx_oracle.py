"""Pins of the oracle's MXFP8 functions against what the MX definition and
the mathematics fix.

The pages name MXFP8 ("AMD Primus adds FP8/MXFP8 kernels ...", section "What
Primus adds for MoE training on MI355X") without defining it; the reading is
the OCP MX v1.0 one: 32-element blocks, E8M0 scale 2^(floor(log2 amax) - 8),
e4m3fn elements clamped to +-448.  Expected values come from hand-worked
blocks (tests/golden/mx_worked_examples.txt), from numpy's frexp and torch's
float8_e4m3fn cast, from numpy fp64 matmuls of dequantised operands, and from
the identity between the padded column-wise form and the row-wise form of the
padded transposed input.
"""
import os

import numpy as np
import pytest
import torch

import oracle as orc
from quantization_grouped_gemm_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mx_worked_examples.txt")


def bits_of(values):
    return wl.bf16_bits(torch.tensor(np.asarray(values, np.float32)).to(torch.bfloat16))


def torch_decode_fn(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def expected_block(x):
    """Scale byte and codes of one block, restated with numpy and torch."""
    a = np.abs(x.astype(np.float64))
    a = a[~np.isnan(a)]
    amax = a.max() if a.size else 0.0
    if amax == 0.0:
        e = -127
    elif np.isinf(amax):
        e = 127
    else:
        _, ex = np.frexp(amax)
        e = int(np.clip(ex - 1 - 8, -127, 127))
    y = np.clip(np.ldexp(x.astype(np.float64), -e), -448.0, 448.0).astype(np.float32)
    codes = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return e + 127, codes


def dequant(q, s, axis_len):
    """decode(q) * 2^(s - 127), s broadcast over blocks of 32 along the last axis."""
    v = torch_decode_fn(q)
    sc = np.repeat(s.astype(np.int64) - 127, 32, axis=-1)[..., :axis_len]
    return np.ldexp(v, sc)


# --------------------------------------------------------------------------- golden
def load_golden():
    cases = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, byte, body = [p.strip() for p in line.split(";")]
            vals = np.zeros(32, np.float32)
            codes = np.zeros(32, np.uint8)
            for item in body.split():
                idx, rest = item.split("=")
                v, c = rest.split("->")
                vals[int(idx)] = np.float32(float(v))
                codes[int(idx)] = int(c, 16)
            cases.append((name, int(byte), vals, codes))
    return cases


@pytest.mark.parametrize("case", load_golden(), ids=lambda c: c[0])
def test_mx_worked_examples(case):
    name, byte, vals, codes = case
    q, s = orc.mx_quant_rowwise(bits_of(vals)[None, :])
    assert int(s[0, 0]) == byte, name
    assert (q[0] == codes).all(), (name, q[0], codes)


def test_golden_file_covers_the_listed_cases():
    names = [c[0] for c in load_golden()]
    assert names == ["three", "clamp", "zero", "one", "tiny", "huge", "edge"]


# --------------------------------------------------------------------------- chain
def block_battery(seed):
    g = np.random.default_rng(seed)
    blocks = []
    for mag in [1.0, 1e-3, 1e3, 1e-30, 1e30, 1e-39, 3e38]:
        blocks.append(g.standard_normal(32) * mag)
    b = g.standard_normal(32)
    b[5] = 0.0
    blocks.append(b)
    blocks.append(np.zeros(32))
    b = g.standard_normal(32)
    b[3] = np.inf
    blocks.append(b)
    b = g.standard_normal(32)
    b[7] = np.nan
    blocks.append(b)
    b = np.full(32, np.nan)
    blocks.append(b)
    # amax just below and at a power of two, and mantissas around 1.75
    for amax in [1.75, 1.8125, 1.9921875, 2.0, 0.99609375]:
        b = g.uniform(-1, 1, 32) * amax
        b[11] = -amax
        blocks.append(b)
    for _ in range(40):
        blocks.append(g.standard_normal(32) * 10.0 ** g.uniform(-20, 20))
    with np.errstate(over="ignore"):  # 3e38-scale blocks overflow to inf on purpose
        return np.stack(blocks).astype(np.float32)


def test_mx_rowwise_matches_numpy_exponent_and_torch_cast():
    x = block_battery(3)
    xb = bits_of(x)
    xr = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).float().numpy()
    q, s = orc.mx_quant_rowwise(xb)
    for i in range(x.shape[0]):
        byte, codes = expected_block(xr[i])
        assert int(s[i, 0]) == byte, (i, xr[i])
        nan = np.isnan(xr[i])
        assert (q[i][~nan] == codes[~nan]).all(), i
        assert np.isnan(torch_decode_fn(q[i][nan])).all()


def test_mx_rowwise_multi_block_rows_and_error_bound():
    g = np.random.default_rng(5)
    x = (g.standard_normal((37, 256)) * np.exp(g.uniform(-8, 8, (37, 1)))).astype(np.float32)
    xb = bits_of(x)
    xr = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).double().numpy()
    q, s = orc.mx_quant_rowwise(xb)
    assert s.shape == (37, 8)
    v = dequant(q, s, 256)
    for r in range(37):
        for b in range(8):
            blk = xr[r, 32 * b:32 * b + 32]
            byte, codes = expected_block(blk.astype(np.float32))
            assert s[r, b] == byte and (q[r, 32 * b:32 * b + 32] == codes).all()
            e = int(s[r, b]) - 127
            y = blk * 2.0 ** -e
            # the block maximum lands in [256, 512) before the clamp
            assert 256 <= np.abs(y).max() < 512
            ok = np.abs(y) <= 448
            # within half an e4m3 spacing (3 mantissa bits) where not clamped;
            # spacing at |y| is 2^(floor(log2|y|) - 3), at least 2^-9 (subnormals)
            sp = np.ldexp(1.0, np.maximum(np.floor(np.log2(np.maximum(np.abs(y), 1e-300))),
                                          -6).astype(int) - 3)
            err = np.abs(v[r, 32 * b:32 * b + 32] * 2.0 ** -e - y)
            assert (err[ok] <= sp[ok] / 2 + 1e-300).all()
            assert (v[r, 32 * b:32 * b + 32][~ok] == np.sign(blk[~ok]) * 448 * 2.0 ** e).all()


# --------------------------------------------------------------------------- colwise
def padded_transpose(x_bits, sizes):
    """bf16 bits of the padded transposed matrix: group e's tokens at P_e, zeros after."""
    rows, cols = x_bits.shape
    out = np.zeros((cols, orc.padded_len(sizes)), np.uint16)
    start, p = 0, 0
    for sz in sizes:
        out[:, p:p + sz] = x_bits[start:start + sz].T
        start += sz
        p += (sz + 127) // 128 * 128
    return out


@pytest.mark.parametrize("sizes,cols", [
    ([5, 0, 19, 8], 16), ([0, 1, 31, 32, 33, 0, 129, 255, 256], 40), ([300], 8), ([0, 0], 4),
    ([1] * 9, 24)])
def test_mx_colwise_padded_is_rowwise_of_the_padded_transpose(sizes, cols):
    g = np.random.default_rng(len(sizes) * 100 + cols)
    m = int(sum(sizes))
    x = (g.standard_normal((m + 3, cols)) * np.exp(g.uniform(-6, 6, (1, cols)))).astype(np.float32)
    xb = bits_of(x)
    off = wl.offsets_from_sizes(sizes)
    q, s = orc.mx_quant_colwise_padded(xb, off)
    pt = padded_transpose(xb, sizes)
    if pt.shape[1] == 0:
        assert q.shape[1] == 0
        return
    q_ref, s_ref = orc.mx_quant_rowwise(pt)
    assert (q == q_ref).all()
    assert (s == s_ref).all()
    # padding-only blocks carry E = -127
    p = 0
    for sz in sizes:
        r = (sz + 127) // 128 * 128
        full = (sz + 31) // 32
        assert (s[:, p // 32 + full:(p + r) // 32] == 0).all()
        p += r


def test_mx_colwise_padded_leaves_tokens_past_the_last_group():
    xb = bits_of(np.ones((50, 8), np.float32))
    q, s = orc.mx_quant_colwise_padded(xb, wl.offsets_from_sizes([10]), ld_q=256, fill=0xAB,
                                       scale_fill=0xCD)
    assert (q[:, 128:] == 0xAB).all() and (s[:, 4:] == 0xCD).all()
    assert (q[:, :10] == 0x78).all() and (q[:, 10:128] == 0).all()  # 1.0 -> 256 -> 0x78
    assert (s[:, 0] == 119).all() and (s[:, 1:4] == 0).all()


# --------------------------------------------------------------------------- GEMM
def random_mx_operand(g, shape, mag_spread=4.0):
    x = g.standard_normal(shape) * np.exp(g.uniform(-mag_spread, mag_spread, shape[:-1] + (1,)))
    return bits_of(x.astype(np.float32))


def test_mx_gemm_m_jagged_matches_numpy_fp64():
    g = np.random.default_rng(7)
    sizes = [3, 0, 70, 129, 1]
    m, n, k = sum(sizes), 40, 96
    qa, sa = orc.mx_quant_rowwise(random_mx_operand(g, (m, k)))
    qb, sb = orc.mx_quant_rowwise(random_mx_operand(g, (len(sizes) * n, k)))
    qb = qb.reshape(len(sizes), n, k)
    sb = sb.reshape(len(sizes), n, k // 32)
    off = wl.offsets_from_sizes(sizes)
    rows = np.repeat(np.arange(m), n)
    cols = np.tile(np.arange(n), m)
    c, bound = orc.mx_gemm_m_jagged_sample(qa, sa, qb, sb, off, rows, cols)
    A = dequant(qa, sa, k)
    B = dequant(qb, sb, k)
    start = 0
    for e, sz in enumerate(sizes):
        ref = A[start:start + sz] @ B[e].T
        mag = np.abs(A[start:start + sz]) @ np.abs(B[e]).T
        got = c.reshape(m, n)[start:start + sz]
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-300)
        assert np.allclose(bound.reshape(m, n)[start:start + sz], 1e-3 * mag, rtol=1e-12)
        start += sz


def test_mx_gemm_k_jagged_padded_matches_numpy_fp64():
    g = np.random.default_rng(9)
    sizes = [40, 0, 200, 33]
    m = sum(sizes)
    n1, n2 = 24, 16
    off = wl.offsets_from_sizes(sizes)
    qa, sa = orc.mx_quant_colwise_padded(random_mx_operand(g, (m, n1)), off)
    qb, sb = orc.mx_quant_colwise_padded(random_mx_operand(g, (m, n2)), off)
    A = dequant(qa, sa, qa.shape[1])
    B = dequant(qb, sb, qb.shape[1])
    grp, rows, cols = np.meshgrid(np.arange(len(sizes)), np.arange(n1), np.arange(n2),
                                  indexing="ij")
    c, bound = orc.mx_gemm_k_jagged_padded_sample(qa, sa, qb, sb, off, m, grp.ravel(),
                                                  rows.ravel(), cols.ravel())
    c = c.reshape(len(sizes), n1, n2)
    p = 0
    for e, sz in enumerate(sizes):
        ref = A[:, p:p + sz] @ B[:, p:p + sz].T
        assert np.allclose(c[e], ref, rtol=1e-12, atol=1e-300)
        if sz == 0:
            assert (c[e] == 0).all()
        p += (sz + 127) // 128 * 128


def test_mx_gemm_detects_a_swapped_block_scale():
    """A mistake the GEMM pins must catch: the scale of block 1 used for block 0."""
    g = np.random.default_rng(11)
    qa, sa = orc.mx_quant_rowwise(random_mx_operand(g, (1, 64), 0.0))
    qb, sb = orc.mx_quant_rowwise(random_mx_operand(g, (1, 64), 0.0))
    sa = sa.copy()
    sa[0] = [120, 100]
    c, _ = orc.mx_gemm_m_jagged_sample(qa, sa, qb[None], sb[None], np.array([1], np.int32),
                                       [0], [0])
    wrong = sa[:, ::-1].copy()
    c2, _ = orc.mx_gemm_m_jagged_sample(qa, wrong, qb[None], sb[None], np.array([1], np.int32),
                                        [0], [0])
    assert c[0] != c2[0]
