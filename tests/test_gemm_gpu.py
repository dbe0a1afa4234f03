"""GPU parity of the FP8 scaled grouped GEMM against the CPU oracle.

The oracle quantises the bf16 inputs itself and evaluates the fp64 reference
and the bound 1e-3 * sum |a||b| per element; the GPU path quantises with the
library's kernels and multiplies on the tensor cores.  The quantisation is
bit-exact (tested separately), so both sides see the same FP8 operands."""
import numpy as np
import pytest
import torch

import oracle as orc
import quantization_grouped_gemm_b200 as qgg
from quantization_grouped_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def bits(t):
    return wl.bf16_bits(t.cpu())


def rand_bf16(seed, shape, std=1.0):
    g = np.random.default_rng(seed)
    return wl.to_bf16(g.standard_normal(shape).astype(np.float32) * np.float32(std))


def m_jagged_case(seed, sizes, n, k, out_dtype=torch.float32, m_total=None, offsets=None):
    m = int(sum(sizes)) if m_total is None else m_total
    e = len(sizes)
    x = rand_bf16(seed, (m, k))
    w = rand_bf16(seed + 1, (e, n, k), 0.02)
    off = wl.offsets_from_sizes(sizes) if offsets is None else np.asarray(offsets, np.int32)
    qa, sa = qgg.fp8_quant_rowwise(x.cuda())
    qb, sb = qgg.fp8_quant_rowwise(w.cuda().reshape(e * n, k))
    canary = torch.full((m, n), float("nan"), dtype=out_dtype, device="cuda")
    out = qgg.fp8_scaled_grouped_gemm(qgg.M_JAGGED, qa, sa, qb.reshape(e, n, k),
                                      sb.reshape(e, n), torch.from_numpy(off).cuda(),
                                      out=canary, out_dtype=out_dtype)
    torch.cuda.synchronize()
    # oracle side: its own quantisation of the same bf16 inputs
    oa, osa, _ = orc.quant_rowwise(bits(x))
    ob, osb, _ = orc.quant_rowwise(bits(w.reshape(e * n, k)))
    return out.float().cpu().numpy(), (oa, osa, ob.reshape(e, n, k), osb.reshape(e, n), off)


def check_all(out, ref_args, rows=None, extra_rel=0.0):
    oa, osa, ob, osb, off = ref_args
    m, n = out.shape
    if rows is None:
        rows = np.arange(m)
    rr, cc = np.meshgrid(rows, np.arange(n), indexing="ij")
    c, b = orc.gemm_m_jagged_sample(oa, osa, ob, osb, off, rr.ravel(), cc.ravel())
    got = out[rr.ravel(), cc.ravel()]
    inside = ~np.isnan(c)
    err = np.abs(got[inside] - c[inside])
    tol = b[inside] + extra_rel * np.abs(c[inside])
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, (bad.size, err[bad[:5]], tol[bad[:5]])
    # rows outside every group stay untouched
    assert np.isnan(got[~inside]).all()


def test_m_jagged_tiny_moe_every_element():
    w = wl.tiny_moe()
    e, n, k = 4, 128, 256
    sizes = list(w.group_sizes)
    out, ref = m_jagged_case(1001, sizes, n, k)
    check_all(out, ref)


@pytest.mark.parametrize("sizes,n,k", [
    ([0, 1, 15, 17, 129, 300], 384, 320),
    ([7], 16, 16),
    ([200, 0, 0, 57], 272, 1040),
    ([1, 2, 3], 8, 128),
])
def test_m_jagged_ragged_every_element(sizes, n, k):
    out, ref = m_jagged_case(sum(sizes) + n + k, sizes, n, k)
    check_all(out, ref)


def test_m_jagged_bf16_output():
    sizes = [33, 0, 130]
    out, ref = m_jagged_case(5, sizes, 256, 512, out_dtype=torch.bfloat16)
    check_all(out, ref, extra_rel=2.0 ** -8)


def test_m_jagged_rows_past_last_offset_untouched():
    out, ref = m_jagged_case(6, [40, 60], 128, 256, m_total=150, offsets=[40, 100])
    check_all(out, ref)
    assert np.isnan(out[100:]).all()


def test_m_jagged_many_tiles_persistent_wraparound():
    """More tiles than SMs x 2 accumulators: every CTA reuses both TMEM buffers."""
    sizes = [1000, 3, 2100, 0, 1500, 640, 1]
    n, k = 512, 384
    out, ref = m_jagged_case(7, sizes, n, k)
    rows = np.unique(np.concatenate([np.cumsum(sizes) - 1, np.cumsum(sizes)[:-1],
                                     np.random.default_rng(0).integers(0, sum(sizes), 200)]))
    rows = rows[(rows >= 0) & (rows < sum(sizes))]
    check_all(out, ref, rows=rows)


# groups averaging >= 256 rows run on SM pairs (cta_group::2, 256-row tiles)
@pytest.mark.parametrize("sizes,n,k", [
    ([600, 900, 0, 1200], 384, 320),
    ([256, 512, 257, 255, 1], 256, 128),
    ([4096], 528, 1040),
    ([3000, 17, 700], 96, 256),
])
def test_m_jagged_pair_tiles_every_element(sizes, n, k):
    out, ref = m_jagged_case(sum(sizes) + 3 * n + k, sizes, n, k)
    check_all(out, ref)


def test_m_jagged_pair_tiles_bf16_and_rows_past_last_offset():
    out, ref = m_jagged_case(77, [700, 500], 256, 512, out_dtype=torch.bfloat16, m_total=1300,
                             offsets=[700, 1200])
    check_all(out, ref, extra_rel=2.0 ** -8)
    assert np.isnan(out[1200:]).all()


def test_m_jagged_pair_tiles_exact_small_k_with_unit_scales():
    g = np.random.default_rng(19)
    m, n, k = 1100, 272, 16
    sizes = [520, 0, 580]
    table = orc.decode_table(orc.E4M3FN)
    allowed = np.array([c for c in range(256) if np.isfinite(table[c]) and
                        1.0 <= abs(table[c]) < 16.0], np.uint8)
    qa = allowed[g.integers(0, allowed.size, (m, k))]
    qb = allowed[g.integers(0, allowed.size, (3, n, k))]
    ones_a = np.ones(m, np.float32)
    ones_b = np.ones((3, n), np.float32)
    off = wl.offsets_from_sizes(sizes)
    out = qgg.fp8_scaled_grouped_gemm(qgg.M_JAGGED, torch.from_numpy(qa).cuda(),
                                      torch.from_numpy(ones_a).cuda(),
                                      torch.from_numpy(qb).cuda(),
                                      torch.from_numpy(ones_b).cuda(),
                                      torch.from_numpy(off).cuda()).cpu().numpy()
    rr, cc = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    c, _ = orc.gemm_m_jagged_sample(qa, ones_a, qb, ones_b, off, rr.ravel(), cc.ravel())
    assert (out.ravel() == c).all()


def test_m_jagged_exact_small_k_with_unit_scales():
    """Codes with exponents in [1, 16) and unit scales: products and sums of up to
    16 terms are exact in fp32, so the tensor cores must match fp64 exactly."""
    g = np.random.default_rng(9)
    m, n, k, e = 300, 48, 16, 3
    sizes = [100, 0, 200]
    table = orc.decode_table(orc.E4M3FN)
    allowed = np.array([c for c in range(256) if np.isfinite(table[c]) and
                        1.0 <= abs(table[c]) < 16.0], np.uint8)
    qa = allowed[g.integers(0, allowed.size, (m, k))]
    qb = allowed[g.integers(0, allowed.size, (e, n, k))]
    ones_a = np.ones(m, np.float32)
    ones_b = np.ones((e, n), np.float32)
    off = wl.offsets_from_sizes(sizes)
    out = qgg.fp8_scaled_grouped_gemm(qgg.M_JAGGED, torch.from_numpy(qa).cuda(),
                                      torch.from_numpy(ones_a).cuda(),
                                      torch.from_numpy(qb).cuda(),
                                      torch.from_numpy(ones_b).cuda(),
                                      torch.from_numpy(off).cuda()).cpu().numpy()
    rr, cc = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    c, _ = orc.gemm_m_jagged_sample(qa, ones_a, qb, ones_b, off, rr.ravel(), cc.ravel())
    assert (out.ravel() == c).all()


# ----------------------------------------------------------------- K-jagged (dW)
def k_jagged_case(seed, sizes, n, k, ld_pad=32):
    m = int(sum(sizes))
    dh = rand_bf16(seed, (m, n), 1e-3)
    x = rand_bf16(seed + 1, (m, k))
    off = wl.offsets_from_sizes(sizes)
    offd = torch.from_numpy(off).cuda()
    ld = (m + ld_pad + 15) // 16 * 16
    qa, sa = qgg.fp8_quant_colwise_jagged(dh.cuda(), offd, qgg.LAYOUT_TRANSPOSED, ld_q=ld)
    qb, sb = qgg.fp8_quant_colwise_jagged(x.cuda(), offd, qgg.LAYOUT_TRANSPOSED, ld_q=ld)
    e = len(sizes)
    out = torch.full((e, n, k), float("nan"), device="cuda")
    qgg.fp8_scaled_grouped_gemm(qgg.K_JAGGED, qa, sa, qb, sb, offd, m_total=m, out=out)
    torch.cuda.synchronize()
    oa, osa, _ = orc.quant_colwise_jagged(bits(dh), off, orc.TRANSPOSED, ld_q=ld)
    ob, osb, _ = orc.quant_colwise_jagged(bits(x), off, orc.TRANSPOSED, ld_q=ld)
    return out.cpu().numpy(), (oa, osa, ob, osb, off, m)


def check_k_all(out, ref):
    oa, osa, ob, osb, off, m = ref
    e, n, k = out.shape
    ee, ii, jj = np.meshgrid(np.arange(e), np.arange(n), np.arange(k), indexing="ij")
    c, b = orc.gemm_k_jagged_sample(oa, osa, ob, osb, off, m, ee.ravel(), ii.ravel(), jj.ravel())
    got = out.ravel()
    err = np.abs(got - c)
    bad = np.nonzero(~(err <= b))[0]
    assert bad.size == 0, (bad.size, got[bad[:5]], c[bad[:5]], b[bad[:5]])


@pytest.mark.parametrize("sizes,n,k", [
    ([0, 5, 17, 130, 1, 250], 200, 136),
    ([129], 128, 256),
    ([3, 700, 0, 44], 72, 264),
    ([16, 16, 16], 8, 8),
])
def test_k_jagged_every_element(sizes, n, k):
    out, ref = k_jagged_case(sum(sizes) * 3 + n, sizes, n, k)
    check_k_all(out, ref)
    for e, sz in enumerate(sizes):
        if sz == 0:
            assert (out[e] == 0).all()


@pytest.mark.parametrize("sizes,n,k", [
    ([0, 5, 17, 130, 1, 250], 200, 136),
    ([3, 700, 0, 44, 128, 256], 72, 264),
])
def test_k_jagged_padded_operands_every_element(sizes, n, k):
    """Operands in the padded transposed layout (groups at 128-token
    boundaries, zeros in the gaps) give the oracle's products on the plain
    operands.  The code buffers start filled with NaN codes, so a token the
    GEMM read outside the groups' padded ranges, or a gap left unwritten,
    would turn outputs into NaN."""
    m = int(sum(sizes))
    e = len(sizes)
    seed = 5 * m + n
    dh = rand_bf16(seed, (m, n), 1e-3)
    x = rand_bf16(seed + 1, (m, k))
    off = wl.offsets_from_sizes(sizes)
    offd = torch.from_numpy(off).cuda()
    ld = (m + 128 * e + 127) // 128 * 128
    qa = torch.full((n, ld), 0x7F, dtype=torch.uint8, device="cuda")
    qb = torch.full((k, ld), 0x7F, dtype=torch.uint8, device="cuda")
    qa, sa = qgg.fp8_quant_colwise_jagged(dh.cuda(), offd, qgg.LAYOUT_TRANSPOSED_PADDED, q=qa)
    qb, sb = qgg.fp8_quant_colwise_jagged(x.cuda(), offd, qgg.LAYOUT_TRANSPOSED_PADDED, q=qb)
    out = torch.full((e, n, k), float("nan"), device="cuda")
    qgg.fp8_scaled_grouped_gemm(qgg.K_JAGGED_PADDED, qa, sa, qb, sb, offd, m_total=m, out=out)
    torch.cuda.synchronize()
    oa, osa, _ = orc.quant_colwise_jagged(bits(dh), off, orc.TRANSPOSED)
    ob, osb, _ = orc.quant_colwise_jagged(bits(x), off, orc.TRANSPOSED)
    out = out.cpu().numpy()
    check_k_all(out, (oa, osa, ob, osb, off, m))
    for g, sz in enumerate(sizes):
        if sz == 0:
            assert (out[g] == 0).all()


def test_k_jagged_group_starts_at_every_residue_of_a_block():
    """Groups whose starts fall at every position inside a 128-token block (and
    whose ends too), so that every pattern of skipped 32-token steps and
    masked pieces at both edges of a block is met."""
    g = np.random.default_rng(128)
    sizes = [int(v) for v in g.integers(1, 300, 60)]
    sizes[3:6] = [0, 128, 1]
    m = sum(sizes)
    starts = np.cumsum([0] + sizes[:-1]) % 128
    assert len(set(starts.tolist())) > 40
    out, ref = k_jagged_case(4242, sizes, 40, 72, ld_pad=100)
    check_k_all(out, ref)


@pytest.mark.parametrize("sizes,n,k,odt", [
    ([300, 0, 1, 1000], 1408, 2048, torch.float32),
    ([129, 5, 260], 24, 40, torch.float32),
    ([700, 33] * 20, 96, 520, torch.float32),
    ([257, 0, 90], 200, 136, torch.bfloat16),
])
def test_k_jagged_padded_odd_shapes(sizes, n, k, odt):
    """The padded contraction-jagged GEMM on shapes whose n and k are not tile
    multiples, with many groups (more tiles than SMs), an empty group and bf16
    output; every element against the oracle (bf16 output: within the bound
    plus the bf16 rounding of the output, 2^-8 relative)."""
    m = int(sum(sizes))
    e = len(sizes)
    dh = rand_bf16(3 * m + n, (m, n), 1e-3)
    x = rand_bf16(3 * m + n + 1, (m, k))
    off = wl.offsets_from_sizes(sizes)
    offd = torch.from_numpy(off).cuda()
    P = qgg.LAYOUT_TRANSPOSED_PADDED
    qa, sa = qgg.fp8_quant_colwise_jagged(dh.cuda(), offd, P)
    qb, sb = qgg.fp8_quant_colwise_jagged(x.cuda(), offd, P)
    out = torch.full((e, n, k), float("nan"), dtype=odt, device="cuda")
    qgg.fp8_scaled_grouped_gemm(qgg.K_JAGGED_PADDED, qa, sa, qb, sb, offd, m_total=m, out=out)
    torch.cuda.synchronize()
    oa, osa, _ = orc.quant_colwise_jagged(bits(dh), off, orc.TRANSPOSED)
    ob, osb, _ = orc.quant_colwise_jagged(bits(x), off, orc.TRANSPOSED)
    ee, ii, jj = np.meshgrid(np.arange(e), np.arange(n), np.arange(k), indexing="ij")
    c, b = orc.gemm_k_jagged_sample(oa, osa, ob, osb, off, m, ee.ravel(), ii.ravel(), jj.ravel())
    got = out.float().cpu().numpy().ravel()
    tol = b + (np.abs(c) * 2.0 ** -8 if odt == torch.bfloat16 else 0.0)
    bad = np.nonzero(~(np.abs(got - c) <= tol))[0]
    assert bad.size == 0, (bad.size, got[bad[:5]], c[bad[:5]], tol[bad[:5]])
    for g, sz in enumerate(sizes):
        if sz == 0:
            assert (out[g] == 0).all()
