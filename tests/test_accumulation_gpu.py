"""Adversarial accumulation: all-positive FP8 operands over the longest
contractions the workloads reach.

With all-positive operands no rounding error of the fp32 accumulation can
cancel against another, and sum |a||b| equals the product itself, so the
per-element bound 1e-3 * sum |a||b| is a plain relative bound of 1e-3 on every
output.  A sequential fp32 sum of n terms can lose up to n * 2^-24 of the total
(16384 * 2^-24 ~ 9.8e-4 at the longest contraction here), which is why these
cases are the thinnest margin of the GEMM's tolerance.  The pages' worry is the
same: a wrong result that nothing flags ("AMD Boosts PyTorch FP8 Training on
Instinct GPUs", third paragraph).

Every case compares the tensor-core result with the oracle's fp64 reference of
the oracle's own quantisation of the same bf16 inputs.  The worst ratio
error / bound is printed (run with -s to see it).
"""
import numpy as np
import pytest
import torch

import oracle as orc
import quantization_grouped_gemm_b200 as qgg
from quantization_grouped_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def bits(t):
    return wl.bf16_bits(t.cpu())


def positive_bf16(seed, shape, std=1.0):
    g = np.random.default_rng(seed)
    a = np.abs(g.standard_normal(shape).astype(np.float32)) * np.float32(std)
    return wl.to_bf16(a + np.float32(std * 1e-3))  # strictly positive


def worst_ratio(got, c, b, what):
    assert (c > 0).all() and (b > 0).all(), "all-positive operands give positive products"
    err = np.abs(got.astype(np.float64) - c)
    bad = np.nonzero(~(err <= b))[0]
    ratio = float((err / b).max())
    print(f"\n{what}: worst |err| / (1e-3 sum|a||b|) = {ratio:.4f} over {c.size} outputs")
    assert bad.size == 0, (bad.size, got[bad[:4]], c[bad[:4]], b[bad[:4]])
    return ratio


@pytest.mark.parametrize("mode", [qgg.K_JAGGED, qgg.K_JAGGED_PADDED])
def test_k_jagged_all_positive_16384_token_group_every_element(mode):
    """One group of 16384 tokens (the longest contraction the DeepSeek-MoE-16B
    routing allows one expert) plus a short one; every output element."""
    sizes = [16384, 37]
    m, n, k, e = sum(sizes), 256, 256, len(sizes)
    dh = positive_bf16(61, (m, n), 1e-3)
    x = positive_bf16(62, (m, k))
    off = wl.offsets_from_sizes(sizes)
    offd = torch.from_numpy(off).cuda()
    layout = qgg.LAYOUT_TRANSPOSED if mode == qgg.K_JAGGED else qgg.LAYOUT_TRANSPOSED_PADDED
    qa, sa = qgg.fp8_quant_colwise_jagged(dh.cuda(), offd, layout)
    qb, sb = qgg.fp8_quant_colwise_jagged(x.cuda(), offd, layout)
    out = torch.full((e, n, k), float("nan"), device="cuda")
    qgg.fp8_scaled_grouped_gemm(mode, qa, sa, qb, sb, offd, m_total=m, out=out)
    torch.cuda.synchronize()
    oa, osa, _ = orc.quant_colwise_jagged(bits(dh), off, orc.TRANSPOSED)
    ob, osb, _ = orc.quant_colwise_jagged(bits(x), off, orc.TRANSPOSED)
    ee, ii, jj = np.meshgrid(np.arange(e), np.arange(n), np.arange(k), indexing="ij")
    c, b = orc.gemm_k_jagged_sample(oa, osa, ob, osb, off, m, ee.ravel(), ii.ravel(), jj.ravel())
    worst_ratio(out.cpu().numpy().ravel(), c, b, f"K-jagged mode {mode}, 16384-token group")


@pytest.mark.parametrize("sizes", [[512], [100, 60]])
def test_m_jagged_all_positive_k_16384_every_element(sizes):
    """Token-jagged GEMM with a contraction of 16384: the SM-pair kernel (one
    512-row group) and the one-SM kernel (two small groups)."""
    m, n, k, e = sum(sizes), 256, 16384, len(sizes)
    x = positive_bf16(63, (m, k))
    w = positive_bf16(64, (e, n, k), 0.02)
    off = wl.offsets_from_sizes(sizes)
    qa, sa = qgg.fp8_quant_rowwise(x.cuda())
    qb, sb = qgg.fp8_quant_rowwise(w.cuda().reshape(e * n, k))
    out = qgg.fp8_scaled_grouped_gemm(qgg.M_JAGGED, qa, sa, qb.reshape(e, n, k),
                                      sb.reshape(e, n), torch.from_numpy(off).cuda())
    torch.cuda.synchronize()
    oa, osa, _ = orc.quant_rowwise(bits(x))
    ob, osb, _ = orc.quant_rowwise(bits(w.reshape(e * n, k)))
    rr, cc = np.meshgrid(np.arange(m), np.arange(n), indexing="ij")
    c, b = orc.gemm_m_jagged_sample(oa, osa, ob.reshape(e, n, k), osb.reshape(e, n), off,
                                    rr.ravel(), cc.ravel())
    worst_ratio(out.cpu().numpy().ravel(), c, b, f"M-jagged groups {sizes}, K=16384")


@pytest.mark.parametrize("mode", [qgg.K_JAGGED, qgg.K_JAGGED_PADDED])
def test_k_jagged_all_positive_deepseek_moe16b_largest_group(mode):
    """The DeepSeek-MoE-16B backward routing (64 Zipf groups, 98304 rows) with
    |grad_out| and |X|: the weight gradient of the largest group (the longest
    contraction of the workload) on a block of sampled (row, column) outputs,
    plus sampled outputs of every other group."""
    w = wl.deepseek_moe_16b_backward()
    g_abs = w.grad_out.abs() + torch.tensor(1e-6, dtype=torch.bfloat16)
    x_abs = w.x.abs() + torch.tensor(1e-3, dtype=torch.bfloat16)
    m, n, k, e = g_abs.shape[0], g_abs.shape[1], x_abs.shape[1], w.num_groups
    off = w.offsets
    offd = torch.from_numpy(off).cuda()
    layout = qgg.LAYOUT_TRANSPOSED if mode == qgg.K_JAGGED else qgg.LAYOUT_TRANSPOSED_PADDED
    qa, sa = qgg.fp8_quant_colwise_jagged(g_abs.cuda(), offd, layout)
    qb, sb = qgg.fp8_quant_colwise_jagged(x_abs.cuda(), offd, layout)
    out = qgg.fp8_scaled_grouped_gemm(mode, qa, sa, qb, sb, offd, m_total=m)
    torch.cuda.synchronize()
    rng = np.random.default_rng(65)
    ci = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 22)]))
    cj = np.unique(np.concatenate([[0, k - 1], rng.integers(0, k, 22)]))
    oa, osa, _ = orc.quant_colwise_jagged(bits(g_abs[:, torch.from_numpy(ci)]), off,
                                          orc.TRANSPOSED)
    ob, osb, _ = orc.quant_colwise_jagged(bits(x_abs[:, torch.from_numpy(cj)]), off,
                                          orc.TRANSPOSED)
    big = int(np.argmax(w.group_sizes))
    assert w.group_sizes[big] > 14000
    li, lj = np.meshgrid(np.arange(len(ci)), np.arange(len(cj)), indexing="ij")
    grp = np.full(li.size, big)
    others = rng.integers(0, e, 3000)
    grp = np.concatenate([grp, others])
    li = np.concatenate([li.ravel(), rng.integers(0, len(ci), 3000)])
    lj = np.concatenate([lj.ravel(), rng.integers(0, len(cj), 3000)])
    keep = w.group_sizes[grp] > 0
    grp, li, lj = grp[keep], li[keep], lj[keep]
    c, b = orc.gemm_k_jagged_sample(oa, osa, ob, osb, off, m, grp, li, lj)
    got = out[torch.from_numpy(grp).cuda(), torch.from_numpy(ci[li]).cuda(),
              torch.from_numpy(cj[lj]).cuda()].cpu().numpy()
    worst_ratio(got, c, b, f"K-jagged mode {mode}, DeepSeek-MoE-16B routing (largest group "
                           f"{int(w.group_sizes[big])} tokens)")
