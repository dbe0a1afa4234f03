"""FP8 weight caching: the cached codes are reused while the weight is
unchanged and recomputed after an in-place update ("AMD Primus adds FP8/MXFP8
kernels ...", "What Primus adds for MoE training on MI355X")."""
import numpy as np
import pytest
import torch

import oracle as orc
import quantization_grouped_gemm_b200 as qgg
from quantization_grouped_gemm_b200 import workloads as wl


def test_cache_decides_on_version_and_storage_without_a_gpu():
    calls = []

    def fake(w, fmt=0, scale_max=0.0, q=None, scales=None):
        calls.append(w._version)
        return (q if q is not None else torch.zeros(w.shape, dtype=torch.uint8),
                scales if scales is not None else torch.zeros(w.shape[0]))

    c = qgg.Fp8WeightCache(quantize=fake)
    w = torch.ones(4, 8, dtype=torch.bfloat16)
    q1, s1 = c.rowwise(w)
    q2, s2 = c.rowwise(w)
    assert q1 is q2 and s1 is s2 and len(calls) == 1 and c.hits == 1
    w.mul_(2)  # an optimizer-style in-place update
    q3, _ = c.rowwise(w)
    assert len(calls) == 2 and q3 is q1  # recomputed into the same buffers
    c.rowwise(w, fmt=qgg.E4M3FNUZ)  # another format is another entry
    assert len(calls) == 3
    c.rowwise(w.clone())  # another tensor
    assert len(calls) == 4 and c.misses == 4


@pytest.mark.gpu
def test_cached_codes_are_reused_and_refreshed_after_an_update():
    w = wl.normal_bf16(77, 2, (3 * 96, 128), 0.02).cuda()
    c = qgg.Fp8WeightCache()
    q, s = c.rowwise(w)
    torch.cuda.synchronize()
    ref_q, ref_s, _ = orc.quant_rowwise(wl.bf16_bits(w.cpu()))
    assert (q.cpu().numpy() == ref_q).all()
    q.fill_(0xAB)  # a reuse must not run the kernel again
    q2, _ = c.rowwise(w)
    torch.cuda.synchronize()
    assert q2 is q and (q2 == 0xAB).all() and c.hits == 1
    w.mul_(3)  # in-place update: the next call quantises again
    q3, s3 = c.rowwise(w)
    torch.cuda.synchronize()
    ref_q3, ref_s3, _ = orc.quant_rowwise(wl.bf16_bits(w.cpu()))
    assert (q3.cpu().numpy() == ref_q3).all()
    assert (s3.cpu().numpy().view(np.uint32) == ref_s3.view(np.uint32)).all()


def test_mx_cache_decides_on_version_without_a_gpu():
    calls = []

    def fake(w, *rest, q=None, scales=None):
        calls.append(w._version)
        return (q if q is not None else torch.zeros(w.shape, dtype=torch.uint8),
                scales if scales is not None else torch.zeros(1, dtype=torch.int32))

    c = qgg.Fp8WeightCache(quantize=fake)
    w = torch.ones(4, 64, dtype=torch.bfloat16)
    off = torch.tensor([2, 4], dtype=torch.int32)
    q1, _ = c.mx_rowwise(w)
    assert c.mx_rowwise(w)[0] is q1 and len(calls) == 1
    c.mx_colwise_padded(w, off)
    c.mx_colwise_padded(w, off)
    assert len(calls) == 2 and c.hits == 2
    w.add_(1)
    assert c.mx_rowwise(w)[0] is q1 and len(calls) == 3
    off.add_(0)  # the offsets' in-place version counts too
    c.mx_colwise_padded(w, off)
    assert len(calls) == 4


@pytest.mark.gpu
def test_mx_cached_codes_match_the_oracle_and_refresh():
    w = wl.normal_bf16(78, 2, (2 * 128, 96), 0.02).cuda()
    c = qgg.Fp8WeightCache()
    q, s = c.mx_rowwise(w)
    torch.cuda.synchronize()
    ref_q, ref_s = orc.mx_quant_rowwise(wl.bf16_bits(w.cpu()))
    assert (q.cpu().numpy() == ref_q).all()
    assert (qgg.mx_scales_to_blocks(s, 3).cpu().numpy() == ref_s).all()
    q.fill_(0xAB)
    assert (c.mx_rowwise(w)[0] == 0xAB).all()
    w.mul_(5)
    q2, s2 = c.mx_rowwise(w)
    torch.cuda.synchronize()
    ref_q2, ref_s2 = orc.mx_quant_rowwise(wl.bf16_bits(w.cpu()))
    assert (q2.cpu().numpy() == ref_q2).all()
    assert (qgg.mx_scales_to_blocks(s2, 3).cpu().numpy() == ref_s2).all()
