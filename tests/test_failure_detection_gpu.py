"""Failure detection on the GPU without a fault.

Every device-side wait of the library is bounded: when it gives up it ORs
FP8QGG_STATUS_TIMEOUT into the caller's status word and the kernel returns, so
the context stays usable.  Here the wait of a tall unit's cast for the unit's
merged absmax is made to run out on purpose: the test hook
fp8qgg_test_unit_wait makes it also wait for chunk arrivals that never come
(a count that nothing reaches) and shortens its limit to a few milliseconds.
The call must return, report the timeout, and leave the device able to run a
normal call that matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import quantization_grouped_gemm_b200 as qgg
from quantization_grouped_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout", [qgg.LAYOUT_SAME, qgg.LAYOUT_TRANSPOSED,
                                    qgg.LAYOUT_TRANSPOSED_PADDED])
def test_unit_absmax_wait_runs_out_and_is_reported(layout):
    sizes = [2500, 7, 1300]  # two groups taller than one chunk: their casts wait
    w = wl.random_jagged(77, sizes, 192)
    x = w.x.cuda()
    off = torch.from_numpy(w.offsets).cuda()
    lib = qgg.lib()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.fp8qgg_test_unit_wait(1, 3_000_000) == 0  # one arrival too many, 3 ms
    try:
        qgg.fp8_quant_colwise_jagged(x, off, layout, status=status)
        torch.cuda.synchronize()
    finally:
        assert lib.fp8qgg_test_unit_wait(0, 0) == 0
    assert int(status.item()) & qgg.STATUS_TIMEOUT
    # the device still runs normal calls, with the right results
    status.zero_()
    q, s = qgg.fp8_quant_colwise_jagged(x, off, qgg.LAYOUT_SAME, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    q_ref, s_ref, _ = orc.quant_colwise_jagged(wl.bf16_bits(w.x), w.offsets, orc.SAME)
    assert (q.cpu().numpy() == q_ref).all()
    assert (s.cpu().numpy().view(np.uint32) == s_ref.view(np.uint32)).all()
