"""Failure detection on the GPU without a fault.

Every wait in the library's kernels is bounded; when one runs out the kernel
records a status bit and returns normally. This test makes one wait run out
(a barrier that nothing completes) and checks that the host sees the timeout,
that reading the status clears it, and that the context is still usable.
"""

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

TIMEOUT = 7
BIT_SELFTEST = 0x10


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_06_b200 as q
    return q


def test_bounded_wait_reports_timeout_and_context_survives(q):
    st, _ = q.qlora_device_status()
    assert st == 0
    q.qlora_selftest_wait_timeout(20000)          # 20 ms wait that nothing completes
    st, bits = q.qlora_device_status()
    assert st == TIMEOUT and bits == BIT_SELFTEST
    st, bits = q.qlora_device_status()            # reading cleared it
    assert st == 0 and bits == 0
    # the context still runs kernels correctly afterwards
    w = synth.weight(256, 512, seed=5).cuda()
    qw = q.qlora_quantize_nf4(w)
    w_hat = q.qlora_dequantize(qw)
    torch.cuda.synchronize()
    assert torch.isfinite(w_hat.float()).all()
    assert q.qlora_device_status() == (0, 0)
