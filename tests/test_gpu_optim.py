"""GPU parity of the AdamW step for the adapters, with the Adam states in
device memory and paged out to pinned host memory (the GPU addresses them
directly). Compared with the float64 oracle over several steps; the bf16
copy must be exactly the rounding of the fp32 master."""

import numpy as np
import pytest
import torch

from oracle import bf16, optim

pytestmark = pytest.mark.gpu

HP = dict(lr=2e-3, betas=(0.9, 0.995), eps=1e-8, weight_decay=0.01)


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_06_b200 as q
    return q


@pytest.mark.parametrize("n,offset,paged", [(966656, 0, False), (966656, 0, True), (1001, 1, True), (7, 0, False)])
def test_adamw_parity(q, n, offset, paged):
    g = torch.Generator().manual_seed(n + offset)
    p0 = torch.randn(n + offset, generator=g) * 0.02
    master = p0.clone().cuda()
    m = torch.zeros(n + offset, pin_memory=paged) if paged else torch.zeros(n + offset, device="cuda")
    v = torch.zeros(n + offset, pin_memory=paged) if paged else torch.zeros(n + offset, device="cuda")
    param = torch.empty(n + offset, dtype=torch.bfloat16, device="cuda")
    po, mo, vo = p0[offset:].double().numpy(), np.zeros(n), np.zeros(n)
    for t in range(1, 4):
        grad = torch.randn(n + offset, generator=g) * 0.01
        q.qlora_adamw_step(master[offset:], grad[offset:].cuda(), m[offset:], v[offset:], t, param=param[offset:], **HP)
        torch.cuda.synchronize()
        po, mo, vo = optim.adamw_step(po, grad[offset:].double().numpy(), mo, vo, t, HP["lr"], HP["betas"][0],
                                      HP["betas"][1], HP["eps"], HP["weight_decay"])
        got = master[offset:].cpu().double().numpy()
        # fp32 state against the float64 oracle: where m cancels to near zero
        # its absolute rounding (~1e-10) is amplified by step_size / denom, so
        # the bound has an absolute part of 1e-5 * lr
        assert np.allclose(got, po, rtol=1e-6, atol=1e-5 * HP["lr"])
        # m = b1 m + (1 - b1) g can cancel to near zero: compare it against the
        # size of its terms (|g| ~ 1e-2, fp32 rounding ~1e-9 absolute)
        assert np.allclose(m[offset:].cpu().double().numpy(), mo, rtol=1e-5, atol=1e-9)
        assert np.allclose(v[offset:].cpu().double().numpy(), vo, rtol=1e-5, atol=1e-14)
        rb = bf16.round_f32_to_bf16_bits(master[offset:].cpu().numpy())
        assert np.array_equal(param[offset:].cpu().view(torch.int16).numpy().view(np.uint16), rb)
    assert q.qlora_device_status() == (0, 0)
