"""GPU parity of the AdamW step for the adapters, with the Adam states in
device memory and paged out to pinned host memory (the GPU addresses them
directly). Compared with the float64 oracle over several steps; the bf16
copy must be exactly the rounding of the fp32 master."""

import numpy as np
import pytest
import torch

from oracle import bf16, optim

pytestmark = pytest.mark.gpu

def _hp32():
    # the C ABI carries the hyperparameters as fp32: the oracle takes the same values
    f = lambda x: float(np.float32(x))
    return f(HP["lr"]), f(HP["betas"][0]), f(HP["betas"][1]), f(HP["eps"]), f(HP["weight_decay"])


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
        po, mo, vo = optim.adamw_step(po, grad[offset:].double().numpy(), mo, vo, t, *_hp32())
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


def test_paged_chain_matches_oracle(q):
    # D2H gradient, CPU update on pinned states as a stream host function, H2D bf16 adapter
    n = 300_001
    g = torch.Generator().manual_seed(11)
    master_h = (torch.randn(n, generator=g) * 0.02).pin_memory()
    m_h, v_h = torch.zeros(n).pin_memory(), torch.zeros(n).pin_memory()
    grad_h = torch.empty(n).pin_memory()
    param_h = torch.empty(n, dtype=torch.bfloat16).pin_memory()
    param_d = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    po, mo, vo = master_h.double().numpy().copy(), np.zeros(n), np.zeros(n)
    side = torch.cuda.Stream()
    for t in range(1, 4):
        grad_d = (torch.randn(n, generator=g) * 0.01).cuda()
        side.wait_stream(torch.cuda.current_stream())
        q.qlora_adamw_paged(grad_d, master_h, m_h, v_h, grad_h, t, param_dev=param_d, param_host=param_h,
                            stream=side, **HP)
        side.synchronize()
        po, mo, vo = optim.adamw_step(po, grad_d.cpu().double().numpy(), mo, vo, t, *_hp32())
        assert np.allclose(master_h.double().numpy(), po, rtol=1e-6, atol=1e-5 * HP["lr"])
        rb = bf16.round_f32_to_bf16_bits(master_h.numpy())
        assert np.array_equal(param_d.cpu().view(torch.int16).numpy().view(np.uint16), rb)


@pytest.mark.parametrize("n,offset", [(966656, 0), (1001, 1)])
def test_staged_states_match_device_states_bit_for_bit(q, n, offset):
    # m, v in pinned host memory staged through device buffers by copies on
    # the stream: the same kernel on the same values as device-resident states
    g = torch.Generator().manual_seed(5 * n + offset)
    p0 = torch.randn(n + offset, generator=g) * 0.02
    master_a, master_b = p0.clone().cuda(), p0.clone().cuda()
    m_d, v_d = torch.zeros(n + offset, device="cuda"), torch.zeros(n + offset, device="cuda")
    m_h, v_h = torch.zeros(n + offset).pin_memory(), torch.zeros(n + offset).pin_memory()
    m_s, v_s = torch.empty(n + offset, device="cuda"), torch.empty(n + offset, device="cuda")
    pa = torch.empty(n + offset, dtype=torch.bfloat16, device="cuda")
    pb = torch.empty(n + offset, dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    for t in range(1, 4):
        grad = (torch.randn(n + offset, generator=g) * 0.01).cuda()
        q.qlora_adamw_step(master_a[offset:], grad[offset:], m_d[offset:], v_d[offset:], t, param=pa[offset:], **HP)
        side.wait_stream(torch.cuda.current_stream())
        q.qlora_adamw_staged(master_b[offset:], grad[offset:], m_h[offset:], v_h[offset:], m_s[offset:],
                             v_s[offset:], t, param=pb[offset:], stream=side, **HP)
        side.synchronize()
        torch.cuda.synchronize()
        assert torch.equal(master_a, master_b)
        assert torch.equal(m_d.cpu(), m_h) and torch.equal(v_d.cpu(), v_h)
        assert torch.equal(pa.view(torch.int16), pb.view(torch.int16))
    assert q.qlora_device_status() == (0, 0)


def test_staged_rejects_bad_arguments_before_enqueueing(q):
    n = 64
    master = torch.zeros(n, device="cuda")
    grad = torch.zeros(n, device="cuda")
    m_h, v_h = torch.zeros(n).pin_memory(), torch.zeros(n).pin_memory()
    m_s, v_s = torch.empty(n, device="cuda"), torch.empty(n, device="cuda")
    with pytest.raises(q.QloraError):
        q.qlora_adamw_staged(master, grad, m_h, v_h, m_s, v_s, 0)          # step must be >= 1
    with pytest.raises(q.QloraError):
        q.qlora_adamw_staged(master, grad, m_h, v_h, m_s, v_s, 1, eps=0.0)
    assert torch.equal(m_h, torch.zeros(n))
