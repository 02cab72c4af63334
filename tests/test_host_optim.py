"""The paged optimizer's host-side update (qlora_adamw_host) against the
float64 AdamW oracle, on CPU (no GPU involved): several steps on a vector
large enough to be split across the library's worker threads, and the bf16
copy equal to the rounding of the fp32 master."""

import numpy as np
import torch

from oracle import bf16, optim

def _hp32():
    # the C ABI carries the hyperparameters as fp32: the oracle takes the same values
    f = lambda x: float(np.float32(x))
    return f(HP["lr"]), f(HP["betas"][0]), f(HP["betas"][1]), f(HP["eps"]), f(HP["weight_decay"])


HP = dict(lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.02)


def test_host_adamw_matches_oracle():
    import bit_nf4_quantized_06_b200 as q
    n = 200_003
    g = torch.Generator().manual_seed(5)
    master = torch.randn(n, generator=g) * 0.02
    m, v = torch.zeros(n), torch.zeros(n)
    param = torch.empty(n, dtype=torch.bfloat16)
    po, mo, vo = master.double().numpy().copy(), np.zeros(n), np.zeros(n)
    for t in range(1, 5):
        grad = torch.randn(n, generator=g) * 0.01
        q.qlora_adamw_host(master, grad, m, v, t, param=param, **HP)
        po, mo, vo = optim.adamw_step(po, grad.double().numpy(), mo, vo, t, *_hp32())
        assert np.allclose(master.double().numpy(), po, rtol=1e-6, atol=1e-5 * HP["lr"])
        assert np.allclose(m.double().numpy(), mo, rtol=1e-5, atol=1e-9)
        assert np.allclose(v.double().numpy(), vo, rtol=1e-5, atol=1e-14)
        assert np.array_equal(param.view(torch.int16).numpy().view(np.uint16),
                              bf16.round_f32_to_bf16_bits(master.numpy()))


def test_host_adamw_rejects_bad_hyperparameters():
    import ctypes
    import bit_nf4_quantized_06_b200 as q
    x = torch.zeros(8)
    hp = q.AdamwParams(1e-3, 0.9, 0.999, 0.0, 0.0, 1)                  # eps must be > 0
    assert q.lib.qlora_adamw_host(q._ptr(x), None, q._ptr(x), q._ptr(x), q._ptr(x), 8, ctypes.byref(hp)) == 1
