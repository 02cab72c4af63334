"""GPU test of qlora_linear_fwd_noalloc, the forward for callers that cannot
hand the library a workspace (their device memory belongs to a pool of their
own, or an allocation is not allowed where they run). It uses one
library-owned scratch array of QLORA_NOALLOC_SCRATCH_BYTES instead, so it
must give exactly what qlora_linear_fwd gives with a caller workspace of that
size, call after call, although every call reuses the same array; and it must
refuse problems whose workspace would not fit in the array.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import linear, nf4

pytestmark = pytest.mark.gpu

TOL = 5e-3
SCRATCH = 8 * 1024 * 1024          # QLORA_NOALLOC_SCRATCH_BYTES
QLORA_ERR_WORKSPACE = 4


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_06_b200 as q
    return q


def _np(t):
    return t.detach().cpu().float().numpy()


def _same_size_workspace(device):
    # a caller workspace of exactly the scratch array's size: the workspace
    # forward then takes the same plan as the allocation-free one
    return torch.empty(SCRATCH, dtype=torch.uint8, device=device)


@pytest.mark.parametrize("n,k,m,r", [(512, 512, 300, 8), (384, 1024, 16, 100), (1000, 512, 3, 12)])
def test_noalloc_forward_matches_workspace_forward_twice(q, n, k, m, r):
    alpha = 16.0
    for call in range(2):                      # two calls in a row on the shared scratch
        seed = 7 * call + n + m
        w = synth.weight(n, k, seed=seed).cuda()
        x = synth.tokens(m, k, seed=seed).cuda()
        a = synth.lora_a(r, k, seed=seed).cuda()
        b = synth.lora_b(n, r, seed=seed).cuda()
        qw = q.qlora_quantize_nf4(w)
        y_same, u_same = q.qlora_linear_fwd(qw, x, a, b, alpha, ws=_same_size_workspace(x.device))
        y_ref, u_ref = q.qlora_linear_fwd(qw, x, a, b, alpha)
        y, u = q.qlora_linear_fwd_noalloc(qw, x, a, b, alpha)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_same.view(torch.int16))
        assert torch.equal(u.view(torch.int16), u_same.view(torch.int16))
        assert linear.rel_fro(_np(y), _np(y_ref)) <= TOL
        assert linear.rel_fro(_np(u), _np(u_ref)) <= TOL
        st, bits = q.qlora_device_status()
        assert st == 0, bits


def _first_too_large(q, n, k, r, m0=17):
    m = m0
    while q.qlora_fwd_workspace_bytes(m, n, k, r) <= SCRATCH:
        m += 1
    return m


def test_noalloc_near_its_limit_matches_oracle(q):
    # the 7B down projection (d_out 4096, d_in 11008, r = 64) at the token
    # count just below the first one whose workspace no longer fits in the
    # scratch array (3,072 on 148 SMs)
    n, k, r, alpha = 4096, 11008, 64, 16.0
    m = _first_too_large(q, n, k, r) - 1
    need = q.qlora_fwd_workspace_bytes(m, n, k, r)
    assert SCRATCH // 2 < need <= SCRATCH
    p = synth.Problem("down-near-limit", n, k, m, r, alpha, backward=False)
    t = synth.make(p, seed=3)
    qw = q.qlora_quantize_nf4(t["w"].cuda())
    x, a, b = (t[k_].cuda() for k_ in ("x", "a", "b"))
    for _ in range(2):
        y, u = q.qlora_linear_fwd_noalloc(qw, x, a, b, alpha)
        y_same, u_same = q.qlora_linear_fwd(qw, x, a, b, alpha, ws=_same_size_workspace(x.device))
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_same.view(torch.int16))
        assert torch.equal(u.view(torch.int16), u_same.view(torch.int16))
    o = nf4.quantize(t["w"].float().numpy())
    w_hat = nf4.dequantize(o["codes"], o["q2"], o["smax"]).astype(np.float64)
    s = alpha / r
    xn, an, bn = (t[k_].float().numpy().astype(np.float64) for k_ in ("x", "a", "b"))
    rows = np.array([0, 1, 127, 128, m // 2, m - 1])
    y_ref = xn[rows] @ w_hat.T + s * (xn[rows] @ an.T) @ bn.T
    assert linear.rel_fro(_np(y)[rows], y_ref) <= TOL
    assert linear.rel_fro(_np(u), s * (xn @ an.T)) <= TOL
    assert q.qlora_device_status() == (0, 0)


def test_noalloc_rejects_the_first_size_beyond_its_scratch(q):
    # the first token count whose workspace exceeds the array is refused
    # before anything is launched, with real buffers in place
    n, k, r, alpha = 4096, 11008, 64, 16.0
    m = _first_too_large(q, n, k, r)
    assert m < 8192
    qw = q.qlora_quantize_nf4(synth.weight(n, k, seed=1).cuda())
    x = synth.tokens(m, k, seed=1).cuda()
    a = synth.lora_a(r, k, seed=1).cuda()
    b = synth.lora_b(n, r, seed=1).cuda()
    with pytest.raises(q.QloraError) as e:
        q.qlora_linear_fwd_noalloc(qw, x, a, b, alpha)
    assert e.value.status == QLORA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert q.qlora_device_status() == (0, 0)


def test_noalloc_rejects_problems_beyond_its_scratch(q):
    n, k, r = 256, 4096, 64
    m = 200000
    assert q.qlora_fwd_workspace_bytes(m, n, k, r) > SCRATCH
    s = q.Nf4Struct(n, k, 64, 256, 256, 256, 256)      # never dereferenced: rejected first
    st = q.lib.qlora_linear_fwd_noalloc(ctypes.byref(s), ctypes.c_void_p(256), m, ctypes.c_void_p(256),
                                        ctypes.c_void_p(256), r, 16.0, ctypes.c_void_p(256), None, None)
    assert st == QLORA_ERR_WORKSPACE
