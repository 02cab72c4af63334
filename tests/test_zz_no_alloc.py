"""GPU test of qlora_linear_fwd_noalloc, the forward for callers that cannot
hand the library a workspace (their device memory belongs to a pool of their
own, or an allocation is not allowed where they run). It must give what
qlora_linear_fwd gives with a caller workspace, call after call, although
every call reuses the same library-owned scratch array.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import linear

pytestmark = pytest.mark.gpu

TOL = 5e-3


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_06_b200 as q
    return q


def _np(t):
    return t.detach().cpu().float().numpy()


@pytest.mark.parametrize("n,k,m,r", [(512, 512, 300, 8), (384, 1024, 16, 100)])
def test_noalloc_forward_matches_workspace_forward_twice(q, n, k, m, r):
    alpha = 16.0
    for call in range(2):                      # two calls in a row on the shared scratch
        seed = 7 * call + n + m
        w = synth.weight(n, k, seed=seed).cuda()
        x = synth.tokens(m, k, seed=seed).cuda()
        a = synth.lora_a(r, k, seed=seed).cuda()
        b = synth.lora_b(n, r, seed=seed).cuda()
        qw = q.qlora_quantize_nf4(w)
        y_ref, u_ref = q.qlora_linear_fwd(qw, x, a, b, alpha)
        y, u = q.qlora_linear_fwd_noalloc(qw, x, a, b, alpha)
        torch.cuda.synchronize()
        assert linear.rel_fro(_np(y), _np(y_ref)) <= TOL
        assert linear.rel_fro(_np(u), _np(u_ref)) <= TOL
        st, bits = q.qlora_device_status()
        assert st == 0, bits


def test_noalloc_rejects_problems_beyond_its_scratch(q):
    n, k, r = 256, 4096, 64
    m = 200000
    assert q.qlora_fwd_workspace_bytes(m, n, k, r) > 8 * 1024 * 1024
    s = q.Nf4Struct(n, k, 64, 256, 256, 256, 256)      # never dereferenced: rejected first
    st = q.lib.qlora_linear_fwd_noalloc(ctypes.byref(s), ctypes.c_void_p(256), m, ctypes.c_void_p(256),
                                        ctypes.c_void_p(256), r, 16.0, ctypes.c_void_p(256), None, None)
    assert st == 4      # QLORA_ERR_WORKSPACE
