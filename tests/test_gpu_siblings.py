"""Fused sibling projections (q/k/v or gate/up sharing x): the weights are
concatenated along d_out and quantized once, the adapters stacked along the
rank (A_cat = [A_q; A_k; A_v]) with B block-diagonal, so one forward streams
x and x A^T once. With alpha scaled by the number of siblings (s = alpha / r
per projection is unchanged), the fused call gives each projection's output.

The stored format is bit-identical to quantizing each weight on its own when
every weight holds a whole number of 256-block groups (true for d_in a
multiple of 64 and d_out * d_in / 64 a multiple of 256)."""

import numpy as np
import pytest
import torch

import synth
from oracle import linear, nf4

pytestmark = pytest.mark.gpu
TOL = 5e-3


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_06_b200 as q
    return q


def _np(t):
    return t.detach().cpu().float().numpy()


def _block_diag(bs):
    n = sum(b.shape[0] for b in bs)
    r = sum(b.shape[1] for b in bs)
    out = torch.zeros((n, r), dtype=torch.bfloat16)
    i = j = 0
    for b in bs:
        out[i:i + b.shape[0], j:j + b.shape[1]] = b
        i += b.shape[0]
        j += b.shape[1]
    return out


@pytest.mark.parametrize("m", [1, 300])
def test_fused_siblings_match_separate_calls(q, m):
    k, n, r, alpha = 512, 512, 16, 16.0
    ws = [synth.weight(n, k, seed=40 + i) for i in range(3)]
    As = [synth.lora_a(r, k, seed=50 + i) for i in range(3)]
    Bs = [(synth.lora_b(n, r, seed=60 + i).float() * 10).to(torch.bfloat16) for i in range(3)]
    x = synth.tokens(m, k, seed=7)
    # separate
    sep = []
    qws = [q.qlora_quantize_nf4(w.cuda()) for w in ws]
    for qw, a, b in zip(qws, As, Bs):
        y, _ = q.qlora_linear_fwd(qw, x.cuda(), a.cuda(), b.cuda(), alpha)
        sep.append(y)
    # fused
    w_cat = torch.cat(ws, 0).cuda()
    qc = q.qlora_quantize_nf4(w_cat)
    a_cat = torch.cat(As, 0).cuda()
    b_bd = _block_diag(Bs).cuda()
    y_cat, _ = q.qlora_linear_fwd(qc, x.cuda(), a_cat, b_bd, 3 * alpha)
    torch.cuda.synchronize()
    # stored format identical to the separate quantizations
    assert torch.equal(qc.codes.cpu(), torch.cat([qw.codes.cpu() for qw in qws]))
    assert torch.equal(qc.scale_codes.cpu(), torch.cat([qw.scale_codes.cpu() for qw in qws]))
    assert torch.equal(qc.absmax.cpu(), torch.cat([qw.absmax.cpu() for qw in qws]))
    for i in range(3):
        o = nf4.quantize(ws[i].float().numpy())
        w_hat = nf4.dequantize(o["codes"], o["q2"], o["smax"])
        y_ref, _ = linear.forward(_np(x), w_hat, _np(As[i]), _np(Bs[i]), alpha / r)
        assert linear.rel_fro(_np(y_cat[:, i * n:(i + 1) * n]), y_ref) <= TOL
        assert linear.rel_fro(_np(y_cat[:, i * n:(i + 1) * n]), _np(sep[i])) <= TOL
    assert q.qlora_device_status() == (0, 0)


def test_fused_siblings_backward(q):
    # dX sums the three projections' contributions; dA_cat stacks the dA's;
    # the diagonal blocks of dB are the dB's (off-diagonal blocks are not
    # parameters and are left to the optimizer to ignore)
    k, n, r, alpha, m = 512, 384, 16, 16.0, 257
    ws = [synth.weight(n, k, seed=70 + i) for i in range(2)]
    As = [synth.lora_a(r, k, seed=80 + i) for i in range(2)]
    Bs = [(synth.lora_b(n, r, seed=90 + i).float() * 10).to(torch.bfloat16) for i in range(2)]
    x, dy = synth.tokens(m, k, seed=8), synth.grad_out(m, 2 * n, seed=9)
    qc = q.qlora_quantize_nf4(torch.cat(ws, 0).cuda())
    dx, da, db = q.qlora_linear_bwd(qc, x.cuda(), None, dy.cuda(), torch.cat(As, 0).cuda(),
                                    _block_diag(Bs).cuda(), 2 * alpha)
    torch.cuda.synchronize()
    dx_ref = 0
    for i in range(2):
        o = nf4.quantize(ws[i].float().numpy())
        w_hat = nf4.dequantize(o["codes"], o["q2"], o["smax"])
        dxi, dai, dbi = linear.backward(_np(x), _np(dy)[:, i * n:(i + 1) * n], w_hat, _np(As[i]), _np(Bs[i]),
                                        alpha / r)
        dx_ref = dx_ref + dxi
        assert linear.rel_fro(_np(da)[i * r:(i + 1) * r], dai) <= TOL
        assert linear.rel_fro(_np(db)[i * n:(i + 1) * n, i * r:(i + 1) * r], dbi) <= TOL
    assert linear.rel_fro(_np(dx), dx_ref) <= TOL
