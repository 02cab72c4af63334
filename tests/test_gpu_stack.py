"""GPU parity on the whole 7B-shaped stack's own weights.

The stack benchmark draws every projection's W, A and B on the GPU
(synth.stack_linear) and its activations with synth.stack_activations. Here
the same tensors go through the CUDA path and the CPU oracle:

* layers 0 and 31, all seven projections (q, k, v, o 4096x4096; gate, up
  11008x4096; down 4096x11008): codes, scale codes and s_max bit-exact over
  the whole weight; forward y and dX on sampled token rows, dA and dB in
  full, at 4096 tokens with r = 64, within 5e-3 of the fp64 oracle on the
  oracle's own restored weight;
* layers 1..30, one projection each (rotating through the seven): the first
  and last 64 rows (whole double-quantization groups for both widths)
  bit-exact against the oracle's quantizer.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import linear, nf4

pytestmark = pytest.mark.gpu

TOL = 5e-3
M, R, ALPHA = 4096, 64, 16.0


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_06_b200 as q
    return q


@pytest.fixture(scope="module")
def acts():
    return synth.stack_activations(M, device="cuda")


def _np(t):
    return t.detach().cpu().float().numpy()


def _check_quant(qw, o, rows=None):
    codes = qw.codes.view(qw.n_out, qw.k_in // 2).cpu().numpy()
    q2 = qw.scale_codes.cpu().numpy()
    smax = qw.absmax.cpu().numpy()
    if rows is None:
        assert np.array_equal(codes, o["codes"])
        assert np.array_equal(q2, o["q2"])
        assert np.array_equal(smax.view(np.uint32), o["smax"].view(np.uint32))
        return
    lo, hi = rows
    kb = qw.k_in // 64
    assert np.array_equal(codes[lo:hi], o["codes"])
    assert np.array_equal(q2[lo * kb:hi * kb], o["q2"])
    g0, g1 = lo * kb // 256, hi * kb // 256
    assert np.array_equal(smax[g0:g1].view(np.uint32), o["smax"].view(np.uint32))


@pytest.mark.parametrize("layer", [0, 31])
@pytest.mark.parametrize("idx", range(7), ids=[p[0] for p in synth.STACK7B_LAYER])
def test_stack_layer_full(q, acts, layer, idx):
    xs, dys = acts
    _, n, k = synth.STACK7B_LAYER[idx]
    w, a, b = synth.stack_linear(layer, idx, r=R, device="cuda")
    qw = q.qlora_quantize_nf4(w)
    x, dy = xs[k], dys[n]
    y, u = q.qlora_linear_fwd(qw, x, a, b, ALPHA)
    dx, da, db = q.qlora_linear_bwd(qw, x, u, dy, a, b, ALPHA)
    torch.cuda.synchronize()
    assert q.qlora_device_status() == (0, 0)

    o = nf4.quantize(_np(w))
    _check_quant(qw, o)
    w_hat = nf4.dequantize(o["codes"], o["q2"], o["smax"]).astype(np.float64)
    del o
    s = ALPHA / R
    xn, an, bn, dyn = (_np(t).astype(np.float64) for t in (x, a, b, dy))
    rows = np.array([0, 1, 255, 256, 2047, 4095])
    y_ref = xn[rows] @ w_hat.T + s * (xn[rows] @ an.T) @ bn.T
    assert linear.rel_fro(_np(y)[rows], y_ref) <= TOL
    v = dyn @ bn
    dx_ref = dyn[rows] @ w_hat + s * v[rows] @ an
    assert linear.rel_fro(_np(dx)[rows], dx_ref) <= TOL
    assert linear.rel_fro(_np(da), s * (v.T @ xn)) <= TOL
    assert linear.rel_fro(_np(db), s * (dyn.T @ (xn @ an.T))) <= TOL


def test_stack_middle_layers_sampled_rows(q):
    for layer in range(1, 31):
        idx = layer % 7
        _, n, k = synth.STACK7B_LAYER[idx]
        w, _, _ = synth.stack_linear(layer, idx, r=R, device="cuda")
        qw = q.qlora_quantize_nf4(w)
        torch.cuda.synchronize()
        for lo, hi in ((0, 64), (n - 64, n)):
            o = nf4.quantize(_np(w[lo:hi]))
            _check_quant(qw, o, rows=(lo, hi))
        del w, qw
    assert q.qlora_device_status() == (0, 0)
