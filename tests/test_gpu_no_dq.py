"""GPU parity of the 4.5-bit format (no double quantization: one fp32 scale
per 64-weight block, «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나», § "메모리 회계").
Codes and block scales bit-exact with the oracle; restore bit-exact (also
inside the tensor-core GEMM); forward, backward, decode and merge within the
usual bounds."""

import numpy as np
import pytest
import torch

import synth
from oracle import bf16 as obf16
from oracle import linear, nf4

pytestmark = pytest.mark.gpu
TOL = 5e-3


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_06_b200 as q
    return q


def _np(t):
    return t.detach().cpu().float().numpy()


def _bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("n,k,outl", [(512, 512, False), (200, 192, True), (11008, 4096, True)])
def test_quantize_and_restore_bit_exact(q, n, k, outl):
    w = synth.weight(n, k, seed=n, outliers=outl)
    o = nf4.quantize(w.float().numpy())
    qw = q.qlora_quantize_nf4(w.cuda(), dq=False)
    w_hat = q.qlora_dequantize(qw)
    torch.cuda.synchronize()
    assert qw.scale_codes.numel() == 0
    assert np.array_equal(qw.codes.cpu().numpy(), o["codes"].ravel())
    assert np.array_equal(qw.absmax.cpu().numpy().view(np.uint32), o["absmax"].view(np.uint32))
    assert np.array_equal(_bits(w_hat), nf4.dequantize_bits_no_dq(o["codes"], o["absmax"]))


def test_gemm_restore_exact_without_dq(q):
    n, k, r = 320, 192, 16
    w = synth.weight(n, k, seed=5, outliers=True)
    o = nf4.quantize(w.float().numpy())
    qw = q.qlora_quantize_nf4(w.cuda(), dq=False)
    x = torch.eye(k, dtype=torch.bfloat16)
    y, _ = q.qlora_linear_fwd_ex(qw, x.cuda(), synth.lora_a(r, k).cuda(),
                                 torch.zeros((n, r), dtype=torch.bfloat16).cuda(), 16.0, path=q.FWD_GEMM)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y).T, nf4.dequantize_bits_no_dq(o["codes"], o["absmax"]))


@pytest.mark.parametrize("n,k,m,r,path", [(512, 512, 300, 8, "gemm"), (384, 1024, 16, 64, "gemm"),
                                          (4096, 4096, 1, 64, "gemv"), (1000, 512, 9, 12, "gemv"),
                                          (1000, 192, 5, 8, "gemv"), (24, 4096, 1, 16, "gemv")])
def test_forward_parity_without_dq(q, n, k, m, r, path):
    alpha = 16.0
    w = synth.weight(n, k, seed=k + m, outliers=True)
    x, a, b = synth.tokens(m, k, seed=2), synth.lora_a(r, k, seed=3), synth.lora_b(n, r, seed=4)
    o = nf4.quantize(w.float().numpy())
    w_hat = nf4.dequantize_no_dq(o["codes"], o["absmax"])
    y_ref, _ = linear.forward(_np(x), w_hat, _np(a), _np(b), alpha / r)
    qw = q.qlora_quantize_nf4(w.cuda(), dq=False)
    mode = q.FWD_GEMM if path == "gemm" else q.FWD_GEMV
    y, _ = q.qlora_linear_fwd_ex(qw, x.cuda(), a.cuda(), b.cuda(), alpha, path=mode)
    torch.cuda.synchronize()
    assert linear.rel_fro(_np(y), y_ref) <= TOL
    assert q.qlora_device_status() == (0, 0)


def test_backward_parity_without_dq(q):
    n, k, m, r, alpha = 384, 512, 257, 32, 16.0
    w = synth.weight(n, k, seed=9, outliers=True)
    x, a, b = synth.tokens(m, k, seed=2), synth.lora_a(r, k, seed=3), synth.lora_b(n, r, seed=4)
    dy = synth.grad_out(m, n, seed=5)
    o = nf4.quantize(w.float().numpy())
    w_hat = nf4.dequantize_no_dq(o["codes"], o["absmax"])
    dx_ref, da_ref, db_ref = linear.backward(_np(x), _np(dy), w_hat, _np(a), _np(b), alpha / r)
    qw = q.qlora_quantize_nf4(w.cuda(), dq=False)
    dx, da, db = q.qlora_linear_bwd(qw, x.cuda(), None, dy.cuda(), a.cuda(), b.cuda(), alpha)
    torch.cuda.synchronize()
    assert linear.rel_fro(_np(dx), dx_ref) <= TOL
    assert linear.rel_fro(_np(da), da_ref) <= TOL
    assert linear.rel_fro(_np(db), db_ref) <= TOL


def test_merge_without_dq(q):
    n, k, r, alpha = 256, 384, 16, 16.0
    w = synth.weight(n, k, seed=12, outliers=True)
    a = synth.lora_a(r, k, seed=3)
    b = (synth.lora_b(n, r, seed=4).float() * 20.0).to(torch.bfloat16)
    o = nf4.quantize(w.float().numpy())
    w_hat = nf4.dequantize_no_dq(o["codes"], o["absmax"])
    ref = linear.merge_bits(w_hat, _np(a), _np(b), float(np.float32(alpha) / np.float32(r)))
    qw = q.qlora_quantize_nf4(w.cuda(), dq=False)
    got = _bits(q.qlora_merge_lora(qw, a.cuda(), b.cuda(), alpha))
    key = lambda z: np.where(z.astype(np.int32) & 0x8000, -(z.astype(np.int32) & 0x7FFF), z.astype(np.int32))
    d = np.abs(key(got) - key(ref))
    assert d.max() <= 1 and np.mean(d != 0) < 1e-3
