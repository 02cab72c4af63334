"""GPU parity for the two further scale codes of the double quantization
(QLORA_DQ_U8_255: the unsigned 255-step grid; QLORA_DQ_S8_MID: the signed
code centred on the group's mid-range, two constants per group), against the
oracle's definitions (oracle/nf4.py, scale-code variants):

* quantizer: codes, scale codes and group constants bit-exact;
* restore: the standalone restore, the restore inside the forward and dX
  GEMMs (x = I, dY = I) and inside the decode GEMV (one-hot tokens) bit-exact;
* forward, backward, decode and merge within their usual tolerances.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import bf16 as obf16
from oracle import linear, nf4

pytestmark = pytest.mark.gpu

TOL = 5e-3
CODES = [("u8_255", 1), ("s8_mid", 2)]


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_06_b200 as q
    return q


@pytest.fixture(autouse=True)
def _status_clear(q):
    yield
    st, bits = q.qlora_device_status()
    assert st == 0 and bits == 0, f"device status {st} bits {bits:#x}"


def _np(t):
    return t.detach().cpu().float().numpy()


def _bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def _weight(n, k, seed):
    w = synth.weight(n, k, seed=seed, outliers=True)
    if n >= 4:
        w[1, : min(k, 128)] = 0                       # zero blocks
        w[3, :] = w[3, :].abs().max()                 # a row of equal scales
    return w


@pytest.mark.parametrize("code,cid", CODES, ids=[c for c, _ in CODES])
@pytest.mark.parametrize("n,k", [(512, 512), (37, 192), (1024, 1088), (3, 64)])
def test_quantize_and_restore_bit_exact(q, code, cid, n, k):
    w = _weight(n, k, seed=n + k)
    o = nf4.quantize_code(w.float().numpy(), code)
    qw = q.qlora_quantize_nf4(w.cuda(), dq_code=cid)
    wh = q.qlora_dequantize(qw)
    torch.cuda.synchronize()
    assert np.array_equal(qw.codes.cpu().numpy(), o["codes"].ravel())
    assert np.array_equal(qw.scale_codes.cpu().numpy(), o["q2"])
    assert np.array_equal(qw.absmax.cpu().numpy().view(np.uint32), o["gdata"].ravel().view(np.uint32))
    assert np.array_equal(_bits(wh), nf4.dequantize_bits_code(o["codes"], o["q2"], o["gdata"], code))


@pytest.mark.parametrize("code,cid", CODES, ids=[c for c, _ in CODES])
@pytest.mark.parametrize("n,k", [(320, 192), (256, 512)])
def test_gemm_restores_exactly(q, code, cid, n, k):
    # x = I (k tokens; 512 tokens take the 512-token tiles for the unsigned
    # code) and dY = I (n tokens) with B = 0 give W_hat^T and W_hat bit for bit
    r = 16
    w = _weight(n, k, seed=3 * n + k)
    o = nf4.quantize_code(w.float().numpy(), code)
    ref = nf4.dequantize_bits_code(o["codes"], o["q2"], o["gdata"], code)
    qw = q.qlora_quantize_nf4(w.cuda(), dq_code=cid)
    a = synth.lora_a(r, k).cuda()
    b = torch.zeros((n, r), dtype=torch.bfloat16, device="cuda")
    y, _ = q.qlora_linear_fwd_ex(qw, torch.eye(k, dtype=torch.bfloat16, device="cuda"), a, b, 16.0, path=q.FWD_GEMM)
    dx, _, _ = q.qlora_linear_bwd(qw, synth.tokens(n, k).cuda(), None, torch.eye(n, dtype=torch.bfloat16, device="cuda"),
                                  a, b, 16.0)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y).T, ref)
    assert np.array_equal(_bits(dx), ref)


@pytest.mark.parametrize("code,cid", CODES, ids=[c for c, _ in CODES])
def test_gemv_restores_exactly(q, code, cid):
    n, k, r = 1001, 4096, 8
    w = _weight(n, k, seed=11)
    o = nf4.quantize_code(w.float().numpy(), code)
    ref = nf4.dequantize_bits_code(o["codes"], o["q2"], o["gdata"], code)
    qw = q.qlora_quantize_nf4(w.cuda(), dq_code=cid)
    x = torch.zeros((3, k), dtype=torch.bfloat16)
    x[0, 5] = 1
    x[2, 4000] = 1
    y, _ = q.qlora_linear_fwd_ex(qw, x.cuda(), synth.lora_a(r, k).cuda(), torch.zeros((n, r), dtype=torch.bfloat16,
                                 device="cuda"), 16.0, path=q.FWD_GEMV)
    torch.cuda.synchronize()
    yb = _bits(y)
    assert np.array_equal(yb[0], ref[:, 5]) and np.array_equal(yb[2], ref[:, 4000]) and np.all(yb[1] == 0)


@pytest.mark.parametrize("code,cid", CODES, ids=[c for c, _ in CODES])
@pytest.mark.parametrize("n,k,m,r", [(1000, 512, 300, 16), (384, 1024, 513, 64), (4096, 4096, 1, 64)])
def test_forward_backward_parity(q, code, cid, n, k, m, r):
    alpha = 16.0
    s = alpha / r
    t = {"w": _weight(n, k, seed=n + m), "x": synth.tokens(m, k, seed=1), "a": synth.lora_a(r, k, seed=2),
         "b": synth.lora_b(n, r, seed=3), "dy": synth.grad_out(m, n, seed=4)}
    o = nf4.quantize_code(t["w"].float().numpy(), code)
    w_hat = nf4.dequantize_code(o["codes"], o["q2"], o["gdata"], code)
    y_ref, u_ref = linear.forward(_np(t["x"]), w_hat, _np(t["a"]), _np(t["b"]), s)
    qw = q.qlora_quantize_nf4(t["w"].cuda(), dq_code=cid)
    x, a, b, dy = (t[k_].cuda() for k_ in ("x", "a", "b", "dy"))
    y, u = q.qlora_linear_fwd(qw, x, a, b, alpha)
    torch.cuda.synchronize()
    assert linear.rel_fro(_np(y), y_ref) <= TOL
    if m > 16:
        dx_ref, da_ref, db_ref = linear.backward(_np(t["x"]), _np(t["dy"]), w_hat, _np(t["a"]), _np(t["b"]), s)
        dx, da, db = q.qlora_linear_bwd(qw, x, u, dy, a, b, alpha)
        torch.cuda.synchronize()
        assert linear.rel_fro(_np(dx), dx_ref) <= TOL
        assert linear.rel_fro(_np(da), da_ref) <= TOL
        assert linear.rel_fro(_np(db), db_ref) <= TOL


@pytest.mark.parametrize("code,cid", CODES, ids=[c for c, _ in CODES])
def test_merge_parity(q, code, cid):
    n, k, r, alpha = 256, 384, 16, 16.0
    w = _weight(n, k, seed=12)
    a = synth.lora_a(r, k, seed=3)
    b = (synth.lora_b(n, r, seed=4).float() * 20.0).to(torch.bfloat16)
    o = nf4.quantize_code(w.float().numpy(), code)
    w_hat = nf4.dequantize_code(o["codes"], o["q2"], o["gdata"], code)
    ref = linear.merge_bits(w_hat, _np(a), _np(b), float(np.float32(alpha) / np.float32(r)))
    qw = q.qlora_quantize_nf4(w.cuda(), dq_code=cid)
    got = _bits(q.qlora_merge_lora(qw, a.cuda(), b.cuda(), alpha))
    # the GPU adds the rank-r product formed in fp32 on the tensor cores:
    # besides the one bf16 rounding it may differ from the exact sum by the
    # product's fp32 error, at most about 2^-20 of sum_j |s B_nj A_jk| for
    # these ranks, which can be several bf16 steps where W_hat and s B A
    # nearly cancel
    gv = obf16.bf16_bits_to_f32(got).astype(np.float64)
    rv = obf16.bf16_bits_to_f32(ref).astype(np.float64)
    s_ = float(np.float32(alpha) / np.float32(r))
    mag = s_ * (np.abs(_np(b).astype(np.float64)) @ np.abs(_np(a).astype(np.float64)))
    step = np.spacing(np.abs(rv).astype(np.float32)).astype(np.float64) * 2.0 ** 16   # one bf16 step of ref
    assert np.all(np.abs(gv - rv) <= step + 2.0 ** -20 * mag)
    assert np.mean(got != ref) < 1e-3
