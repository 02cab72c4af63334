"""Stream-K schedule of the CTA-pair GEMMs (forward y and backward dX).

When the output tiles do not divide evenly over the CTA pairs, each pair takes
an equal range of (tile, k-tile) work and a tile cut between two pairs is
finished from an fp32 partial passed through the workspace. The cases here
have a prime tile count (149 > any pair count of a 148-SM part, and a
multiple of none) with only 2-4 k-tiles per tile, so most tiles are cut,
often right after their first k-tile; both token-group widths (NH = 1, 2) and
both directions are covered.

* the schedule is forced to stream-K (the automatic rule keeps reductions
  this short data-parallel);
* outputs against the fp64 oracle (relative Frobenius error <= 5e-3), with
  the full workspace (stream-K) and, for the forward, with the least
  workspace the call accepts (which falls back to data-parallel);
* x = I and dY = I with B = 0: every output element is a single product, so
  the GEMMs with cut tiles must still reproduce W_hat bit for bit -- a partial
  added to the wrong rows, columns or tile breaks this.
"""

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


@pytest.fixture(autouse=True)
def _status_clear(q):
    yield
    st, bits = q.qlora_device_status()
    assert st == 0 and bits == 0, f"device status {st} bits {bits:#x}"


@pytest.fixture(autouse=True)
def _stream_k(q):
    # these reductions are short (1-8 k-tiles), where the automatic rule stays data-parallel
    q.qlora_set_gemm_schedule(q.SCHED_STREAM_K)
    yield
    q.qlora_set_gemm_schedule(q.SCHED_AUTO)


def _np(t):
    return t.detach().cpu().float().numpy()


def _bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def _ws(q, m, n, k, r, full=True):
    nbytes = q.qlora_workspace_bytes(m, n, k, r) if full else q.qlora_fwd_workspace_bytes(m, n, k, r)
    return torch.empty(nbytes + 256, dtype=torch.uint8, device="cuda")


FWD_CASES = [
    # n, k, m, r     forward tiles = ceil(n / 256) * ceil(m / (256 NH)), NH = 2 if m > 256 else 1
    (38104, 128, 512, 16),    # 149 x 1 tiles of 512 tokens, 2 + 1 k-tiles, ragged last feature tile
    (38144, 64, 200, 8),      # NH = 1: 149 tiles of 256 tokens (200 valid), 1 + 1 k-tiles
    (2560, 128, 4096, 64),    # 10 x 8 tiles: cut tiles in every token group
]


@pytest.mark.parametrize("n,k,m,r", FWD_CASES)
@pytest.mark.parametrize("full_ws", [True, False], ids=["stream-k", "data-parallel"])
def test_forward_cut_tiles(q, n, k, m, r, full_ws):
    alpha = 16.0
    t = {"w": synth.weight(n, k, seed=n + m), "x": synth.tokens(m, k, seed=m), "a": synth.lora_a(r, k, seed=r),
         "b": synth.lora_b(n, r, seed=k)}
    o = nf4.quantize(t["w"].float().numpy())
    w_hat = nf4.dequantize(o["codes"], o["q2"], o["smax"])
    y_ref, _ = linear.forward(_np(t["x"]), w_hat, _np(t["a"]), _np(t["b"]), alpha / r)
    qw = q.qlora_quantize_nf4(t["w"].cuda())
    y, _ = q.qlora_linear_fwd_ex(qw, t["x"].cuda(), t["a"].cuda(), t["b"].cuda(), alpha, path=q.FWD_GEMM,
                                 ws=_ws(q, m, n, k, r, full_ws))
    torch.cuda.synchronize()
    assert linear.rel_fro(_np(y), y_ref) <= TOL


BWD_CASES = [
    # n, k, m, r     dX tiles = ceil(k / 256) * ceil(m / (256 NH))
    (192, 38144, 300, 16),    # 149 x 1 tiles, reduction over d_out = 3 + 1 k-tiles, ragged tokens
    (128, 38144, 160, 8),     # NH = 1: 149 tiles, 2 + 1 k-tiles
]


@pytest.mark.parametrize("n,k,m,r", BWD_CASES)
def test_backward_cut_tiles(q, n, k, m, r):
    alpha = 16.0
    s = alpha / r
    t = {"w": synth.weight(n, k, seed=k + m), "x": synth.tokens(m, k, seed=n), "a": synth.lora_a(r, k, seed=m),
         "b": synth.lora_b(n, r, seed=r), "dy": synth.grad_out(m, n, seed=k)}
    o = nf4.quantize(t["w"].float().numpy())
    w_hat = nf4.dequantize(o["codes"], o["q2"], o["smax"])
    dx_ref, da_ref, db_ref = linear.backward(_np(t["x"]), _np(t["dy"]), w_hat, _np(t["a"]), _np(t["b"]), s)
    qw = q.qlora_quantize_nf4(t["w"].cuda())
    x, a, b, dy = (t[k_].cuda() for k_ in ("x", "a", "b", "dy"))
    ws = _ws(q, m, n, k, r)
    _, u = q.qlora_linear_fwd_ex(qw, x, a, b, alpha, path=q.FWD_GEMM, ws=ws)
    dx, da, db = q.qlora_linear_bwd(qw, x, u, dy, a, b, alpha, ws=ws)
    torch.cuda.synchronize()
    assert linear.rel_fro(_np(dx), dx_ref) <= TOL
    assert linear.rel_fro(_np(da), da_ref) <= TOL
    assert linear.rel_fro(_np(db), db_ref) <= TOL


def test_forward_cut_tiles_restore_w_exactly(q):
    # x = I (512 tokens = K), B = 0: y = W_hat^T bit for bit; 149 x 1 tiles, 8 + 1 k-tiles each
    n, k, r = 38144, 512, 16
    w = synth.weight(n, k, seed=21)
    o = nf4.quantize(w.float().numpy())
    qw = q.qlora_quantize_nf4(w.cuda())
    x = torch.eye(k, dtype=torch.bfloat16)
    a = synth.lora_a(r, k)
    b = torch.zeros((n, r), dtype=torch.bfloat16)
    y, _ = q.qlora_linear_fwd_ex(qw, x.cuda(), a.cuda(), b.cuda(), 16.0, path=q.FWD_GEMM, ws=_ws(q, k, n, k, r))
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y).T, nf4.dequantize_bits(o["codes"], o["q2"], o["smax"]))


def test_backward_cut_tiles_restore_w_exactly(q):
    # dY = I (512 tokens = d_out), B = 0: dX = W_hat bit for bit; 149 x 1 dX tiles, 8 + 1 k-tiles each
    n, k, r = 512, 38144, 16
    w = synth.weight(n, k, seed=22)
    o = nf4.quantize(w.float().numpy())
    qw = q.qlora_quantize_nf4(w.cuda())
    dy = torch.eye(n, dtype=torch.bfloat16)
    x = synth.tokens(n, k)
    a = synth.lora_a(r, k)
    b = torch.zeros((n, r), dtype=torch.bfloat16)
    dx, _, _ = q.qlora_linear_bwd(qw, x.cuda(), None, dy.cuda(), a.cuda(), b.cuda(), 16.0, ws=_ws(q, n, n, k, r))
    torch.cuda.synchronize()
    assert np.array_equal(_bits(dx), nf4.dequantize_bits(o["codes"], o["q2"], o["smax"]))


def test_fwd_bwd_in_cuda_graph_match_direct_calls(q):
    # a forward and a backward call (each a chain of programmatic dependent
    # launches; the stream-K flags zeroed by a memset before the chain)
    # captured in one CUDA graph and replayed with new inputs: bit-identical to
    # direct calls every time, so the flags start at zero on every replay and
    # every kernel of the chain sees its predecessor's results
    n, k, m, r, alpha = 2560, 128, 4096, 64, 16.0
    qw = q.qlora_quantize_nf4(synth.weight(n, k, seed=21).cuda())
    a = synth.lora_a(r, k, seed=22).cuda()
    b = (synth.lora_b(n, r, seed=23).float() * 20).to(torch.bfloat16).cuda()
    x = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    dy = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    u = torch.empty((m, r), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    da = torch.empty((r, k), dtype=torch.float32, device="cuda")
    db = torch.empty((n, r), dtype=torch.float32, device="cuda")
    ws = _ws(q, m, n, k, r)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        q.qlora_linear_fwd(qw, x, a, b, alpha, y=y, u=u, ws=ws, stream=st)
    st.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        q.qlora_linear_fwd(qw, x, a, b, alpha, y=y, u=u, ws=ws, stream=st)
        q.qlora_linear_bwd(qw, x, u, dy, a, b, alpha, dx=dx, da=da, db=db, ws=ws, stream=st)
    for trial in range(3):
        x.copy_(synth.tokens(m, k, seed=300 + trial))
        dy.copy_(synth.grad_out(m, n, seed=400 + trial))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        y2, u2 = q.qlora_linear_fwd(qw, x, a, b, alpha)
        dx2, da2, db2 = q.qlora_linear_bwd(qw, x, u2, dy, a, b, alpha)
        torch.cuda.synchronize()
        assert torch.equal(_bits_t(y), _bits_t(y2)) and torch.equal(_bits_t(u), _bits_t(u2))
        assert torch.equal(_bits_t(dx), _bits_t(dx2))
        assert torch.equal(da, da2) and torch.equal(db, db2)
    del g


def _bits_t(t):
    return t.view(torch.int16)
