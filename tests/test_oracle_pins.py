"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test names the fact it checks: a number the pages print (fixtures under
tests/golden/), a closed form, an identity of the construction, brute force
on tiny inputs, or finite differences. A plausible slip in the oracle (a
dropped term, a wrong sign, a transposed operand, an off-by-one in a group
or nibble) fails at least one of them.
"""

import json
import math
import os
from statistics import NormalDist

import numpy as np
import pytest
import torch

import synth
from oracle import bf16, brute, linear, nf4, optim

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _w(n, k, seed=0, outliers=False):
    return synth.weight(n, k, seed=seed, outliers=outliers).float().numpy()


# --------------------------------------------------------------------------- bf16

def test_bf16_rounding_matches_torch_cast():
    # library routine: torch's float32 -> bfloat16 cast is round-to-nearest-even
    g = torch.Generator().manual_seed(11)
    v = torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 8)
    ours = bf16.round_to_bf16(v.numpy())
    ref = v.to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


# --------------------------------------------------------------------------- codebook

def test_codebook_shape_endpoints_zero():
    c = nf4.codebook()
    assert c.dtype == np.float32 and c.shape == (16,)
    assert c[0] == -1.0 and c[15] == 1.0          # normalised to [-1, 1]
    assert c[7] == 0.0                            # the exact zero
    assert np.all(np.diff(c.astype(np.float64)) > 0)
    assert int(np.sum(c < 0)) == 7 and int(np.sum(c > 0)) == 8


def test_codebook_levels_are_normal_quantiles():
    # Each level times Phi^-1(delta) must sit at its quantile point; checked with
    # math.erf, not with the inverse CDF the oracle uses.
    c = nf4.codebook_f64()
    delta = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))
    z = NormalDist().inv_cdf(delta)
    assert abs(nf4.normal_cdf(z) - delta) < 1e-13
    pos = sorted(delta + j * (0.5 - delta) / 8 for j in range(8))
    neg = sorted(delta + j * (0.5 - delta) / 7 for j in range(7))
    for i, p in enumerate(pos):           # c[8..15] ascending <-> p ascending
        assert abs(nf4.normal_cdf(c[8 + i] * z) - p) < 1e-12
    for i, p in enumerate(neg):           # c[6], c[5], ... c[0]: more negative as p grows
        assert abs(nf4.normal_cdf(-c[6 - i] * z) - p) < 1e-12


def test_codebook_dense_near_zero():
    # levels are denser near zero than at the tails (normal quantiles)
    gaps = np.diff(nf4.codebook_f64())
    assert gaps[7] < gaps[14] and gaps[6] < gaps[0]
    assert np.all(np.diff(gaps[7:]) > 0)     # positive side: gaps grow outward
    assert np.all(np.diff(gaps[:7]) < 0)     # negative side: gaps shrink toward 0


def test_midpoints_between_levels():
    c = nf4.codebook().astype(np.float64)
    m = nf4.midpoints().astype(np.float64)
    assert m.shape == (15,)
    assert np.all(c[:-1] < m) and np.all(m < c[1:])
    assert np.all(np.abs(m - (c[:-1] + c[1:]) / 2) <= np.spacing(np.float32(1.0)))


def test_midpoints_are_float32_of_the_exact_mean():
    # reading 2: m_j is the float32 nearest (ties to even) to the exact real
    # mean of two adjacent float32 levels; checked bit for bit against exact
    # rational arithmetic, so a mean summed in float32 or rounded another way
    # fails wherever it lands on a different float32
    from fractions import Fraction
    c = [float(v) for v in nf4.codebook()]
    m = nf4.midpoints()
    for j in range(15):
        want = np.float32(brute.f32_round((Fraction(c[j]) + Fraction(c[j + 1])) / 2))
        assert m[j].view(np.uint32) == want.view(np.uint32), j


def test_encode_tie_goes_to_the_lower_level():
    # reading 2: a quotient exactly on m_j takes index j (the lower level),
    # one float32 above it takes j + 1, one below it j. With a scale of 1
    # the quotient fl32(w / 1) is w itself, so w = m_j is an exact tie.
    from fractions import Fraction
    c = [float(v) for v in nf4.codebook()]
    for j in range(15):
        mj = np.float32(brute.f32_round((Fraction(c[j]) + Fraction(c[j + 1])) / 2))
        row = np.array([mj, np.nextafter(mj, np.float32(2)), np.nextafter(mj, np.float32(-2))], np.float32)
        w = np.zeros((1, 64), np.float32)
        w[0, :3] = row
        q = nf4.encode(w, np.array([1.0], np.float32))[0, :3]
        assert q.tolist() == [j, j + 1, j], j


def test_no_bf16_quotient_comes_near_a_midpoint():
    # For bf16 weights the tie rule is never exercised: over every bf16
    # scale s in [1, 2) and every bf16 w with 0 < w <= s (the quotient is
    # invariant under powers of two for normal values, and a subnormal has
    # fewer significant bits, so this covers every finite pair) the float32
    # quotient stays at least 2 float32 steps away from every midpoint
    # (18 at the closest). So the encoder's decision for bf16 inputs equals
    # the literal nearest level wherever the two midpoints readings differ by
    # less than that, which the brute-force pin below relies on.
    bits = np.arange(0x0080, 0x7F80, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    s_all = vals[(vals >= 1.0) & (vals < 2.0)]
    w_all = vals[(vals > 0) & (vals <= 2.0)]
    mids = np.abs(nf4.midpoints()).view(np.int32).astype(np.int64)
    closest = np.iinfo(np.int64).max
    for s in s_all:
        qv = (w_all[w_all <= s] / s).astype(np.float32).view(np.int32).astype(np.int64)
        qv.sort()
        pos = np.searchsorted(qv, mids)
        for j, p in enumerate(pos):
            for i in (p - 1, p):
                if 0 <= i < qv.size:
                    closest = min(closest, abs(int(qv[i]) - int(mids[j])))
    assert closest >= 2


# --------------------------------------------------------------------------- storage budget

def test_bit_budget_matches_pages():
    g = _golden("bit_budget.json")
    n, k = 8192, 22016
    assert nf4.bits_per_param(n, k, dq=False) == g["bits_nf4_fp32_block_scale"]
    b = nf4.bits_per_param(n, k, dq=True)
    assert round(b, g["bits_nf4_double_quant_decimals"]) == g["bits_nf4_double_quant"]
    # closed form 4 + 8/64 + 32/(64*256) for whole groups
    assert b == pytest.approx(4 + 8 / 64 + 32 / (64 * 256), abs=1e-12)
    saving_gb = (4.5 - b) / 8 * g["params_65b"] / 1e9
    assert abs(saving_gb - g["dq_saving_65b_gb_approx"]) < g["dq_saving_65b_gb_tolerance"]


def test_lora_param_count_matches_pages():
    g = _golden("lora_param_count.json")
    d, r = g["d"], g["r"]
    a = synth.lora_a(r, d)
    b = synth.lora_b(d, r)
    assert a.numel() + b.numel() == g["low_rank_numbers"]
    assert round(d * d / 1e6, 1) == g["full_numbers_millions_approx"]


# --------------------------------------------------------------------------- quantizer

@pytest.mark.parametrize("seed,outliers", [(0, False), (1, True), (2, False)])
def test_quantizer_matches_brute_force(seed, outliers):
    n, k = 6, 192                       # 18 blocks -> one partial DQ group
    w = _w(n, k, seed, outliers)
    w[2, 64:128] = 0.0                  # a zero block
    w[4, :64] = -w[4, :64]
    out = nf4.quantize(w)
    levels = [float(v) for v in nf4.codebook()]
    q_rows, scales = brute.quantize_rows(w.tolist(), levels)
    q_b = np.array(q_rows, dtype=np.uint8)
    # the literal argmin over all 16 levels agrees everywhere: no bf16
    # quotient comes within 2 float32 steps of a midpoint (pinned above)
    assert np.array_equal(out["q"], q_b)
    assert np.array_equal(np.array(scales, dtype=np.float32), out["absmax"])
    packed_b = np.array([brute.pack_row(r) for r in q_rows], dtype=np.uint8)
    packed_o = nf4.pack(q_b)
    assert np.array_equal(packed_b, packed_o)
    q2_b, smax_b = brute.double_quantize(scales)
    assert np.array_equal(np.array(q2_b, dtype=np.uint8), out["q2"])
    assert np.array_equal(np.array(smax_b, dtype=np.float32), out["smax"])


def test_zero_block_and_zero_group():
    w = np.zeros((2, 128), dtype=np.float32)
    out = nf4.quantize(w)
    assert np.all(out["q"] == nf4.ZERO_CODE)
    assert np.all(out["codes"] == 0x77)
    assert np.all(out["q2"] == 0) and np.all(out["smax"] == 0)
    assert np.all(nf4.dequantize(out["codes"], out["q2"], out["smax"]) == 0)


def test_round_trip_of_levels():
    # w = c_j * s (bf16) in a block whose max is s  ->  index j exactly
    c = nf4.codebook()
    s = np.float32(0.0371)
    levels = bf16.round_to_bf16((c * s).astype(np.float32))
    row = np.tile(levels, 4)[None, :]             # 64 values, contains +-s
    s_b = bf16.round_to_bf16(np.array([s], np.float32))[0]
    row[0, 15] = s_b
    row[0, 0] = -s_b
    q = nf4.quantize(row)["q"][0]
    assert np.array_equal(q, np.tile(np.arange(16, dtype=np.uint8), 4))


def test_encode_error_within_half_gap():
    w = _w(64, 512, seed=3, outliers=True)
    out = nf4.quantize(w)
    s = np.repeat(out["absmax"], 64).reshape(w.shape)
    x = (w / s).astype(np.float32).astype(np.float64)
    c = nf4.codebook().astype(np.float64)
    err = np.abs(x - c[out["q"]])
    assert err.max() <= nf4.max_level_gap() / 2 + 1e-7


def test_pack_unpack_round_trip_and_nibble_order():
    g = np.random.default_rng(0)
    q = g.integers(0, 16, size=(5, 64), dtype=np.uint8)
    assert np.array_equal(nf4.unpack(nf4.pack(q)), q)
    one = np.zeros((1, 64), dtype=np.uint8)
    one[0, 0], one[0, 1] = 0xA, 0x3
    assert nf4.pack(one)[0, 0] == 0xA3       # element 0 -> high nibble


def test_outlier_touches_only_its_block_and_group():
    w = _w(8, 4096, seed=4)                  # 512 blocks -> 2 groups of 256
    base = nf4.quantize(w)
    w2 = w.copy()
    w2[3, 1000] = np.float32(bf16.round_to_bf16(np.array([w[3, 1000] * 20 + 0.5], np.float32))[0])
    pert = nf4.quantize(w2)
    blk = (3 * 4096 + 1000) // 64
    grp = blk // 256
    q_diff = np.nonzero(np.any(base["q"].reshape(-1, 64) != pert["q"].reshape(-1, 64), axis=1))[0]
    assert set(q_diff.tolist()) <= {blk}
    q2_diff = np.nonzero(base["q2"] != pert["q2"])[0]
    assert set((q2_diff // 256).tolist()) <= {grp}
    sm_diff = np.nonzero(base["smax"] != pert["smax"])[0]
    assert set(sm_diff.tolist()) <= {grp}


# --------------------------------------------------------------------------- double quantization

def test_double_quant_error_bound():
    w = _w(256, 4096, seed=5, outliers=True)
    out = nf4.quantize(w)
    s = out["absmax"].astype(np.float64)
    s_hat = nf4.restored_scale(out["q2"], out["smax"]).astype(np.float64)
    smax = out["smax"].astype(np.float64)[np.arange(s.size) // 256]
    err = np.abs(s - s_hat)
    assert np.all(err <= smax / 256 * (1 + 1e-6))              # the printed bound
    top = out["q2"] == 255
    assert np.all(err[~top] <= smax[~top] / 512 * (1 + 1e-6))  # every other code: half a step
    # each group's largest block lands on the top code, restored to 255/256 of s_max
    for g in range(out["smax"].size):
        sl = slice(256 * g, 256 * (g + 1))
        i = np.argmax(s[sl])
        assert out["q2"][sl][i] == 255
    assert nf4.n_groups(out["absmax"].size) == out["smax"].size


def test_double_quant_extra_error_is_tiny():
    # extra error from re-quantizing the scales stays below 0.01 % of the
    # weight norm (relative Frobenius error, DQ minus plain fp32 scales)
    w = _w(512, 4096, seed=6)
    out = nf4.quantize(w)
    c = nf4.codebook()
    plain = (c[out["q"]].reshape(-1, 64) * out["absmax"].reshape(-1, 1)).reshape(w.shape)
    dq = nf4.dequantize(out["codes"], out["q2"], out["smax"])
    e_plain = linear.rel_fro(plain, w)
    e_dq = linear.rel_fro(dq, w)
    assert e_dq - e_plain < 1e-4
    assert 0.0 < e_plain < 0.2


def test_dequant_error_bound():
    w = _w(128, 2048, seed=7, outliers=True)
    out = nf4.quantize(w)
    w_hat = nf4.dequantize(out["codes"], out["q2"], out["smax"]).astype(np.float64)
    s = np.repeat(out["absmax"], 64).reshape(w.shape).astype(np.float64)
    smax = np.repeat(out["smax"].astype(np.float64)[np.arange(out["absmax"].size) // 256], 64).reshape(w.shape)
    bound = s * nf4.max_level_gap() / 2 + smax / 256 + np.abs(w_hat) * 2.0 ** -8
    assert np.all(np.abs(w.astype(np.float64) - w_hat) <= bound * (1 + 1e-6))


def test_dequant_is_bf16_of_level_times_scale():
    # closed form per element, written with Python floats and struct-free rounding
    w = _w(4, 256, seed=8)
    out = nf4.quantize(w)
    got = nf4.dequantize(out["codes"], out["q2"], out["smax"])
    c = [float(v) for v in nf4.codebook()]
    for n in range(4):
        for k in range(0, 256, 7):
            b = (n * 256 + k) // 64
            s_hat = brute.f32_round(float(out["q2"][b]) * float(out["smax"][b // 256])) / 256.0
            v = brute.f32_round(c[out["q"][n, k]] * s_hat)
            ref = float(bf16.round_to_bf16(np.array([v], np.float32))[0])
            assert got[n, k] == ref


# --------------------------------------------------------------------------- linear

def _small(m=3, n=5, k=64, r=4, seed=9):
    g = np.random.default_rng(seed)
    rb = lambda *s: bf16.round_to_bf16(g.standard_normal(s).astype(np.float32))
    return rb(m, k), rb(n, k), rb(r, k), rb(n, r), rb(m, n)


def test_forward_matches_brute_loops():
    x, w, a, b, _ = _small()
    s = 16.0 / 4
    y, u = linear.forward(x, w, a, b, s)
    yb = np.array(brute.forward(x.tolist(), w.tolist(), a.tolist(), b.tolist(), s))
    assert np.allclose(y, yb, rtol=1e-12, atol=1e-12)
    assert np.allclose(u, np.array(brute.matmul_nt(x.tolist(), a.tolist())), rtol=1e-12, atol=1e-12)


def test_forward_b_zero_is_base_model():
    x, w, a, b, _ = _small()
    y, _ = linear.forward(x, w, a, np.zeros_like(b), 2.0)
    assert np.array_equal(y, x.astype(np.float64) @ w.astype(np.float64).T)


def test_forward_w_zero_is_lora_only():
    x, w, a, b, _ = _small()
    y, _ = linear.forward(x, np.zeros_like(w), a, b, 0.5)
    ref = 0.5 * np.array(brute.matmul_nt(np.array(brute.matmul_nt(x.tolist(), a.tolist())).tolist(), b.tolist()))
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_backward_matches_finite_differences():
    # L = <dY, y> is linear in each of x, A, B separately, so central
    # differences are exact up to rounding (Proposition 1: the gradients of
    # the LoRA path are the true gradients; W gets none).
    p = synth.TINY
    t = synth.make(p, seed=0)
    w = nf4.dequantize(**{k: v for k, v in nf4.quantize(t["w"].float().numpy()).items() if k in ("codes", "q2", "smax")})
    x, a, b, dy = (t[k].float().numpy().astype(np.float64) for k in ("x", "a", "b", "dy"))
    x, a, b, dy = x[:4, :128], a[:, :128], b[:64], dy[:4, :64]
    w = w[:64, :128].astype(np.float64)
    s = p.scale
    dx, da, db = linear.backward(x, dy, w, a, b, s)
    h = 1e-3
    g = np.random.default_rng(1)

    def fd(arr, idx):
        plus, minus = arr.copy(), arr.copy()
        plus[idx] += h
        minus[idx] -= h
        return plus, minus

    for name, arr, grad in (("x", x, dx), ("a", a, da), ("b", b, db)):
        for _ in range(12):
            idx = tuple(int(g.integers(0, d)) for d in arr.shape)
            p_, m_ = fd(arr, idx)
            args = {"x": x, "a": a, "b": b}
            args_p = dict(args, **{name: p_})
            args_m = dict(args, **{name: m_})
            lp = linear.loss(args_p["x"], dy, w, args_p["a"], args_p["b"], s)
            lm = linear.loss(args_m["x"], dy, w, args_m["a"], args_m["b"], s)
            num = (lp - lm) / (2 * h)
            assert abs(num - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx])), (name, idx)


def test_backward_has_no_weight_gradient_and_b_zero():
    # B = 0 at the start: dA vanishes, dB does not (B receives gradient in step one)
    x, w, a, b, dy = _small()
    dx, da, db = linear.backward(x, dy, w, a, np.zeros_like(b), 4.0)
    assert np.all(da == 0)
    assert np.any(db != 0)
    assert np.array_equal(dx, dy.astype(np.float64) @ w.astype(np.float64))
    assert len(linear.backward(x, dy, w, a, b, 4.0)) == 3     # dX, dA, dB only


def test_rel_fro():
    a = np.array([3.0, 4.0])
    assert linear.rel_fro(a * 1.01, a) == pytest.approx(0.01)


# --------------------------------------------------------------------------- merge for export

def test_merge_matches_exact_rational_loops():
    # exact rational sum, one rounding to bf16, against the vectorised oracle
    for s in (4.0, 16.0 / 12.0, -0.375):
        x, w, a, b, _ = _small(n=6, k=64, r=5, seed=21)
        got = linear.merge_bits(w, a, b, s)
        ref = np.array(brute.merge(w.tolist(), a.tolist(), b.tolist(), s), dtype=np.uint16)
        assert np.array_equal(got, ref)


def test_merge_rounding_at_bf16_ties():
    # W_hat + s B A placed exactly on, and one float64 step either side of,
    # bf16 rounding ties: the oracle must follow round-to-nearest-even there
    w = np.array([[1.0, 1.0, 1.0, 1.0]], dtype=np.float32)
    half_ulp = 2.0 ** -8                  # bf16 spacing at 1.0 is 2^-7
    a = np.array([[half_ulp, 3 * half_ulp, half_ulp + 2.0 ** -40, half_ulp - 2.0 ** -40]])
    b = np.array([[1.0]])
    got = linear.merge_bits(w, a, b, 1.0)
    ref = np.array(brute.merge(w.tolist(), a.tolist(), b.tolist(), 1.0), dtype=np.uint16)
    assert np.array_equal(got, ref)
    # 1 + 2^-8 ties to 1.0 (even); 1 + 3*2^-8 ties to 1 + 2^-6 (even); off-tie values go to the nearer side
    assert got[0, 0] == 0x3F80 and got[0, 1] == 0x3F82 and got[0, 2] == 0x3F81 and got[0, 3] == 0x3F80


def test_merge_with_b_zero_is_restored_weight():
    w = synth.weight(64, 128, seed=4).float().numpy()
    o = nf4.quantize(w)
    w_hat = nf4.dequantize(o["codes"], o["q2"], o["smax"])
    a = synth.lora_a(8, 128).float().numpy()
    got = linear.merge_bits(w_hat, a, np.zeros((64, 8)), 2.0)
    assert np.array_equal(got, nf4.dequantize_bits(o["codes"], o["q2"], o["smax"]))


def test_merged_forward_matches_adapter_forward():
    # the merged model's forward equals the base + adapter forward up to the
    # bf16 rounding of the merged weight
    t = synth.make(synth.TINY)
    o = nf4.quantize(t["w"].float().numpy())
    w_hat = nf4.dequantize(o["codes"], o["q2"], o["smax"])
    x, a, b = (t[k_].float().numpy() for k_ in ("x", "a", "b"))
    b = b * 50.0                          # make the adapter term visible next to W_hat
    s = synth.TINY.scale
    merged = bf16.bf16_bits_to_f32(linear.merge_bits(w_hat, a, b, s))
    y_ref, _ = linear.forward(x, w_hat, a, b, s)
    y_m = x.astype(np.float64) @ merged.astype(np.float64).T
    assert linear.rel_fro(y_m, y_ref) <= 2.0 ** -8
    assert linear.rel_fro(y_m, x.astype(np.float64) @ w_hat.astype(np.float64).T) > 1e-2


# --------------------------------------------------------------------------- AdamW for the adapters

def test_adamw_first_step_closed_form():
    # t = 1, wd = 0: m_hat = g and v_hat = g^2, so the step is lr * g / (|g| + eps)
    g = np.array([0.5, -2.0, 1e-3, 0.0, -7.25])
    p0 = np.array([1.0, -1.0, 0.5, 0.25, 3.0])
    p1, m1, v1 = optim.adamw_step(p0, g, np.zeros(5), np.zeros(5), 1, 1e-3, 0.9, 0.999, 1e-8, 0.0)
    assert np.allclose(p1, p0 - 1e-3 * g / (np.abs(g) + 1e-8), rtol=1e-14, atol=1e-15)
    assert np.allclose(m1, 0.1 * g) and np.allclose(v1, 0.001 * g * g)


def test_adamw_matches_torch_adamw():
    # the update rule equals the library's AdamW (float64) over several steps
    rng = np.random.default_rng(3)
    p = rng.standard_normal(300)
    m = np.zeros(300)
    v = np.zeros(300)
    tp = torch.tensor(p.copy(), dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=2e-3, betas=(0.9, 0.995), eps=1e-7, weight_decay=0.05)
    for t in range(1, 6):
        g = rng.standard_normal(300)
        p, m, v = optim.adamw_step(p, g, m, v, t, 2e-3, 0.9, 0.995, 1e-7, 0.05)
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
    assert np.allclose(p, tp.detach().numpy(), rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------------------- format without double quantization

def test_no_dq_restore_matches_brute_force_and_bound():
    # 4.5-bit format: the block scale is stored as fp32 and used as is
    w = synth.weight(6, 128, seed=31, outliers=True).float().numpy()
    o = nf4.quantize(w)
    got = nf4.dequantize_no_dq(o["codes"], o["absmax"])
    levels = [float(x) for x in nf4.codebook()]
    for i in range(6):
        for j in range(128):
            b = (i * 128 + j) // 64
            expect = bf16.round_to_bf16(np.float32(levels[o["q"][i, j]]) * np.float32(o["absmax"][b]))
            assert got[i, j] == expect
    # error within half the largest level gap of the block scale, plus bf16 rounding
    s_b = np.repeat(o["absmax"].reshape(6, 2), 64, axis=1)
    assert np.all(np.abs(w - got) <= s_b * nf4.max_level_gap() / 2 + np.abs(got) * 2.0 ** -8 + 1e-30)


# --------------------------------------------------------------------------- scale-code variants
# The 255-step unsigned grid and the signed mid-range code, both readings of
# the same double-quantization paragraph (8-bit codes of the block scales,
# 32-bit constants per group, error bounded by the grid step).

def _scales(n, seed, spread=1.0):
    g = np.random.default_rng(seed)
    s = np.abs(g.normal(0.05, 0.01 * spread, size=n)).astype(np.float32)
    return bf16.round_to_bf16(s)


@pytest.mark.parametrize("code", ["u8_255", "s8_mid"])
@pytest.mark.parametrize("seed", [0, 1])
def test_scale_codes_match_brute_force(code, seed):
    # 600 scales: two full groups and a short one, with a zero scale, a
    # repeated maximum and an outlier
    s = _scales(600, seed)
    s[5] = 0.0
    s[300] = s[301] = np.float32(0.5)
    s[599] = np.float32(3.0)
    q2, gd = nf4.double_quantize_code(s, code)
    sh = nf4.restored_scale_code(q2, gd, code)
    if code == "u8_255":
        q_b, smax_b, sh_b = brute.double_quantize_u8_255([float(v) for v in s])
        assert np.array_equal(q2.astype(np.int64), np.array(q_b))
        assert np.array_equal(gd, np.array(smax_b, np.float32))
    else:
        q_b, gd_b, sh_b = brute.double_quantize_s8_mid([float(v) for v in s])
        assert np.array_equal(q2.view(np.int8).astype(np.int64), np.array(q_b))
        assert np.array_equal(gd, np.array(gd_b, np.float32))
    assert np.array_equal(sh.view(np.uint32), np.array(sh_b, np.float32).view(np.uint32))


def test_scale_code_u8_255_bound_and_top_code():
    # |s - s_hat| <= s_max / 510 up to float32 rounding (the float32 ratio can
    # move a code on a half-step by up to 255 * 2^-23 of a step, and the
    # restore rounds once more: a slack of 2^-20 s_max covers both); the
    # group maximum is exact
    s = _scales(256 * 8, 3, spread=3.0)
    q2, smax = nf4.double_quantize_code(s, "u8_255")
    sh = nf4.restored_scale_code(q2, smax, "u8_255")
    g = np.arange(s.size) // 256
    err = np.abs(s.astype(np.float64) - sh.astype(np.float64))
    assert np.all(err <= smax[g].astype(np.float64) * (1.0 / 510.0 + 2.0 ** -20))
    top = s == smax[g]
    assert np.all(q2[top] == 255) and np.array_equal(sh[top], s[top])
    # and it is never worse than the printed 1/256 grid's bound
    assert err.max() <= smax.max() / 256.0


def test_scale_code_s8_mid_bound_and_centering():
    # |s - s_hat| <= half / 254 up to float32 rounding (half = half the
    # group's spread); the centred code beats the printed grid on N(0, 0.02)
    # weights, whose block scales sit close together
    w = _w(512, 1024, seed=4)
    a = nf4.block_absmax(w)
    q2, gd = nf4.double_quantize_code(a, "s8_mid")
    sh = nf4.restored_scale_code(q2, gd, "s8_mid")
    g = np.arange(a.size) // 256
    half = gd[g, 1].astype(np.float64)
    err = np.abs(a.astype(np.float64) - sh.astype(np.float64))
    assert np.all(err <= half / 254.0 + 2.0 ** -22 * np.abs(a))
    q2u, smax = nf4.double_quantize(a)
    err_u = np.abs(a.astype(np.float64) - nf4.restored_scale(q2u, smax).astype(np.float64))
    # the signed step 2 half / 254 against the printed s_max / 256: with the
    # mean half / s_max of these groups (about 0.3) the error ratio is about 0.6
    ratio = 2.0 * 256.0 / 254.0 * float(np.mean(gd[:, 1] / nf4.group_smax(a)))
    assert np.sqrt(np.mean(err ** 2)) < min(0.75, 1.15 * ratio) * np.sqrt(np.mean(err_u ** 2))
    assert q2.view(np.int8).min() == -127 and q2.view(np.int8).max() == 127


def test_scale_code_special_groups():
    # a group of equal scales (half = 0: every code 0, s_hat = s exactly), an
    # all-zero group, and the 255-grid's zero group
    s = np.concatenate([np.full(256, 0.0625, np.float32), np.zeros(256, np.float32)])
    q2, gd = nf4.double_quantize_code(s, "s8_mid")
    assert np.all(q2 == 0) and np.array_equal(nf4.restored_scale_code(q2, gd, "s8_mid"), s)
    q2, smax = nf4.double_quantize_code(s, "u8_255")
    assert np.all(q2[256:] == 0) and np.all(q2[:256] == 255)
    assert np.array_equal(nf4.restored_scale_code(q2, smax, "u8_255"), s)


def test_scale_code_bit_budgets():
    # 4-bit codes + an 8-bit scale code per 64 weights + the group constants
    # per 256 blocks (16384 weights): one float32 for the unsigned codes, two
    # for the signed one
    n, k = 1024, 4096
    assert nf4.bits_per_param_code(n, k, "u8_255") == pytest.approx(4 + 8 / 64 + 32 / 16384, abs=0)
    assert nf4.bits_per_param_code(n, k, "u8_256") == nf4.bits_per_param(n, k)
    assert nf4.bits_per_param_code(n, k, "s8_mid") == pytest.approx(4 + 8 / 64 + 64 / 16384, abs=0)
    assert round(nf4.bits_per_param_code(n, k, "u8_255"), 2) == _golden("bit_budget.json")["bits_nf4_double_quant"]


@pytest.mark.parametrize("code", ["u8_255", "s8_mid"])
def test_restore_with_scale_code_is_bf16_of_level_times_scale(code):
    w = _w(8, 640, seed=7, outliers=True)
    o = nf4.quantize_code(w, code)
    bits = nf4.dequantize_bits_code(o["codes"], o["q2"], o["gdata"], code)
    sh = nf4.restored_scale_code(o["q2"], o["gdata"], code)
    c = [float(v) for v in nf4.codebook()]
    for i in range(0, 8 * 640, 97):
        r, kk = divmod(i, 640)
        q = int(o["q"][r, kk])
        want = brute.bf16_round_bits(brute.Fraction(brute.f32_round(brute.Fraction(c[q]) * brute.Fraction(float(sh[i // 64])))))
        assert int(bits[r, kk]) == want
