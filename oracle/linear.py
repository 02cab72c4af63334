"""Forward and backward of the QLoRA linear in float64 (test infrastructure only).

Shapes (row-major, tokens in rows):
    W_hat [N, K]  restored base weight (d_out x d_in)
    x     [M, K]  input tokens
    A     [r, K]  LoRA down projection
    B     [N, r]  LoRA up projection
    s = alpha / r

Forward, «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나», § "QLoRA의 수식":
h = dequant(W) x + (alpha/r) B A x, written here for token rows:
    y = x W_hat^T + s (x A^T) B^T.

Backward, same page, § "명제 1 · QLoRA Backward Unbiasedness", and "48GB GPU
Fine-Tuning a 65B Model ...", § "QLoRA Puts the Two Methods in Different
Places": the base weight is frozen (no gradient into W); gradients reach x
through the restored W and the LoRA path, and reach A and B:
    dX = dY W_hat + s (dY B) A
    dA = s (dY B)^T x
    dB = s dY^T (x A^T)

Merge for export, "48GB GPU Fine-Tuning a 65B Model ...", § "LoRA Freezes
the Original Weights ..." (after training B A has W's shape and is added to
W) and § "QLoRA Puts the Two Methods in Different Places" (with a 4-bit base
the adapters are added to the restored 16-bit weights, not to the codes):
    W_merged = bf16(W_hat + s B A)     (one rounding, from the exact sum)

Every operand is widened to float64 before the products; numpy's matmul is
the only library primitive used.
"""

import numpy as np

from .bf16 import round_f32_to_bf16_bits


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def forward(x, w_hat, a, b, s):
    """Return (y, u) with u = x A^T (unscaled), both float64."""
    x, w_hat, a, b = _f64(x), _f64(w_hat), _f64(a), _f64(b)
    u = x @ a.T
    y = x @ w_hat.T + float(s) * (u @ b.T)
    return y, u


def backward(x, dy, w_hat, a, b, s):
    """Return (dX, dA, dB) in float64."""
    x, dy, w_hat, a, b = _f64(x), _f64(dy), _f64(w_hat), _f64(a), _f64(b)
    s = float(s)
    v = dy @ b
    dx = dy @ w_hat + s * (v @ a)
    da = s * (v.T @ x)
    db = s * (dy.T @ (x @ a.T))
    return dx, da, db


def loss(x, dy, w_hat, a, b, s):
    """L = <dY, y(x, A, B)>: the scalar whose gradients ``backward`` returns."""
    y, _ = forward(x, w_hat, a, b, s)
    return float(np.sum(_f64(dy) * y))


def rel_fro(got, ref):
    """Relative Frobenius error ||got - ref|| / ||ref||."""
    got, ref = _f64(got), _f64(ref)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def merge_bits(w_hat, a, b, s):
    """Merged weight bf16(W_hat + s B A) as uint16 bit patterns [N, K].

    The sum is formed in float64 and rounded once to bf16 (nearest, ties to
    even): first to float32 by rounding to odd, then to bf16; rounding to odd
    at 24 bits makes the second rounding equal the direct bf16 rounding of
    the float64 value.
    """
    m = _f64(w_hat) + float(s) * (_f64(b) @ _f64(a))
    return round_f32_to_bf16_bits(_round_f64_to_f32_odd(m))


def _round_f64_to_f32_odd(x):
    """float64 -> float32 rounding to odd (keeps a later bf16 rounding exact)."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    back = f.astype(np.float64)
    inexact = back != x
    bits = f.view(np.uint32).copy()
    # an inexact result with an even last bit is moved one step toward x
    fix = inexact & ((bits & 1) == 0)
    toward_up = x > back
    step = np.where(toward_up == (f >= 0), 1, -1).astype(np.int64)
    bits = np.where(fix, (bits.astype(np.int64) + step).astype(np.uint32), bits)
    return bits.view(np.float32)
