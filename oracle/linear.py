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

Every operand is widened to float64 before the products; numpy's matmul is
the only library primitive used.
"""

import numpy as np


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
