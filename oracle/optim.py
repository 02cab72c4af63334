"""AdamW step for the LoRA adapters in float64 (test infrastructure only).

«QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나», § "메모리 회계: 세 겹의 최적화"
(Paged Optimizer paragraph): only the adapters A and B are trained, with
Adam's two states m and v per parameter, and those states may live in CPU
pinned memory. The pages name Adam but print no update rule; the reading
taken is AdamW (decoupled weight decay) with bias correction, in the order:

    m   <- beta1 m + (1 - beta1) g
    v   <- beta2 v + (1 - beta2) g^2
    p   <- p (1 - lr wd)
    p   <- p - (lr / (1 - beta1^t)) m / (sqrt(v) / sqrt(1 - beta2^t) + eps)

with t the 1-based step count.
"""

import math

import numpy as np


def adamw_step(p, g, m, v, t, lr, beta1, beta2, eps, wd):
    """One step; returns new (p, m, v) as float64 arrays."""
    p, g, m, v = (np.asarray(a, dtype=np.float64) for a in (p, g, m, v))
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    bc1 = 1.0 - beta1 ** t
    bc2 = 1.0 - beta2 ** t
    p = p * (1.0 - lr * wd)
    p = p - (lr / bc1) * m / (np.sqrt(v) / math.sqrt(bc2) + eps)
    return p, m, v
