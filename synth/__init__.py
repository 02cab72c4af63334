"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle legs.

Holds none of the method's arithmetic: it only draws random tensors. Every
tensor is drawn in float32 on the CPU with ``torch.Generator('cpu')`` and
rounded to bfloat16 (round-to-nearest-even, torch's cast), so the same seed
gives the same bits on every machine.

Distributions (one derived seed per tensor, base seed 0 by default):
    W  ~ N(0, 0.02)                seed + 0
    x  ~ N(0, 1)                   seed + 1
    A  ~ U(-1/sqrt(K), 1/sqrt(K))  seed + 2
    B  ~ N(0, 0.01)                seed + 3
    dY ~ N(0, 1)                   seed + 4
    outlier mask U(0,1) < 0.001    seed + 5   (entries of W scaled x20
                                               before the bf16 cast)

The whole 7B-shaped stack (6.5 billion weights) is the exception: its
tensors are drawn on the GPU with a device generator (stack_linear,
stack_activations), deterministic for a given device type.
"""

import math
from dataclasses import dataclass

import torch

SEED_W, SEED_X, SEED_A, SEED_B, SEED_DY, SEED_MASK = 0, 1, 2, 3, 4, 5


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weight(n, k, seed=0, outliers=False, std=0.02):
    """Frozen base weight W [n, k] bf16, optionally with 0.1% entries x20."""
    w = torch.randn((n, k), generator=_gen(seed + SEED_W), dtype=torch.float32) * std
    if outliers:
        mask = torch.rand((n, k), generator=_gen(seed + SEED_MASK), dtype=torch.float32) < 0.001
        w = torch.where(mask, w * 20.0, w)
    return w.to(torch.bfloat16)


def tokens(m, k, seed=0):
    """Input activations x [m, k] bf16 ~ N(0, 1)."""
    return torch.randn((m, k), generator=_gen(seed + SEED_X), dtype=torch.float32).to(torch.bfloat16)


def lora_a(r, k, seed=0):
    """LoRA down projection A [r, k] bf16 ~ U(+-1/sqrt(k))."""
    bound = 1.0 / math.sqrt(k)
    a = (torch.rand((r, k), generator=_gen(seed + SEED_A), dtype=torch.float32) * 2.0 - 1.0) * bound
    return a.to(torch.bfloat16)


def lora_b(n, r, seed=0, std=0.01):
    """LoRA up projection B [n, r] bf16 ~ N(0, 0.01)."""
    return (torch.randn((n, r), generator=_gen(seed + SEED_B), dtype=torch.float32) * std).to(torch.bfloat16)


def grad_out(m, n, seed=0):
    """Upstream gradient dY [m, n] bf16 ~ N(0, 1)."""
    return torch.randn((m, n), generator=_gen(seed + SEED_DY), dtype=torch.float32).to(torch.bfloat16)


@dataclass(frozen=True)
class Problem:
    """One quantized-linear workload: W [n, k], x [m, k], LoRA rank r, alpha."""
    name: str
    n: int
    k: int
    m: int
    r: int
    alpha: float
    outliers: bool = False
    backward: bool = True

    @property
    def scale(self):
        return self.alpha / self.r


# The workloads, by what they are.
TINY = Problem("tiny-512x512-m16-r8", 512, 512, 16, 8, 16.0)
DECODE = Problem("decode-gemv-4096x4096-m1-r64", 4096, 4096, 1, 64, 16.0, backward=False)
MLP7B = Problem("7b-mlp-11008x4096-m4096-r64", 11008, 4096, 4096, 64, 16.0)
GATE65B = Problem("65b-gate-up-22016x8192-m4096-r64-outliers", 22016, 8192, 4096, 64, 16.0, outliers=True)
DOWN65B = Problem("65b-down-8192x22016-m4096-r64-outliers", 8192, 22016, 4096, 64, 16.0, outliers=True)

# The 7B-shaped stack: per layer q, k, v, o (4096x4096), gate, up (11008x4096), down (4096x11008).
STACK7B_LAYER = (
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008),
)
STACK7B_LAYERS = 32
STACK7B_SEED = 10_000          # + 16 * layer + projection index
STACK7B_ACT_SEED = 20_000      # activations and upstream gradients of the stack


def stack_linear(layer, idx, r=64, device="cuda"):
    """W [n, k], A [r, k], B [n, r] (bf16, on `device`) of projection `idx`
    of `layer` in the 7B-shaped stack, drawn on the device from one
    generator seeded STACK7B_SEED + 16 * layer + idx, in the order W, A, B:
    W ~ N(0, 0.02), A ~ U(+-1/sqrt(k)), B ~ N(0, 0.01). Generated on the GPU
    because the whole stack holds 6.5 billion weights."""
    _, n, k = STACK7B_LAYER[idx]
    gen = torch.Generator(device=device)
    gen.manual_seed(STACK7B_SEED + 16 * layer + idx)
    w = (torch.randn((n, k), generator=gen, device=device) * 0.02).to(torch.bfloat16)
    a = (torch.rand((r, k), generator=gen, device=device) * 2 - 1).mul_(k ** -0.5).to(torch.bfloat16)
    b = (torch.randn((n, r), generator=gen, device=device) * 0.01).to(torch.bfloat16)
    return w, a, b


def stack_activations(m=4096, device="cuda"):
    """Inputs x [m, k] for k in (4096, 11008) and upstream gradients dY [m, n]
    for n in (4096, 11008) of the stack's linears (bf16, N(0, 1)), drawn on
    the device from one generator seeded STACK7B_ACT_SEED."""
    gen = torch.Generator(device=device)
    gen.manual_seed(STACK7B_ACT_SEED)
    xs = {k: torch.randn((m, k), generator=gen, device=device).to(torch.bfloat16) for k in (4096, 11008)}
    dys = {n: torch.randn((m, n), generator=gen, device=device).to(torch.bfloat16) for n in (4096, 11008)}
    return xs, dys


def make(p: Problem, seed=0):
    """All input tensors of a problem (CPU, bf16)."""
    out = {
        "w": weight(p.n, p.k, seed, p.outliers),
        "x": tokens(p.m, p.k, seed),
        "a": lora_a(p.r, p.k, seed),
        "b": lora_b(p.n, p.r, seed),
    }
    if p.backward:
        out["dy"] = grad_out(p.m, p.n, seed)
    return out
