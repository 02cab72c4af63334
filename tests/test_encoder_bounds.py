"""The facts the GPU encoder's fast path relies on (k_quantize_nf4), checked on
the host against the oracle's definitions -- not the kernel itself, which the
GPU parity tests compare bit for bit:

* with r within 2 ulp of 1/s (s a normal bf16 scale below 2^126, |w| <= s),
  |fl32(w * r) - fl32(w / s)| < 3.4e-7, below the 5e-7 guard;
* the 33 cells rint(16 x + 16), each widened by twice the guard, hold at most
  one level midpoint, and every other midpoint lies wholly below or above;
* eight codes packed as two exact float sums (q1 + 16 q0 + 256 q3 + 4096 q2,
  likewise for q4..q7) read back through the 2^23 offset give the stored
  byte order (element 2i in the high nibble of byte i).
"""

import numpy as np

from oracle import bf16 as obf16
from oracle import nf4

GUARD = 5e-7


def _bf16(x):
    return obf16.round_to_bf16(np.asarray(x, dtype=np.float32).ravel())


def test_quotient_error_within_guard():
    rng = np.random.default_rng(17)
    worst = 0.0
    for e in list(range(-126, 126, 7)) + [-126, 125]:
        s = _bf16(np.ldexp(1.0 + rng.random(64), e))
        for sb in s:
            sb = np.float32(sb)
            r0 = np.float32(1.0) / sb
            w = _bf16(rng.uniform(-1.0, 1.0, 256) * np.float64(sb))
            w = w[np.abs(w) <= sb]
            exact = (w / sb).astype(np.float32).astype(np.float64)
            for ulp in (-2, -1, 0, 1, 2):
                r = np.array([r0], dtype=np.float32).view(np.int32) + ulp
                r = r.view(np.float32)[0]
                x = (w * r).astype(np.float32).astype(np.float64)
                worst = max(worst, float(np.max(np.abs(x - exact))))
    assert worst < 3.4e-7 < GUARD


def test_widened_cells_hold_at_most_one_midpoint():
    mid = nf4.midpoints().astype(np.float64)
    assert np.min(np.diff(mid)) > 0.0625 + 4 * GUARD
    for c in range(33):
        lo, hi = (c - 16.5) / 16 - 2 * GUARD, (c - 15.5) / 16 + 2 * GUARD
        assert np.sum((mid >= lo) & (mid <= hi)) <= 1


def test_float_packing_matches_the_byte_order():
    rng = np.random.default_rng(3)
    q = rng.integers(0, 16, size=(1000, 8)).astype(np.float32)
    lo = ((q[:, 0] * 16 + q[:, 1]) + q[:, 3] * 256 + q[:, 2] * 4096 + np.float32(2 ** 23)).astype(np.float32)
    hi = ((q[:, 4] * 16 + q[:, 5]) + q[:, 7] * 256 + q[:, 6] * 4096 + np.float32(2 ** 23)).astype(np.float32)
    word = (hi.view(np.uint32).astype(np.uint64) * 65536 + lo.view(np.uint32) - 0x4B000000) % (1 << 32)
    packed = nf4.pack(q.astype(np.uint8).reshape(1000, 8)).reshape(1000, 4)
    assert np.array_equal(word.astype(np.uint32), packed.view("<u4").ravel())
