"""The facts the GPU encoder's fast path relies on (k_quantize_nf4), checked on
the host against the oracle's definitions -- not the kernel itself, which the
GPU parity tests compare bit for bit:

* with r within 2 ulp of 1/s (s a normal bf16 scale below 2^126, |w| <= s),
  |fl32(w * r) - fl32(w / s)| < 3.4e-7, below the 5e-7 guard;
* the 33 cells rint(16 x + 16), each widened by twice the guard, hold at most
  one level midpoint, and every other midpoint lies wholly below or above;
* away from the guard, the code is the count of midpoints below the cell
  plus one, minus one where the quotient lies below the cell's midpoint
  (the sign bit of d = x - m, never zero there);
* the code word built as the sum of those counts at the eight nibble
  positions minus the sign bits of the eight d's, gathered into place with
  byte permutes (prmt selectors 0x0073, 0x7300, 0x7610), gives the stored
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


def _cells():
    # the encoder's cell table: for cell c, the one midpoint inside the
    # widened cell (4.0 when none) and the count of midpoints below it
    mid = nf4.midpoints().astype(np.float32)
    m_cell, below = np.full(33, 4.0, np.float32), np.zeros(33, np.int64)
    for c in range(33):
        lo, hi = (c - 16.5) / 16 - 2 * GUARD, (c - 15.5) / 16 + 2 * GUARD
        below[c] = np.sum(mid.astype(np.float64) < lo)
        inside = np.nonzero((mid >= lo) & (mid <= hi))[0]
        if inside.size:
            m_cell[c] = mid[inside[0]]
    return m_cell, below


def test_code_is_count_plus_one_minus_sign_bit():
    m_cell, below = _cells()
    mid = nf4.midpoints().astype(np.float32)
    rng = np.random.default_rng(5)
    x = rng.uniform(-1.0, 1.0, 400000).astype(np.float32)
    x = np.concatenate([x, np.float32([-1.0, 1.0, 0.0, -0.0])])
    cell = np.rint(x.astype(np.float64) * 16 + 16).astype(np.int64)
    d = (x - m_cell[cell]).astype(np.float32)
    far = np.abs(d.astype(np.float64)) >= GUARD
    sign = (d.view(np.uint32) >> 31).astype(np.int64)
    code = below[cell] + 1 - sign
    ref = np.searchsorted(mid, x, side="left")       # #{j : m_j < x}
    assert far.mean() > 0.999
    assert np.array_equal(code[far], ref[far])


def _prmt(a, b, sel):
    src = [(int(a) >> (8 * i)) & 0xFF for i in range(4)] + [(int(b) >> (8 * i)) & 0xFF for i in range(4)]
    return sum(src[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def test_word_assembly_matches_the_byte_order():
    rng = np.random.default_rng(3)
    m_cell, below = _cells()
    for _ in range(2000):
        b1 = rng.integers(1, 17, size=8)               # count below + 1 (16 in the top cell)
        s = rng.integers(0, 2, size=8)
        s[b1 == 16] = 1                                  # the top cell has no midpoint: d < 0
        q = b1 - s
        d_bits = [int(rng.integers(0, 1 << 31)) | (int(si) << 31) for si in s]   # any d with that sign
        bsum = 0
        for h in range(4):
            bsum += int(b1[2 * h]) * (16 << (8 * h)) + int(b1[2 * h + 1]) * (1 << (8 * h))
        ev = _prmt(_prmt(d_bits[0], d_bits[2], 0x0073), _prmt(d_bits[4], d_bits[6], 0x7300), 0x7610)
        od = _prmt(_prmt(d_bits[1], d_bits[3], 0x0073), _prmt(d_bits[5], d_bits[7], 0x7300), 0x7610)
        word = (bsum - ((ev >> 3) & 0x10101010) - ((od >> 7) & 0x01010101)) % (1 << 32)
        packed = nf4.pack(q.astype(np.uint8).reshape(1, 8)).reshape(4)
        assert word == int(packed.view("<u4")[0])
