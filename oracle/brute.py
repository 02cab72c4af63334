"""Literal pure-Python versions for tiny inputs (test infrastructure only).

These loops restate the quantizer and the linear in the most direct way
possible, element by element, so that the vectorised numpy oracle can be
checked against them:

* the scale is the largest |w| of each 64-weight block and the stored index
  is the level nearest to w/scale, found by scanning all 16 levels ("48GB
  GPU Fine-Tuning a 65B Model ...", § "Quantization Keeps the Patterns and
  Reduces Bits per Number");
* the forward and backward are explicit triple loops of the formulas in
  «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나», § "QLoRA의 수식" and
  § "명제 1";
* the merge for export adds s B A to the restored weight and rounds the
  exact sum once to bf16 ("48GB GPU Fine-Tuning a 65B Model ...",
  § "QLoRA Puts the Two Methods in Different Places").

Float32 divisions are evaluated exactly with ``fractions.Fraction`` and
rounded once to binary32 (ties to even), so no numpy or float64
intermediate rounding is involved.
"""

from fractions import Fraction


def f32_round(q):
    """Round an exact rational to the nearest binary32 (ties to even), as a float."""
    q = Fraction(q)
    if q == 0:
        return 0.0
    sign = -1.0 if q < 0 else 1.0
    q = abs(q)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1
    e = max(e, -126)                      # subnormal spacing below 2^-126
    ulp = Fraction(2) ** (e - 23)
    n = q / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * float(fl * ulp)


def f32_div(a, b):
    """fl32(a / b) for float a, b, with a single rounding."""
    return f32_round(Fraction(a) / Fraction(b))


def nearest_level_index(x, levels):
    """argmin_j |x - levels[j]| by a linear scan; ties keep the lower index."""
    best, best_d = 0, abs(x - levels[0])
    for j in range(1, len(levels)):
        d = abs(x - levels[j])
        if d < best_d:
            best, best_d = j, d
    return best


def quantize_rows(rows, levels, block=64):
    """rows: list of lists of floats (bf16-exact). Returns (q rows, absmax list)."""
    q_rows, scales = [], []
    for row in rows:
        qr = []
        for b0 in range(0, len(row), block):
            blk = row[b0:b0 + block]
            s = 0.0
            for v in blk:
                if abs(v) > s:
                    s = abs(v)
            scales.append(s)
            for v in blk:
                if s == 0.0:
                    qr.append(7)
                else:
                    qr.append(nearest_level_index(f32_div(v, s), levels))
        q_rows.append(qr)
    return q_rows, scales


def pack_row(qr):
    out = []
    for i in range(0, len(qr), 2):
        out.append((qr[i] << 4) | qr[i + 1])
    return out


def double_quantize(scales, group=256):
    """Per group: s_max; per block: the 8-bit code of s/s_max on a 1/256 grid."""
    smax, q2 = [], []
    for g0 in range(0, len(scales), group):
        grp = scales[g0:g0 + group]
        m = 0.0
        for s in grp:
            if s > m:
                m = s
        smax.append(m)
        for s in grp:
            if m == 0.0:
                q2.append(0)
            else:
                r = f32_div(256.0 * s, m)
                k = round(r)          # Python round(): half to even
                q2.append(min(255, k))
    return q2, smax


def matmul_nt(a, b):
    """a [M][K], b [N][K] -> a b^T [M][N] by explicit loops (float64)."""
    out = []
    for i in range(len(a)):
        row = []
        for j in range(len(b)):
            acc = 0.0
            for k in range(len(a[i])):
                acc += a[i][k] * b[j][k]
            row.append(acc)
        out.append(row)
    return out


def forward(x, w_hat, a, b, s):
    """y[m][n] = sum_k x[m][k] w_hat[n][k] + s * sum_j (sum_k x[m][k] a[j][k]) b[n][j]."""
    base = matmul_nt(x, w_hat)
    u = matmul_nt(x, a)
    y = []
    for m in range(len(x)):
        row = []
        for n in range(len(w_hat)):
            lora = 0.0
            for j in range(len(a)):
                lora += u[m][j] * b[n][j]
            row.append(base[m][n] + s * lora)
        y.append(row)
    return y


def bf16_round_bits(q):
    """Round an exact rational to the nearest bfloat16 (ties to even); uint16 bits."""
    q = Fraction(q)
    if q == 0:
        return 0
    sign = 0x8000 if q < 0 else 0
    q = abs(q)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1
    if Fraction(2) ** (e + 1) <= q:
        e += 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 7)          # 8 significant bits
    n = q / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    val = fl * ulp                        # exact, representable (or the next binade)
    if val == 0:
        return sign
    ee = val.numerator.bit_length() - val.denominator.bit_length()
    if Fraction(2) ** ee > val:
        ee -= 1
    if ee < -126:                         # subnormal: exponent field 0
        frac = int(val / Fraction(2) ** -133)
        return sign | frac
    frac = int((val / Fraction(2) ** ee - 1) * 128)
    return sign | ((ee + 127) << 7) | frac


def merge(w_hat, a, b, s):
    """bf16 bits of W_hat[n][k] + s * sum_j B[n][j] A[j][k], summed exactly, one rounding."""
    n, k, r = len(w_hat), len(w_hat[0]), len(a)
    sf = Fraction(s)
    out = []
    for i in range(n):
        row = []
        for c in range(k):
            acc = Fraction(0)
            for j in range(r):
                acc += Fraction(b[i][j]) * Fraction(a[j][c])
            row.append(bf16_round_bits(Fraction(w_hat[i][c]) + sf * acc))
        out.append(row)
    return out


def double_quantize_u8_255(scales, group=256):
    """The 255-step unsigned scale code, one exact rounding per operation:
    q2 = min(255, rint_even(fl32(fl32(255 s) / s_max))), s_hat = fl32(fl32(q2 s_max) / 255)."""
    q2, smax_l, s_hat = [], [], []
    for g0 in range(0, len(scales), group):
        grp = scales[g0:g0 + group]
        smax = max(grp)
        smax_l.append(smax)
        for s in grp:
            if smax == 0:
                q = 0
            else:
                ratio = f32_round(Fraction(f32_round(Fraction(255) * Fraction(s))) / Fraction(smax))
                q = min(255, _rint_even(Fraction(ratio)))
            q2.append(q)
            s_hat.append(f32_round(Fraction(f32_round(Fraction(q) * Fraction(smax))) / 255))
    return q2, smax_l, s_hat


def double_quantize_s8_mid(scales, group=256):
    """The signed mid-range scale code, one exact rounding per operation:
    mid = fl32(fl32(lo + hi) / 2), half = fl32(fl32(hi - lo) / 2),
    q2 = clamp(rint_even(fl32(fl32(127 fl32(s - mid)) / half)), -127, 127),
    s_hat = fl32(mid + fl32(fl32(q2 half) / 127))."""
    q2, gdata, s_hat = [], [], []
    for g0 in range(0, len(scales), group):
        grp = scales[g0:g0 + group]
        lo, hi = min(grp), max(grp)
        mid = f32_round(Fraction(f32_round(Fraction(lo) + Fraction(hi))) / 2)
        half = f32_round(Fraction(f32_round(Fraction(hi) - Fraction(lo))) / 2)
        gdata.append((mid, half))
        for s in grp:
            if half == 0:
                q = 0
            else:
                t = f32_round(Fraction(s) - Fraction(mid))
                ratio = f32_round(Fraction(f32_round(127 * Fraction(t))) / Fraction(half))
                q = max(-127, min(127, _rint_even(Fraction(ratio))))
            q2.append(q)
            s_hat.append(f32_round(Fraction(mid) + Fraction(f32_round(Fraction(f32_round(Fraction(q) * Fraction(half))) / 127))))
    return q2, gdata, s_hat


def _rint_even(q):
    """Round a rational to the nearest integer, ties to even."""
    fl = q.numerator // q.denominator
    rem = q - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return int(fl)
