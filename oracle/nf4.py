"""NF4 blockwise quantization with double quantization (test infrastructure only).

Plain numpy statement of the storage format and its round trip. Every step
is an IEEE float32 operation exactly as written below; nothing is fused or
reordered.

Definitions and where they come from:

* Blocks of 64 consecutive weights of the row-major matrix, each with the
  absolute maximum as its scale; weights are divided by the scale and the
  nearest of 16 levels is stored as a 4-bit index; one outlier only touches
  its own block — "48GB GPU Fine-Tuning a 65B Model: Where QLoRA Saves GPU
  Memory", § "Quantization Keeps the Patterns and Reduces Bits per Number".
* Levels at normal-distribution quantiles, dense near zero, with an exact
  zero, in [-1, 1] — same section, and "QLoRA: Efficient Finetuning of
  Quantized LLMs", § "How it works".
* Scales re-quantized to 8-bit codes with one FP32 constant s_max, error at
  most s_max/256, restore as c(q) * q2/256 * s_max — «QLoRA는 어떻게 65B
  모델을 GPU 한 장에 올렸나», § "메모리 회계: 세 겹의 최적화" (Double
  Quantization paragraph and the formula under it).

Readings taken where the pages are silent (each listed in the design notes):

1. Codebook construction: 8 positive levels Phi^-1(delta + j*(1/2 - delta)/8),
   j = 0..7, 7 negative levels -Phi^-1(delta + j*(1/2 - delta)/7), j = 0..6,
   plus 0, with delta = ((1 - 1/30) + (1 - 1/32)) / 2; sorted ascending and
   divided by Phi^-1(delta); computed in float64, rounded to float32.
2. Nearest level is decided on x = fl32(w / s) through the float32 midpoints
   m_j = fl32((c_j + c_{j+1}) / 2); a tie (x == m_j) goes to the lower index.
   A block whose scale is 0 stores index 7 (the exact zero) everywhere.
3. Packing: byte i of a row holds element 2i in its high nibble and element
   2i+1 in its low nibble.
4. Double quantization groups are 256 consecutive blocks of the flattened
   row-major block order (the last group may be short);
   q2 = min(255, rint_even(fl32(256 * s / s_max))) stored unsigned;
   s_hat = fl32(q2 * s_max) * 2^-8; a group whose s_max is 0 stores q2 = 0.
5. Dequantized weight: w_hat = bf16_rne(fl32(c[q] * s_hat)).
"""

import math
from statistics import NormalDist

import numpy as np

from .bf16 import round_f32_to_bf16_bits, bf16_bits_to_f32

BLOCK = 64          # weights per absmax block
DQ_GROUP = 256      # blocks per double-quantization group
ZERO_CODE = 7       # index of the exact-zero level


def codebook_f64():
    """The 16 NF4 levels in float64, ascending (reading 1)."""
    delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))
    phi_inv = NormalDist(0.0, 1.0).inv_cdf
    pos = [phi_inv(delta + j * (0.5 - delta) / 8.0) for j in range(8)]
    neg = [-phi_inv(delta + j * (0.5 - delta) / 7.0) for j in range(7)]
    levels = sorted(pos + neg + [0.0])
    top = phi_inv(delta)
    return np.array([v / top for v in levels], dtype=np.float64)


def codebook():
    """The NF4 codebook as float32 (the table every later step uses)."""
    return codebook_f64().astype(np.float32)


def midpoints(c=None):
    """m_j = fl32((c_j + c_{j+1}) / 2), sum and halving in float64 (reading 2)."""
    if c is None:
        c = codebook()
    c64 = np.asarray(c, dtype=np.float32).astype(np.float64)
    return ((c64[:-1] + c64[1:]) / 2.0).astype(np.float32)


def block_absmax(w):
    """Per-block absolute maximum of a row-major [N, K] float32 matrix (K % 64 == 0).

    Returns float32 [N*K/64] in flattened row-major block order.
    """
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    assert k % BLOCK == 0
    return np.max(np.abs(w.reshape(n * k // BLOCK, BLOCK)), axis=1).astype(np.float32)


def encode(w, absmax):
    """4-bit indices q (uint8, one per weight, [N, K]) for blocks with scales ``absmax``."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    wb = w.reshape(-1, BLOCK)
    s = np.asarray(absmax, dtype=np.float32).reshape(-1, 1)
    zero = (s == 0.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        x = (wb / np.where(zero, np.float32(1.0), s)).astype(np.float32)
    m = midpoints()
    # number of midpoints strictly below x  ==  #{j : x > m_j}
    q = np.searchsorted(m, x.ravel(), side="left").reshape(x.shape).astype(np.uint8)
    q[np.broadcast_to(zero, q.shape)] = ZERO_CODE
    return q.reshape(n, k)


def pack(q):
    """Two indices per byte: element 2i -> high nibble, 2i+1 -> low nibble (reading 3)."""
    q = np.asarray(q, dtype=np.uint8)
    n, k = q.shape
    return ((q[:, 0::2] << 4) | q[:, 1::2]).astype(np.uint8)


def unpack(codes):
    """Inverse of :func:`pack`: [N, K/2] bytes -> [N, K] indices."""
    codes = np.asarray(codes, dtype=np.uint8)
    n, kh = codes.shape
    q = np.empty((n, 2 * kh), dtype=np.uint8)
    q[:, 0::2] = codes >> 4
    q[:, 1::2] = codes & 0x0F
    return q


def n_groups(nb):
    return (nb + DQ_GROUP - 1) // DQ_GROUP


def group_smax(absmax):
    """s_max per group of 256 consecutive blocks (the last group may be short)."""
    a = np.asarray(absmax, dtype=np.float32)
    ng = n_groups(a.size)
    pad = np.zeros(ng * DQ_GROUP, dtype=np.float32)
    pad[: a.size] = a
    return np.max(pad.reshape(ng, DQ_GROUP), axis=1).astype(np.float32)


def double_quantize(absmax):
    """8-bit scale codes and group constants (reading 4).

    Returns (q2 uint8 [nb], smax float32 [ng]).
    """
    a = np.asarray(absmax, dtype=np.float32)
    smax = group_smax(a)
    g = np.arange(a.size) // DQ_GROUP
    sm = smax[g]
    zero = (sm == 0.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = ((np.float32(256.0) * a) / np.where(zero, np.float32(1.0), sm)).astype(np.float32)
    q2 = np.minimum(np.float32(255.0), np.rint(ratio)).astype(np.uint8)
    q2[zero] = 0
    return q2, smax


def restored_scale(q2, smax):
    """s_hat = fl32(q2 * s_max) * 2^-8, per block (float32 [nb])."""
    q2 = np.asarray(q2, dtype=np.uint8)
    g = np.arange(q2.size) // DQ_GROUP
    prod = (q2.astype(np.float32) * np.asarray(smax, dtype=np.float32)[g]).astype(np.float32)
    return (prod * np.float32(1.0 / 256.0)).astype(np.float32)


def quantize(w):
    """Full quantizer: float32 [N, K] (bf16-exact values) -> dict of the stored format.

    Keys: codes uint8 [N, K/2], q2 uint8 [nb], smax float32 [ng], and for
    checking, absmax float32 [nb] and q uint8 [N, K].
    """
    w = np.asarray(w, dtype=np.float32)
    absmax = block_absmax(w)
    q = encode(w, absmax)
    q2, smax = double_quantize(absmax)
    return {"codes": pack(q), "q2": q2, "smax": smax, "absmax": absmax, "q": q}


def dequantize_bits(codes, q2, smax):
    """Restored weights as bf16 bit patterns, uint16 [N, K] (reading 5)."""
    q = unpack(codes)
    n, k = q.shape
    s_hat = restored_scale(q2, smax)
    c = codebook()
    prod = (c[q].reshape(-1, BLOCK) * s_hat.reshape(-1, 1)).astype(np.float32)
    return round_f32_to_bf16_bits(prod).reshape(n, k)


def dequantize(codes, q2, smax):
    """Restored weights as float32 values (each exactly a bf16)."""
    return bf16_bits_to_f32(dequantize_bits(codes, q2, smax))


def dequantize_bits_no_dq(codes, absmax):
    """Restore without double quantization (the 4.5-bit format: one fp32
    scale per block, «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나», § "메모리 회계"):
    w_hat = bf16_rne(fl32(c[q] * s_b)), uint16 [N, K]."""
    q = unpack(codes)
    n, k = q.shape
    c = codebook()
    prod = (c[q].reshape(-1, BLOCK) * np.asarray(absmax, dtype=np.float32).reshape(-1, 1)).astype(np.float32)
    return round_f32_to_bf16_bits(prod).reshape(n, k)


def dequantize_no_dq(codes, absmax):
    return bf16_bits_to_f32(dequantize_bits_no_dq(codes, absmax))


def storage_bytes(n, k, dq=True):
    """Bytes of the stored format: (codes, scale codes or fp32 scales, group constants)."""
    nb = n * k // BLOCK
    if dq:
        return n * k // 2, nb, 4 * n_groups(nb)
    return n * k // 2, 4 * nb, 0


def bits_per_param(n, k, dq=True):
    return 8.0 * sum(storage_bytes(n, k, dq)) / float(n * k)


def max_level_gap(c=None):
    if c is None:
        c = codebook()
    c64 = np.asarray(c, dtype=np.float64)
    return float(np.max(np.diff(c64)))


def normal_cdf(z):
    """Phi via math.erf, independent of NormalDist.inv_cdf (used by the pins)."""
    return 0.5 * (1.0 + math.erf(z / math.sqrt(2.0)))


# --------------------------------------------------------------------------- scale-code variants
#
# The printed double quantization (reading 4) codes each block scale on the
# unsigned grid s_max * q2 / 256. Two further codes of the 8-bit scale, both
# readings of the same paragraph («QLoRA는 어떻게 65B 모델을 GPU 한 장에
# 올렸나», § "메모리 회계: 세 겹의 최적화": 8-bit codes of the scales with a
# 32-bit constant per group, error bounded by the grid step):
#
# "u8_255": the unsigned grid with 255 steps, so the top code is exact:
#     q2    = min(255, rint_even(fl32(fl32(255 s) / s_max)))   (0 if s_max = 0)
#     s_hat = fl32(fl32(q2 s_max) / 255)
#   group data: s_max (one float32); error at most s_max / 510 (+ rounding).
#
# "s8_mid": a signed code centred on the group's mid-range, two float32
#   constants per group:
#     lo, hi = min s, max s over the group
#     mid    = fl32(fl32(lo + hi) / 2),  half = fl32(fl32(hi - lo) / 2)
#     q2     = clamp(rint_even(fl32(fl32(127 fl32(s - mid)) / half)), -127, 127)   (0 if half = 0)
#     s_hat  = fl32(mid + fl32(fl32(q2 half) / 127))
#   q2 stored as int8 (two's complement bytes); error at most half / 254
#   (+ rounding), far below s_max / 256 when the group's scales are close.

DQ_CODES = ("u8_256", "u8_255", "s8_mid")


def group_data_floats(code):
    """float32 constants stored per group of 256 block scales."""
    return 2 if code == "s8_mid" else 1


def double_quantize_code(absmax, code):
    """Scale codes and group data of `code` (see above).

    Returns (q2 uint8 [nb] (int8 bits for s8_mid), gdata float32 [ng] or [ng, 2]).
    """
    if code == "u8_256":
        return double_quantize(absmax)
    a = np.asarray(absmax, dtype=np.float32)
    ng = n_groups(a.size)
    g = np.arange(a.size) // DQ_GROUP
    if code == "u8_255":
        smax = group_smax(a)
        sm = smax[g]
        zero = sm == 0.0
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = ((np.float32(255.0) * a).astype(np.float32) / np.where(zero, np.float32(1.0), sm)).astype(np.float32)
        q2 = np.minimum(np.float32(255.0), np.rint(ratio)).astype(np.uint8)
        q2[zero] = 0
        return q2, smax
    if code == "s8_mid":
        pad_hi = np.full(ng * DQ_GROUP, -np.inf, dtype=np.float32)
        pad_lo = np.full(ng * DQ_GROUP, np.inf, dtype=np.float32)
        pad_hi[: a.size] = a
        pad_lo[: a.size] = a
        hi = pad_hi.reshape(ng, DQ_GROUP).max(axis=1)
        lo = pad_lo.reshape(ng, DQ_GROUP).min(axis=1)
        mid = ((lo + hi).astype(np.float32) * np.float32(0.5)).astype(np.float32)
        half = ((hi - lo).astype(np.float32) * np.float32(0.5)).astype(np.float32)
        t = (a - mid[g]).astype(np.float32)
        hz = half[g] == 0.0
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = ((np.float32(127.0) * t).astype(np.float32) / np.where(hz, np.float32(1.0), half[g])).astype(np.float32)
        q = np.clip(np.rint(ratio), -127, 127).astype(np.int8)
        q[hz] = 0
        return q.view(np.uint8), np.stack([mid, half], axis=1).astype(np.float32)
    raise ValueError(code)


def restored_scale_code(q2, gdata, code):
    """s_hat per block for `code` (float32 [nb])."""
    if code == "u8_256":
        return restored_scale(q2, gdata)
    q2 = np.asarray(q2, dtype=np.uint8)
    g = np.arange(q2.size) // DQ_GROUP
    if code == "u8_255":
        prod = (q2.astype(np.float32) * np.asarray(gdata, dtype=np.float32)[g]).astype(np.float32)
        return (prod / np.float32(255.0)).astype(np.float32)
    if code == "s8_mid":
        gd = np.asarray(gdata, dtype=np.float32).reshape(-1, 2)
        mid, half = gd[g, 0], gd[g, 1]
        qs = q2.view(np.int8).astype(np.float32)
        t = ((qs * half).astype(np.float32) / np.float32(127.0)).astype(np.float32)
        return (mid + t).astype(np.float32)
    raise ValueError(code)


def quantize_code(w, code):
    """Quantizer with scale code `code`: dict with codes, q2, gdata (and absmax, q for checking)."""
    w = np.asarray(w, dtype=np.float32)
    absmax = block_absmax(w)
    q = encode(w, absmax)
    q2, gdata = double_quantize_code(absmax, code)
    return {"codes": pack(q), "q2": q2, "gdata": gdata, "absmax": absmax, "q": q}


def dequantize_bits_code(codes, q2, gdata, code):
    """Restored weights (bf16 bits, uint16 [N, K]) for scale code `code`:
    w_hat = bf16_rne(fl32(c[q] * s_hat))."""
    q = unpack(codes)
    n, k = q.shape
    s_hat = restored_scale_code(q2, gdata, code)
    c = codebook()
    prod = (c[q].reshape(-1, BLOCK) * s_hat.reshape(-1, 1)).astype(np.float32)
    return round_f32_to_bf16_bits(prod).reshape(n, k)


def dequantize_code(codes, q2, gdata, code):
    return bf16_bits_to_f32(dequantize_bits_code(codes, q2, gdata, code))


def storage_bytes_code(n, k, code):
    """Bytes of the stored format with scale code `code`: (codes, scale codes, group data)."""
    nb = n * k // BLOCK
    return n * k // 2, nb, 4 * group_data_floats(code) * n_groups(nb)


def bits_per_param_code(n, k, code):
    return 8.0 * sum(storage_bytes_code(n, k, code)) / float(n * k)
