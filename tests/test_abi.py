"""The C-ABI library loads, exports every symbol include/qlora.h declares, and its
host-only logic behaves (no GPU needed: nothing here launches a kernel)."""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import nf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora.h")


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_06_b200 as q
    return q


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"QLORA_API\s+[\w\s\*]*?\b(qlora_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("qlora_quantize_nf4", "qlora_dequantize", "qlora_linear_fwd", "qlora_linear_bwd"):
        assert name in syms


def test_every_declared_symbol_is_exported(q):
    lib = ctypes.CDLL(q.LIB_PATH)
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, missing


def test_codebook_bit_equal_to_oracle(q):
    # the library computes its table by Newton iteration on erfc; the oracle
    # uses statistics.NormalDist: the two fp32 tables must agree bit for bit
    lib_cb = np.array(q.qlora_nf4_codebook(), dtype=np.float32)
    assert np.array_equal(lib_cb.view(np.uint32), nf4.codebook().view(np.uint32))


def test_nf4_bytes_matches_storage_format(q):
    for n, k in ((512, 512), (11008, 4096), (37, 192), (8192, 22016)):
        assert q.qlora_nf4_bytes(n, k) == nf4.storage_bytes(n, k, dq=True)
    with pytest.raises(q.QloraError):
        q.qlora_nf4_bytes(16, 100)      # K % 64 != 0
    with pytest.raises(q.QloraError):
        q.qlora_nf4_bytes(16, 64, 128)  # only groups of 256


def test_status_strings_and_version(q):
    assert q.qlora_status_string(0) == "ok"
    assert "aligned" in q.qlora_status_string(3)
    assert q.qlora_version() >= 100


def test_workspace_bytes_positive_and_monotone(q):
    a = q.qlora_workspace_bytes(16, 512, 512, 8)
    b = q.qlora_workspace_bytes(4096, 11008, 4096, 64)
    assert 0 < a < b
    assert q.qlora_workspace_bytes(16, 512, 512, 0) == 0
    assert q.qlora_workspace_bytes(16, 512, 512, 257) == 0


def test_forward_workspace_within_full_workspace(q):
    for m, n, k, r in [(1, 4096, 4096, 64), (300, 512, 512, 8), (4096, 11008, 4096, 64),
                       (2048, 8192, 22016, 256), (50000, 22016, 8192, 16)]:
        f = q.qlora_fwd_workspace_bytes(m, n, k, r)
        assert 0 < f <= q.qlora_workspace_bytes(m, n, k, r)
    assert q.qlora_fwd_workspace_bytes(16, 512, 512, 0) == 0
    assert q.qlora_fwd_workspace_bytes(-1, 512, 512, 8) == 0


def test_argument_validation_before_any_launch(q):
    lib = q.lib
    s = q.Nf4Struct(512, 512, 64, 256, 0, 0, 0)           # null buffers
    assert lib.qlora_quantize_nf4(ctypes.c_void_p(16), ctypes.byref(s), None) == 1
    s = q.Nf4Struct(512, 500, 64, 256, 16, 16, 16)       # K % 64 != 0
    assert lib.qlora_dequantize(ctypes.byref(s), ctypes.c_void_p(16), None) == 2
    s = q.Nf4Struct(512, 512, 32, 256, 16, 16, 16)       # block must be 64
    assert lib.qlora_dequantize(ctypes.byref(s), ctypes.c_void_p(16), None) == 1
    s = q.Nf4Struct(512, 512, 64, 256, 17, 16, 16)       # misaligned codes
    assert lib.qlora_dequantize(ctypes.byref(s), ctypes.c_void_p(16), None) == 3
    assert lib.qlora_nf4_codebook(None) == 1


def test_merge_argument_validation(q):
    lib = q.lib
    s = q.Nf4Struct(512, 512, 64, 256, 16, 16, 16)
    assert lib.qlora_merge_lora(ctypes.byref(s), ctypes.c_void_p(16), ctypes.c_void_p(16), 0, 16.0,
                                ctypes.c_void_p(16), None) == 2      # r out of range
    assert lib.qlora_merge_lora(ctypes.byref(s), None, ctypes.c_void_p(16), 8, 16.0,
                                ctypes.c_void_p(16), None) == 1      # null A
    assert lib.qlora_merge_lora(ctypes.byref(s), ctypes.c_void_p(24), ctypes.c_void_p(16), 8, 16.0,
                                ctypes.c_void_p(16), None) == 3      # misaligned A


def test_adamw_argument_validation(q):
    lib = q.lib
    hp = q.AdamwParams(1e-3, 0.9, 0.999, 1e-8, 0.0, 0)                 # step must be >= 1
    f = ctypes.c_void_p(16)
    assert lib.qlora_adamw_step(f, None, f, f, f, 10, ctypes.byref(hp), None) == 1
    hp.step = 1
    assert lib.qlora_adamw_step(ctypes.c_void_p(18), None, f, f, f, 10, ctypes.byref(hp), None) == 3
    assert lib.qlora_adamw_step(f, None, f, f, f, 0, ctypes.byref(hp), None) == 0   # nothing to do
    hp.beta1 = 1.0
    assert lib.qlora_adamw_step(f, None, f, f, f, 10, ctypes.byref(hp), None) == 1


def test_nf4_bytes_without_double_quantization(q):
    c, q2, sc = q.qlora_nf4_bytes(4096, 4096, 0)
    assert (c, q2, sc) == (4096 * 4096 // 2, 0, 4 * 4096 * 4096 // 64)
    assert 8 * (c + q2 + sc) / (4096 * 4096) == 4.5
    s = q.Nf4Struct(512, 512, 64, 128, 16, 16, 16)          # dq_group must be 256 or 0
    assert q.lib.qlora_dequantize(ctypes.byref(s), ctypes.c_void_p(16), None) == 1
    s = q.Nf4Struct(512, 512, 64, 0, 16, 0, 16)             # no scale codes needed without DQ
    assert q.lib.qlora_dequantize(ctypes.byref(s), None, None) == 1   # (null output still rejected)


def test_gemm_schedule_setting(q):
    assert q.qlora_get_gemm_schedule() == q.SCHED_AUTO
    with pytest.raises(q.QloraError):
        q.qlora_set_gemm_schedule(3)
    assert q.qlora_get_gemm_schedule() == q.SCHED_AUTO
    try:
        # the workspace size is the same under every setting: it always has
        # room for the stream-K partial slots (one fp32 [128 x 512] per SM)
        # where any setting could use them, also for 64-k-tile reductions
        # that the automatic rule keeps data-parallel
        shapes = [(4096, 4096, 4096, 64), (4096, 22016, 8192, 64), (300, 512, 512, 8)]
        sizes = {}
        for mode in (q.SCHED_AUTO, q.SCHED_STREAM_K, q.SCHED_DATA_PARALLEL):
            q.qlora_set_gemm_schedule(mode)
            sizes[mode] = [q.qlora_workspace_bytes(*sh) for sh in shapes]
            assert q.qlora_fwd_workspace_bytes(4096, 4096, 4096, 64) + 128 * 512 * 4 * 32 <= sizes[mode][0]
            assert q.qlora_fwd_workspace_bytes(4096, 22016, 8192, 64) + 128 * 512 * 4 * 32 <= sizes[mode][1]
        assert sizes[q.SCHED_AUTO] == sizes[q.SCHED_STREAM_K] == sizes[q.SCHED_DATA_PARALLEL]
    finally:
        q.qlora_set_gemm_schedule(q.SCHED_AUTO)


def test_nf4_bytes_of_the_scale_codes(q):
    # the unsigned codes keep one float32 per group of 256 block scales, the
    # signed mid-range code two; the scale codes themselves are one byte each
    n, k = 4096, 4096
    nb, ng = n * k // 64, (n * k // 64 + 255) // 256
    assert q.qlora_nf4_bytes(n, k, 256, q.DQ_U8_256) == (n * k // 2, nb, 4 * ng)
    assert q.qlora_nf4_bytes(n, k, 256, q.DQ_U8_255) == (n * k // 2, nb, 4 * ng)
    assert q.qlora_nf4_bytes(n, k, 256, q.DQ_S8_MID) == (n * k // 2, nb, 8 * ng)
    assert q.lib.qlora_nf4_bytes_ex(n, k, 256, 3, None) == 0          # unknown code
    assert q.lib.qlora_nf4_bytes_ex(n, k, 0, 7, None) > 0             # ignored without DQ
    # rejected before any device work: unknown code, nonzero reserved field
    s = q.Nf4Struct(512, 512, 64, 256, 16, 16, 16, 3, 0)
    assert q.lib.qlora_dequantize(ctypes.byref(s), ctypes.c_void_p(16), None) == 1
    s = q.Nf4Struct(512, 512, 64, 256, 16, 16, 16, 0, 1)
    assert q.lib.qlora_dequantize(ctypes.byref(s), ctypes.c_void_p(16), None) == 1
    assert q.qlora_version() == 10200
