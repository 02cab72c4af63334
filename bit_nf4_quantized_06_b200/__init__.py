"""B200 (sm_100a) QLoRA NF4 + LoRA quantized linear: Python binding.

This module only marshals arguments to the C ABI declared in
``include/qlora.h`` (``libqlora.so``, built in-tree by ``build.py``). Every
step of the computation runs in the library's CUDA kernels; PyTorch supplies
device memory and streams. If the shared library is missing the import
fails: there is no fallback of any kind.

Functions carry the C names:

    qlora_nf4_bytes, qlora_nf4_codebook, qlora_quantize_nf4, qlora_dequantize,
    qlora_workspace_bytes, qlora_fwd_workspace_bytes, qlora_linear_fwd, qlora_linear_fwd_ex,
    qlora_linear_fwd_noalloc, qlora_linear_bwd, qlora_device_status, qlora_status_string, qlora_version,
    qlora_launch_count, qlora_selftest_wait_timeout, qlora_merge_lora, qlora_adamw_step, qlora_adamw_host,
    qlora_adamw_paged, qlora_adamw_staged, qlora_set_gemm_schedule, qlora_get_gemm_schedule
"""

import ctypes
import os

__all__ = [
    "LIB_PATH", "lib", "QloraError", "NF4Weight", "Nf4Struct",
    "qlora_nf4_bytes", "qlora_nf4_codebook", "DQ_U8_256", "DQ_U8_255", "DQ_S8_MID", "qlora_quantize_nf4", "qlora_dequantize",
    "qlora_workspace_bytes", "qlora_fwd_workspace_bytes", "qlora_linear_fwd", "qlora_linear_fwd_ex", "qlora_linear_fwd_noalloc",
    "qlora_linear_bwd",
    "qlora_device_status", "qlora_status_string", "qlora_version", "qlora_launch_count",
    "qlora_selftest_wait_timeout", "qlora_merge_lora", "qlora_adamw_step", "qlora_adamw_host", "qlora_adamw_paged",
    "qlora_adamw_staged", "qlora_set_gemm_schedule", "qlora_get_gemm_schedule",
    "AdamwParams",
    "FWD_AUTO", "FWD_GEMM", "FWD_GEMV", "SCHED_AUTO", "SCHED_DATA_PARALLEL", "SCHED_STREAM_K",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlora.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python bit_nf4_quantized_06_b200/build.py` "
        "(there is no CPU or Python fallback)")

lib = ctypes.CDLL(LIB_PATH)

FWD_AUTO, FWD_GEMM, FWD_GEMV = 0, 1, 2
SCHED_AUTO, SCHED_DATA_PARALLEL, SCHED_STREAM_K = 0, 1, 2
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "SHAPE", 3: "ALIGNMENT", 4: "WORKSPACE",
                5: "UNSUPPORTED_DEVICE", 6: "CUDA", 7: "TIMEOUT"}


class Nf4Struct(ctypes.Structure):
    """Mirror of ``qlora_nf4_t``."""
    _fields_ = [
        ("n_out", ctypes.c_int64),
        ("k_in", ctypes.c_int64),
        ("block", ctypes.c_int32),
        ("dq_group", ctypes.c_int32),
        ("codes", ctypes.c_void_p),
        ("scale_codes", ctypes.c_void_p),
        ("absmax", ctypes.c_void_p),
        ("dq_code", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


_vp, _i64, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
_P = ctypes.POINTER
lib.qlora_nf4_bytes.argtypes = [_i64, _i64, _i32, _P(_sz)]
lib.qlora_nf4_bytes.restype = _sz
lib.qlora_nf4_bytes_ex.argtypes = [_i64, _i64, _i32, _i32, _P(_sz)]
lib.qlora_nf4_bytes_ex.restype = _sz
lib.qlora_nf4_codebook.argtypes = [_P(ctypes.c_float)]
lib.qlora_nf4_codebook.restype = ctypes.c_int
lib.qlora_quantize_nf4.argtypes = [_vp, _P(Nf4Struct), _vp]
lib.qlora_quantize_nf4.restype = ctypes.c_int
lib.qlora_dequantize.argtypes = [_P(Nf4Struct), _vp, _vp]
lib.qlora_dequantize.restype = ctypes.c_int
lib.qlora_workspace_bytes.argtypes = [_i64, _i64, _i64, _i32]
lib.qlora_workspace_bytes.restype = _sz
lib.qlora_fwd_workspace_bytes.argtypes = [_i64, _i64, _i64, _i32]
lib.qlora_fwd_workspace_bytes.restype = _sz
lib.qlora_linear_fwd.argtypes = [_P(Nf4Struct), _vp, _i64, _vp, _vp, _i32, _f32, _vp, _vp, _vp, _sz, _vp]
lib.qlora_linear_fwd.restype = ctypes.c_int
lib.qlora_linear_fwd_ex.argtypes = [_P(Nf4Struct), _vp, _i64, _vp, _vp, _i32, _f32, _vp, _vp, _vp, _sz, _i32,
                                    _vp]
lib.qlora_linear_fwd_ex.restype = ctypes.c_int
lib.qlora_linear_fwd_noalloc.argtypes = [_P(Nf4Struct), _vp, _i64, _vp, _vp, _i32, _f32, _vp, _vp, _vp]
lib.qlora_linear_fwd_noalloc.restype = ctypes.c_int
lib.qlora_linear_bwd.argtypes = [_P(Nf4Struct), _vp, _vp, _vp, _i64, _vp, _vp, _i32, _f32, _vp, _vp, _vp, _vp,
                                 _sz, _vp]
lib.qlora_linear_bwd.restype = ctypes.c_int
lib.qlora_device_status.argtypes = [_vp, _P(ctypes.c_uint32)]
lib.qlora_device_status.restype = ctypes.c_int
lib.qlora_status_string.argtypes = [ctypes.c_int]
lib.qlora_status_string.restype = ctypes.c_char_p
lib.qlora_version.argtypes = []
lib.qlora_version.restype = _i32
class AdamwParams(ctypes.Structure):
    """qlora_adamw_t: lr, beta1, beta2, eps, weight_decay, step (1-based)."""
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int32)]


lib.qlora_adamw_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, ctypes.POINTER(AdamwParams), _vp]
lib.qlora_adamw_step.restype = ctypes.c_int
lib.qlora_adamw_host.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, ctypes.POINTER(AdamwParams)]
lib.qlora_adamw_host.restype = ctypes.c_int
lib.qlora_adamw_paged.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, ctypes.POINTER(AdamwParams), _vp]
lib.qlora_adamw_paged.restype = ctypes.c_int
lib.qlora_adamw_staged.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, ctypes.POINTER(AdamwParams), _vp]
lib.qlora_adamw_staged.restype = ctypes.c_int
lib.qlora_merge_lora.argtypes = [_P(Nf4Struct), _vp, _vp, _i32, _f32, _vp, _vp]
lib.qlora_merge_lora.restype = ctypes.c_int
lib.qlora_selftest_wait_timeout.argtypes = [ctypes.c_uint32, _vp]
lib.qlora_selftest_wait_timeout.restype = ctypes.c_int
lib.qlora_launch_count.argtypes = []
lib.qlora_launch_count.restype = ctypes.c_uint64
lib.qlora_set_gemm_schedule.argtypes = [ctypes.c_int32]
lib.qlora_set_gemm_schedule.restype = ctypes.c_int
lib.qlora_get_gemm_schedule.argtypes = []
lib.qlora_get_gemm_schedule.restype = ctypes.c_int32


class QloraError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = status
        msg = lib.qlora_status_string(status).decode()
        super().__init__(f"{where}: QLORA_ERR_{STATUS_NAMES.get(status, status)} ({msg})")


def _check(status, where):
    if status != 0:
        raise QloraError(status, where)


def _torch():
    import torch
    return torch


def _stream_ptr(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def qlora_version():
    return int(lib.qlora_version())


def qlora_launch_count():
    """Kernels launched by the library in this process so far."""
    return int(lib.qlora_launch_count())


def qlora_set_gemm_schedule(mode):
    """Process-wide schedule of the pair GEMMs: SCHED_AUTO, SCHED_DATA_PARALLEL or SCHED_STREAM_K."""
    _check(lib.qlora_set_gemm_schedule(int(mode)), "qlora_set_gemm_schedule")


def qlora_get_gemm_schedule():
    return int(lib.qlora_get_gemm_schedule())


def qlora_status_string(status):
    return lib.qlora_status_string(int(status)).decode()


# scale codes of the double quantization (qlora_dq_code_t)
DQ_U8_256, DQ_U8_255, DQ_S8_MID = 0, 1, 2


def qlora_nf4_bytes(n_out, k_in, dq_group=256, dq_code=DQ_U8_256):
    """(codes, scale codes, group constants) byte sizes of the stored format."""
    out = (ctypes.c_size_t * 3)()
    total = lib.qlora_nf4_bytes_ex(int(n_out), int(k_in), int(dq_group), int(dq_code), out)
    if total == 0:
        raise QloraError(2, "qlora_nf4_bytes")
    return int(out[0]), int(out[1]), int(out[2])


def qlora_nf4_codebook():
    """The library's 16 fp32 NF4 levels (a list of Python floats)."""
    buf = (ctypes.c_float * 16)()
    _check(lib.qlora_nf4_codebook(buf), "qlora_nf4_codebook")
    return [float(v) for v in buf]


class NF4Weight:
    """Device buffers of one packed NF4 weight. dq=True: codes, 8-bit scale
    codes and the group constants of `dq_code` per 256 blocks (double
    quantization); dq=False: codes and one fp32 scale per 64-weight block (no
    scale codes)."""

    def __init__(self, n_out, k_in, device="cuda", dq=True, dq_code=DQ_U8_256):
        torch = _torch()
        self.dq = bool(dq)
        self.dq_code = int(dq_code) if self.dq else DQ_U8_256
        b_codes, b_q2, b_smax = qlora_nf4_bytes(n_out, k_in, 256 if self.dq else 0, self.dq_code)
        self.n_out, self.k_in = int(n_out), int(k_in)
        self.codes = torch.empty(b_codes, dtype=torch.uint8, device=device)
        self.scale_codes = torch.empty(b_q2, dtype=torch.uint8, device=device)
        self.absmax = torch.empty(b_smax // 4, dtype=torch.float32, device=device)

    def struct(self):
        q2 = self.scale_codes.data_ptr() if self.dq else 0
        return Nf4Struct(self.n_out, self.k_in, 64, 256 if self.dq else 0, self.codes.data_ptr(), q2,
                         self.absmax.data_ptr(), self.dq_code, 0)

    def nbytes(self):
        return self.codes.numel() + self.scale_codes.numel() + 4 * self.absmax.numel()


def qlora_quantize_nf4(w, out=None, stream=None, dq=True, dq_code=DQ_U8_256):
    """Quantize a bf16 CUDA weight [N, K] into an :class:`NF4Weight` (with
    double quantization in scale code `dq_code` unless dq=False, or as `out`
    says)."""
    assert w.is_cuda and w.dim() == 2 and w.is_contiguous()
    q = out if out is not None else NF4Weight(w.shape[0], w.shape[1], device=w.device, dq=dq, dq_code=dq_code)
    s = q.struct()
    _check(lib.qlora_quantize_nf4(_ptr(w), ctypes.byref(s), _stream_ptr(stream)), "qlora_quantize_nf4")
    return q


def qlora_dequantize(q, out=None, stream=None):
    """Restore W_hat [N, K] bf16 from an :class:`NF4Weight`."""
    torch = _torch()
    if out is None:
        out = torch.empty((q.n_out, q.k_in), dtype=torch.bfloat16, device=q.codes.device)
    s = q.struct()
    _check(lib.qlora_dequantize(ctypes.byref(s), _ptr(out), _stream_ptr(stream)), "qlora_dequantize")
    return out


def qlora_workspace_bytes(m, n_out, k_in, r):
    return int(lib.qlora_workspace_bytes(int(m), int(n_out), int(k_in), int(r)))


def qlora_fwd_workspace_bytes(m, n_out, k_in, r):
    return int(lib.qlora_fwd_workspace_bytes(int(m), int(n_out), int(k_in), int(r)))


def _workspace(ws, m, q, r, device):
    torch = _torch()
    need = qlora_workspace_bytes(m, q.n_out, q.k_in, r)
    if ws is None:
        ws = torch.empty(need + 256, dtype=torch.uint8, device=device)
    return ws


def qlora_linear_fwd_ex(q, x, a, b, alpha, path=FWD_AUTO, y=None, u=None, ws=None, stream=None,
                        want_u=True):
    """Forward; returns (y [m, N] bf16, u' [m, r] bf16 or None)."""
    torch = _torch()
    m = x.shape[0]
    r = a.shape[0]
    if y is None:
        y = torch.empty((m, q.n_out), dtype=torch.bfloat16, device=x.device)
    if u is None and want_u:
        u = torch.empty((m, r), dtype=torch.bfloat16, device=x.device)
    ws = _workspace(ws, m, q, r, x.device)
    s = q.struct()
    st = lib.qlora_linear_fwd_ex(ctypes.byref(s), _ptr(x), m, _ptr(a), _ptr(b), r, float(alpha), _ptr(y), _ptr(u),
                                 _ptr(ws), ws.numel(), int(path), _stream_ptr(stream))
    _check(st, "qlora_linear_fwd_ex")
    return y, u


def qlora_linear_fwd(q, x, a, b, alpha, y=None, u=None, ws=None, stream=None, want_u=True):
    """Forward with the library's own path choice; returns (y, u')."""
    torch = _torch()
    m = x.shape[0]
    r = a.shape[0]
    if y is None:
        y = torch.empty((m, q.n_out), dtype=torch.bfloat16, device=x.device)
    if u is None and want_u:
        u = torch.empty((m, r), dtype=torch.bfloat16, device=x.device)
    ws = _workspace(ws, m, q, r, x.device)
    s = q.struct()
    st = lib.qlora_linear_fwd(ctypes.byref(s), _ptr(x), m, _ptr(a), _ptr(b), r, float(alpha), _ptr(y), _ptr(u),
                              _ptr(ws), ws.numel(), _stream_ptr(stream))
    _check(st, "qlora_linear_fwd")
    return y, u


def qlora_linear_fwd_noalloc(q, x, a, b, alpha, y=None, u=None, stream=None, want_u=True):
    """Forward without a caller workspace (library-owned fixed scratch); returns (y, u')."""
    torch = _torch()
    m = x.shape[0]
    r = a.shape[0]
    if y is None:
        y = torch.empty((m, q.n_out), dtype=torch.bfloat16, device=x.device)
    if u is None and want_u:
        u = torch.empty((m, r), dtype=torch.bfloat16, device=x.device)
    s = q.struct()
    st = lib.qlora_linear_fwd_noalloc(ctypes.byref(s), _ptr(x), m, _ptr(a), _ptr(b), r, float(alpha), _ptr(y),
                                      _ptr(u), _stream_ptr(stream))
    _check(st, "qlora_linear_fwd_noalloc")
    return y, u


def qlora_linear_bwd(q, x, u, dy, a, b, alpha, dx=None, da=None, db=None, ws=None, stream=None, want_dx=True):
    """Backward; returns (dX bf16 or None, dA fp32 [r, K], dB fp32 [N, r])."""
    torch = _torch()
    m = x.shape[0]
    r = a.shape[0]
    if dx is None and want_dx:
        dx = torch.empty((m, q.k_in), dtype=torch.bfloat16, device=x.device)
    if da is None:
        da = torch.empty((r, q.k_in), dtype=torch.float32, device=x.device)
    if db is None:
        db = torch.empty((q.n_out, r), dtype=torch.float32, device=x.device)
    ws = _workspace(ws, m, q, r, x.device)
    s = q.struct()
    st = lib.qlora_linear_bwd(ctypes.byref(s), _ptr(x), _ptr(u), _ptr(dy), m, _ptr(a), _ptr(b), r, float(alpha),
                              _ptr(dx), _ptr(da), _ptr(db), _ptr(ws), ws.numel(), _stream_ptr(stream))
    _check(st, "qlora_linear_bwd")
    return dx, da, db


def qlora_device_status(stream=None):
    """(status, bits): synchronises the stream and reads/clears the device status word."""
    bits = ctypes.c_uint32(0)
    st = lib.qlora_device_status(_stream_ptr(stream), ctypes.byref(bits))
    return int(st), int(bits.value)


def qlora_selftest_wait_timeout(limit_us, stream=None):
    """Launch the bounded-wait self test (a wait that nothing completes); the
    timeout shows up in the next qlora_device_status()."""
    _check(lib.qlora_selftest_wait_timeout(int(limit_us), _stream_ptr(stream)), "qlora_selftest_wait_timeout")


def qlora_merge_lora(q, a, b, alpha, out=None, stream=None):
    """bf16(W_hat + (alpha/r) B A) as a new [N, K] bf16 tensor (or into `out`)."""
    torch = _torch()
    r = a.shape[0]
    if out is None:
        out = torch.empty((q.n_out, q.k_in), dtype=torch.bfloat16, device=q.codes.device)
    s = q.struct()
    _check(lib.qlora_merge_lora(ctypes.byref(s), _ptr(a), _ptr(b), r, float(alpha), _ptr(out),
                                _stream_ptr(stream)), "qlora_merge_lora")
    return out


def qlora_adamw_step(master, grad, m, v, step, lr=1e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0,
                     param=None, stream=None):
    """One AdamW step in place on fp32 `master`, `m`, `v` (device tensors or
    pinned host tensors the GPU can address); `param` (bf16, optional)
    receives the bf16 copy. All arguments hold the same number of elements."""
    n = master.numel()
    for t in (grad, m, v) + ((param,) if param is not None else ()):
        if t.numel() != n:
            raise ValueError("qlora_adamw_step: element counts differ")
    hp = AdamwParams(float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay), int(step))
    _check(lib.qlora_adamw_step(_ptr(master), _ptr(param) if param is not None else None, _ptr(grad), _ptr(m),
                                _ptr(v), n, ctypes.byref(hp), _stream_ptr(stream)), "qlora_adamw_step")


def qlora_adamw_staged(master, grad, m_host, v_host, m_stage, v_stage, step, lr=1e-4, betas=(0.9, 0.999),
                       eps=1e-8, weight_decay=0.0, param=None, stream=None):
    """One AdamW step with m, v in pinned host memory, staged through the
    device buffers m_stage, v_stage by copies on `stream` (H2D, update, D2H)."""
    n = master.numel()
    for t in (grad, m_host, v_host, m_stage, v_stage) + ((param,) if param is not None else ()):
        if t.numel() != n:
            raise ValueError("qlora_adamw_staged: element counts differ")
    hp = AdamwParams(float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay), int(step))
    _check(lib.qlora_adamw_staged(_ptr(master), _ptr(param) if param is not None else None, _ptr(grad),
                                  _ptr(m_host), _ptr(v_host), _ptr(m_stage), _ptr(v_stage), n, ctypes.byref(hp),
                                  _stream_ptr(stream)), "qlora_adamw_staged")


def qlora_adamw_host(master, grad, m, v, step, lr=1e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0,
                     param=None):
    """AdamW on the host CPU, in place on CPU fp32 tensors; `param` (CPU
    bf16 tensor, optional) receives the bf16 copy."""
    n = master.numel()
    hp = AdamwParams(float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay), int(step))
    _check(lib.qlora_adamw_host(_ptr(master), _ptr(param) if param is not None else None, _ptr(grad), _ptr(m),
                                _ptr(v), n, ctypes.byref(hp)), "qlora_adamw_host")


def qlora_adamw_paged(grad_dev, master_host, m_host, v_host, grad_host, step, param_dev=None, param_host=None,
                      lr=1e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0, stream=None):
    """Enqueue one paged optimizer step on `stream` (D2H grad, CPU AdamW as a
    stream host function, H2D bf16 adapter). Host tensors must be pinned."""
    n = master_host.numel()
    hp = AdamwParams(float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay), int(step))
    _check(lib.qlora_adamw_paged(_ptr(grad_dev), _ptr(param_dev), _ptr(master_host), _ptr(m_host), _ptr(v_host),
                                 _ptr(grad_host), _ptr(param_host), n, ctypes.byref(hp), _stream_ptr(stream)),
           "qlora_adamw_paged")
